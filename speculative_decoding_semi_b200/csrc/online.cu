// Steps that run between rounds on the device, so that rounds can follow one
// another with no host involvement: the online calibration of the sequential
// temperatures from the round's outcome, and the next round's anchor tokens.
//
// QbitAI article "DSpark: ten concepts are enough", section "online drafter
// calibration": the confidence head's scores are post-processed by sequential
// temperature scaling, and the calibration runs online, correcting itself
// from the acceptance observed on the current workload. Position j's
// temperature is the scale of the logistic survival model sigmoid(c / T_j);
// each round takes one step along the mean gradient of the negative
// log-likelihood of that round's outcomes with respect to theta_j = 1 / T_j,
// over the requests that reached position j (drafts 1..j-1 accepted) and
// verified it (j <= L_b), the outcome being whether draft j was accepted.
// Section "variable-length drafts and hardware-aware scheduling": the whole
// scheduling logic runs on the GPU without the CPU.
#include <algorithm>

#include "common.cuh"

namespace dspark {
namespace {

constexpr int kCalibThreads = 32 * kMaxK;  // one warp per draft position

struct CalibArgs {
  const float* conf;
  const int32_t* verify_len;
  const int32_t* accepted;
  int B, K;
  double eta, t_min, t_max;
  float* temps;
  unsigned* err;
};

__global__ void __launch_bounds__(kCalibThreads) calibrate_kernel(CalibArgs a) {
  const int j = threadIdx.x >> 5, lane = threadIdx.x & 31;  // position j + 1
  if (j >= a.K) return;
  const double theta = 1.0 / static_cast<double>(a.temps[j]);
  double g = 0.0;
  int n = 0;
  for (int b = lane; b < a.B; b += 32) {
    const int L = a.verify_len[b], acc = a.accepted[b];
    if (L < 0 || L > a.K || acc < 0 || acc > L) {
      if (j == 0) set_error(a.err, DSPARK_ERR_DEVICE_ASSERT, 0x50000000u | static_cast<unsigned>(b));
      continue;
    }
    if (acc >= j && L >= j + 1) {
      const double c = static_cast<double>(a.conf[static_cast<long long>(b) * a.K + j]);
      const double s = 1.0 / (1.0 + exp(-c * theta));
      const double y = acc >= j + 1 ? 1.0 : 0.0;
      g += (s - y) * c;
      ++n;
    }
  }
  g = warp_sum(g);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
  if (lane == 0 && n > 0) {
    const double th = theta - a.eta * g / static_cast<double>(n);
    const double T = th > 0.0 ? 1.0 / th : a.t_max;
    a.temps[j] = static_cast<float>(fmin(fmax(T, a.t_min), a.t_max));
  }
}

__global__ void advance_anchor_kernel(const int32_t* out_tokens, const int32_t* n_out, int B, int K, int32_t* anchor,
                                      unsigned* err) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int n = n_out[b];
  if (n < 1 || n > K + 1) {
    set_error(err, DSPARK_ERR_DEVICE_ASSERT, 0x60000000u | static_cast<unsigned>(b));
    return;
  }
  anchor[b] = out_tokens[static_cast<long long>(b) * (K + 1) + n - 1];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace dspark

using namespace dspark;

extern "C" {

dspark_status dspark_calibrate(const float* conf_logits, const int32_t* verify_len, const int32_t* accepted, int B,
                               int K, float eta, float t_min, float t_max, float* temps, void* workspace,
                               size_t ws_bytes, dspark_stream_t stream) {
  if (B < 1 || B > kMaxB || K < 1 || K > kMaxK) return DSPARK_ERR_INVALID_ARG;
  if (!(eta >= 0.f) || !(t_min > 0.f) || !(t_max >= t_min)) return DSPARK_ERR_INVALID_ARG;
  const void* ptrs[] = {conf_logits, verify_len, accepted, temps, workspace};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return DSPARK_ERR_INVALID_ARG;
  if (ws_bytes < kScratchOffset) return DSPARK_ERR_INVALID_ARG;
  CalibArgs a{};
  a.conf = conf_logits;
  a.verify_len = verify_len;
  a.accepted = accepted;
  a.B = B;
  a.K = K;
  a.eta = eta;
  a.t_min = t_min;
  a.t_max = t_max;
  a.temps = temps;
  a.err = reinterpret_cast<unsigned*>(static_cast<char*>(workspace) + kErrOffset);
  calibrate_kernel<<<1, 32 * K, 0, reinterpret_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError() == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
}

dspark_status dspark_advance_anchor(const int32_t* out_tokens, const int32_t* n_out, int B, int K, int32_t* anchor,
                                    void* workspace, size_t ws_bytes, dspark_stream_t stream) {
  if (B < 1 || B > kMaxB || K < 1 || K > kMaxK) return DSPARK_ERR_INVALID_ARG;
  const void* ptrs[] = {out_tokens, n_out, anchor, workspace};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return DSPARK_ERR_INVALID_ARG;
  if (ws_bytes < kScratchOffset) return DSPARK_ERR_INVALID_ARG;
  unsigned* err = reinterpret_cast<unsigned*>(static_cast<char*>(workspace) + kErrOffset);
  advance_anchor_kernel<<<(B + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(out_tokens, n_out, B, K,
                                                                                          anchor, err);
  return cudaGetLastError() == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
}

}  // extern "C"
