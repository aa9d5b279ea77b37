// Semi-autoregressive draft with the low-rank Markov head (CUDA-core path).
//
// QbitAI article "DSpark: ten concepts are enough", section "DSpark = Eagle +
// DFlash": the parallel backbone produces base logits for every position in
// one pass; a light sequential head then injects a prefix-dependent bias left
// to right. Section "a cheaper sequential module: the Markov head": the head
// looks only at the previous token and is factorised at rank 256.
//
// One persistent cooperative kernel runs all K positions. CTA g owns a
// contiguous vocabulary chunk for every request. Per position i:
//   1. z = base + A[t_{i-1}] . Bf for the chunk, written to HBM, with the
//      fp64 sum S_c of exp(z) per request (shift 0; the weight carries the
//      fp32 rounding error of z, found by TwoSum, through exp_fine);
//   2. device-wide arrival (bounded wait);
//   3. request b is selected by CTA b mod G: it combines the G chunk partials
//      in vocabulary order, finds the chunk holding u*W and rescans that chunk
//      of z with the same exp(z - m_c) weights to get t_i;
//   4. device-wide wait for all B tokens (bounded), then position i+1.
// This path serves fp32 factors and is the reference GPU path for bf16; the
// tensor-core path (draft_tc.cu) replaces step 1 for bf16 factors.
#include <algorithm>
#include <cfloat>

#include "common.cuh"
#include "draft_common.cuh"
#include "kernels.h"

namespace dspark {

namespace {

constexpr int DT = 256;  // threads per CTA
constexpr int RB = 8;    // requests per register block

template <bool BF16>
__device__ __forceinline__ float factor_at(const void* p, long long idx) {
  if (BF16) return bf16_bits_to_float(__ldg(reinterpret_cast<const uint16_t*>(p) + idx));
  return __ldg(reinterpret_cast<const float*>(p) + idx);
}

template <bool BF16>
__global__ void __launch_bounds__(DT, 1) draft_generic_kernel(const __grid_constant__ DraftArgs a) {
  extern __shared__ float arow[];  // [RB][r]
  __shared__ double redd[33];
  __shared__ int s_flag;
  __shared__ int s_tok[RB];
  __shared__ double t16[16];
  fill_exp_table(t16, threadIdx.x);
  __syncthreads();
  const int G = gridDim.x, g = blockIdx.x, tid = threadIdx.x;
  const int NU = a.V / 8;
  const int lo = static_cast<int>(static_cast<long long>(g) * NU / G) * 8;
  const int hi = static_cast<int>(static_cast<long long>(g + 1) * NU / G) * 8;
  const int r = a.r;

  for (int i = 0; i < a.K; ++i) {
    // ---- 1. corrected logits and chunk partials, RB requests at a time
    for (int b0 = 0; b0 < a.B; b0 += RB) {
      const int nb = min(RB, a.B - b0);
      if (tid < nb) s_tok[tid] = previous_token(a, b0 + tid, i);
      __syncthreads();
      for (int idx = tid; idx < nb * r; idx += DT) {
        const int bb = idx / r, k = idx - bb * r;
        arow[bb * r + k] = factor_at<BF16>(a.A, static_cast<long long>(s_tok[bb]) * r + k);
      }
      __syncthreads();
      double S[RB];
#pragma unroll
      for (int bb = 0; bb < RB; ++bb) S[bb] = 0.0;
      for (int v = lo + tid; v < hi; v += DT) {
        float acc[RB];
#pragma unroll
        for (int bb = 0; bb < RB; ++bb) acc[bb] = 0.f;
        for (int k = 0; k < r; ++k) {
          const float bf = factor_at<BF16>(a.Bf, static_cast<long long>(k) * a.V + v);
#pragma unroll
          for (int bb = 0; bb < RB; ++bb) acc[bb] = fmaf(arow[bb * r + k], bf, acc[bb]);
        }
#pragma unroll
        for (int bb = 0; bb < RB; ++bb) {
          if (bb < nb) {
            const long long o = (static_cast<long long>(b0 + bb) * a.K + i) * a.V + v;
            const float x0 = a.base[o], y0 = acc[bb];
            const float zz = __fadd_rn(x0, y0);
            const float yv = __fsub_rn(zz, x0);
            const float err = __fadd_rn(__fsub_rn(x0, __fsub_rn(zz, yv)), __fsub_rn(y0, yv));
            a.z[o] = zz;
            S[bb] += exp_fine(zz, err, t16);
          }
        }
      }
#pragma unroll
      for (int bb = 0; bb < RB; ++bb) {
        const double tot = block_sum<DT>(S[bb], redd);
        if (tid == 0 && bb < nb) {
          a.part_m[static_cast<long long>(b0 + bb) * G + g] = 0.f;
          a.part_S[static_cast<long long>(b0 + bb) * G + g] = tot;
        }
      }
      __syncthreads();
    }
    // ---- 2. every chunk of position i is in HBM
    cta_release_add<CtaSync>(&a.sync[2 * i], 1u);
    // ---- 3. select the tokens of my requests
    if (g < a.B) {
      if (!cta_wait_at_least<CtaSync>(&a.sync[2 * i], static_cast<unsigned>(G), a.err, 2u * i, &s_flag)) return;
      for (int b = g; b < a.B; b += G) {
        select_token<DT, CtaSync>(a, b, i, G, 8, t16);
        cta_release_add<CtaSync>(&a.sync[2 * i + 1], 1u);
      }
    }
    // ---- 4. all tokens of position i
    if (i + 1 < a.K) {
      if (!cta_wait_at_least<CtaSync>(&a.sync[2 * i + 1], static_cast<unsigned>(a.B), a.err, 2u * i + 1u, &s_flag))
        return;
    }
  }
}

}  // namespace

size_t draft_tc_extra_bytes(int B, int V, int r);

size_t draft_scratch_bytes(int B, int K, int V, int r) {
  (void)K;
  const size_t G = std::min<size_t>(kMaxGrid, V / 8);
  size_t off = 0;
  off = align_up(off + static_cast<size_t>(B) * G * sizeof(float), 256);
  off = align_up(off + static_cast<size_t>(B) * G * sizeof(double), 256);
  return off + draft_tc_extra_bytes(B, V, r);
}

int draft_grid_size(int V, int sms) { return std::max(1, std::min(std::min(kMaxGrid, sms), V / 8)); }

cudaError_t launch_draft_generic(DraftArgs a, int G, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(RB) * a.r * sizeof(float);
  void* fn = a.bf16 ? reinterpret_cast<void*>(&draft_generic_kernel<true>)
                    : reinterpret_cast<void*>(&draft_generic_kernel<false>);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, DT, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (per_sm < 1 || G > per_sm * sms) return cudaErrorCooperativeLaunchTooLarge;
  void* args[] = {&a};
  return cudaLaunchCooperativeKernel(fn, dim3(G), dim3(DT), args, smem, stream);
}

}  // namespace dspark
