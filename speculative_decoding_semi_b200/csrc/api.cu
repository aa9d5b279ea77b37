// C ABI of libdspark: argument validation, workspace layout and launches.
// Every entry point checks its arguments before launching anything, enqueues
// work on the caller's stream and returns without synchronising.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace dspark {
cudaError_t launch_draft_generic(DraftArgs a, int G, cudaStream_t stream);
int draft_grid_size(int V, int sms);
bool draft_tc_supported(const DraftArgs& a);
int draft_tc_grid(int V, int sms);
cudaError_t launch_draft_tc(DraftArgs a, int G, unsigned* sync, char* extra, cudaStream_t stream);
size_t image_bytes(int B, int r);
}  // namespace dspark

using namespace dspark;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool sizes_ok(int B, int K, int V) {
  return B >= 1 && B <= kMaxB && K >= 1 && K <= kMaxK && V >= 8 && V <= kMaxV && (V % 8) == 0;
}

// Scratch layout after kScratchOffset: schedule | verify | draft.
size_t schedule_region(int B, int K) { return align_up(schedule_scratch_bytes(B, K), 256); }
size_t verify_region(int B, int K, int V) { return align_up(verify_scratch_bytes(B, K, V), 256); }
size_t scratch_bytes(int B, int K, int V, int r) {
  return schedule_region(B, K) + verify_region(B, K, V) + align_up(draft_scratch_bytes(B, K, V, r), 256);
}

// The draft's part of the scratch: part_m [B][gmax] f32, part_S [B][gmax] f64,
// then the tensor-core kernel's extra (operand image, unit sums, RNN state).
struct DraftScratch {
  float* part_m;
  double* part_S;
  char* extra;
};
DraftScratch draft_scratch(char* ws, int B, int K, int V) {
  char* scratch = ws + kScratchOffset + schedule_region(B, K) + verify_region(B, K, V);
  const size_t gmax = std::min<size_t>(kMaxGrid, V / 8);
  const size_t m_bytes = align_up(static_cast<size_t>(B) * gmax * sizeof(float), 256);
  const size_t s_bytes = align_up(static_cast<size_t>(B) * gmax * sizeof(double), 256);
  return DraftScratch{reinterpret_cast<float*>(scratch), reinterpret_cast<double*>(scratch + m_bytes),
                      scratch + m_bytes + s_bytes};
}

// Shapes of the tensor-core kernels (variant B and the RNN head).
bool tc_shape(dspark_dtype factor_dtype, int r, int B, int V) {
  return factor_dtype == DSPARK_BF16 && r % 64 == 0 && r <= 256 && V % 32 == 0 && B <= 512;
}

dspark_status from_cuda(cudaError_t e) { return e == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA; }

}  // namespace

extern "C" {

size_t dspark_workspace_bytes(int B, int K, int V, int r) {
  if (!sizes_ok(B, K, V) || r < 1 || r > kMaxR) return 0;
  return kScratchOffset + align_up(scratch_bytes(B, K, V, r), 256);
}

dspark_status dspark_workspace_init(void* workspace, size_t ws_bytes, dspark_stream_t stream) {
  if (workspace == nullptr || ws_bytes < kScratchOffset || !aligned16(workspace)) return DSPARK_ERR_INVALID_ARG;
  return from_cuda(cudaMemsetAsync(workspace, 0, ws_bytes, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// Variant A (z) or variant B (z == nullptr: base_logits, op_rows, Bf, r).
dspark_status verify_call(const float* target_logits, const int64_t* row_start, const float* z,
                          const float* base_logits, const uint16_t* op_rows, const void* Bf, int r,
                          const double* lse_q, const float* q_tok, const int32_t* draft_tokens,
                          const int32_t* verify_len, const float* u_accept, const float* u_resample, int B, int K,
                          int V, int32_t* accepted, int32_t* out_tokens, int32_t* n_out, void* workspace,
                          size_t ws_bytes, dspark_stream_t stream) {
  if (!sizes_ok(B, K, V)) return DSPARK_ERR_INVALID_ARG;
  const void* ptrs[] = {target_logits, row_start, lse_q, q_tok, draft_tokens, verify_len,
                        u_accept, u_resample, accepted, out_tokens, n_out, workspace};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return DSPARK_ERR_INVALID_ARG;
  if (z != nullptr && !aligned16(z)) return DSPARK_ERR_INVALID_ARG;
  if (ws_bytes < kScratchOffset + schedule_region(B, K) + verify_region(B, K, V)) return DSPARK_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  VerifyArgs a{};
  a.target = target_logits;
  a.row_start = row_start;
  a.z = z;
  a.base = base_logits;
  a.op_rows = op_rows;
  a.Bf = Bf;
  a.r = r;
  if (z == nullptr) {
    // the residual kernel's sums reuse the draft's scratch (slice sums, unit sums)
    const DraftScratch ds = draft_scratch(ws, B, K, V);
    a.res_part = ds.part_S;
    a.res_unit = reinterpret_cast<double*>(ds.extra + image_bytes(B, r));
    a.res_image = reinterpret_cast<uint8_t*>(ds.extra);
  }
  a.lse_q = lse_q;
  a.q_tok = q_tok;
  a.tokens = draft_tokens;
  a.verify_len = verify_len;
  a.u_accept = u_accept;
  a.u_resample = u_resample;
  a.B = B;
  a.K = K;
  a.V = V;
  a.accepted = accepted;
  a.out_tokens = out_tokens;
  a.n_out = n_out;
  a.err = reinterpret_cast<unsigned*>(ws + kErrOffset);
  return from_cuda(launch_verify(a, ws + kScratchOffset + schedule_region(B, K), reinterpret_cast<cudaStream_t>(stream)));
}

// The Markov head (W == nullptr) or the RNN head (W = its recurrent weight);
// variant A writes z, variant B (z == nullptr) writes op_rows instead.
dspark_status draft_call(const float* base_logits, const void* A, const void* W, const void* Bf,
                         dspark_dtype factor_dtype, int r, const int32_t* anchor, const float* u_draft, int B, int K,
                         int V, int32_t* draft_tokens, float* q_tok, double* lse_q, float* z, uint16_t* op_rows,
                         void* workspace, size_t ws_bytes, dspark_stream_t stream) {
  if (!sizes_ok(B, K, V) || r < 1 || r > kMaxR) return DSPARK_ERR_INVALID_ARG;
  if (factor_dtype != DSPARK_F32 && factor_dtype != DSPARK_BF16) return DSPARK_ERR_INVALID_ARG;
  const void* out = z != nullptr ? static_cast<const void*>(z) : static_cast<const void*>(op_rows);
  const void* ptrs[] = {base_logits, A, Bf, anchor, u_draft, draft_tokens, q_tok, lse_q, out, workspace};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return DSPARK_ERR_INVALID_ARG;
  if (W != nullptr && !aligned16(W)) return DSPARK_ERR_INVALID_ARG;
  if (ws_bytes < dspark_workspace_bytes(B, K, V, r)) return DSPARK_ERR_INVALID_ARG;
  if (2u * K * sizeof(unsigned) > kSyncBytes) return DSPARK_ERR_INVALID_ARG;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSPARK_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DSPARK_ERR_CUDA;
  DraftArgs a{};
  a.base = base_logits;
  a.A = A;
  a.Bf = Bf;
  a.W = W;
  a.bf16 = factor_dtype == DSPARK_BF16;
  a.r = r;
  a.anchor = anchor;
  a.u = u_draft;
  a.B = B;
  a.K = K;
  a.V = V;
  a.tokens = draft_tokens;
  a.q_tok = q_tok;
  a.lse_q = lse_q;
  a.z = z;
  a.op_rows = z == nullptr ? op_rows : nullptr;
  a.err = reinterpret_cast<unsigned*>(ws + kErrOffset);
  a.sync = reinterpret_cast<unsigned*>(ws + kSyncOffset);
  // bf16 factors with r % 64 == 0 (r <= 256) and V % 32 == 0 take the
  // tensor-core kernel; other shapes and fp32 factors the CUDA-core kernel
  // (which has the Markov head only)
  const bool tc = draft_tc_supported(a);
  if ((W != nullptr || z == nullptr) && !tc) return DSPARK_ERR_UNSUPPORTED;
  const int G = tc ? draft_tc_grid(V, sms) : draft_grid_size(V, sms);
  const DraftScratch ds = draft_scratch(ws, B, K, V);
  a.part_m = ds.part_m;
  a.part_S = ds.part_S;
  char* extra = ds.extra;

  cudaError_t e = cudaMemsetAsync(a.sync, 0, kSyncBytes, s);
  if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  return from_cuda(tc ? launch_draft_tc(a, G, a.sync, extra, s) : launch_draft_generic(a, G, s));
}

}  // namespace

extern "C" {

dspark_status dspark_markov_draft(const float* base_logits, const void* A, const void* Bf,
                                  dspark_dtype factor_dtype, int r, const int32_t* anchor,
                                  const float* u_draft, int B, int K, int V, int32_t* draft_tokens,
                                  float* q_tok, double* lse_q, float* z, void* workspace,
                                  size_t ws_bytes, dspark_stream_t stream) {
  if (z == nullptr) return DSPARK_ERR_INVALID_ARG;
  return draft_call(base_logits, A, nullptr, Bf, factor_dtype, r, anchor, u_draft, B, K, V, draft_tokens, q_tok,
                    lse_q, z, nullptr, workspace, ws_bytes, stream);
}

dspark_status dspark_rnn_draft(const float* base_logits, const void* A, const void* W, const void* Bf,
                               dspark_dtype factor_dtype, int r, const int32_t* anchor, const float* u_draft, int B,
                               int K, int V, int32_t* draft_tokens, float* q_tok, double* lse_q, float* z,
                               void* workspace, size_t ws_bytes, dspark_stream_t stream) {
  if (W == nullptr || z == nullptr) return DSPARK_ERR_INVALID_ARG;
  return draft_call(base_logits, A, W, Bf, factor_dtype, r, anchor, u_draft, B, K, V, draft_tokens, q_tok, lse_q, z,
                    nullptr, workspace, ws_bytes, stream);
}

dspark_status dspark_markov_draft_b(const float* base_logits, const void* A, const void* Bf,
                                    dspark_dtype factor_dtype, int r, const int32_t* anchor,
                                    const float* u_draft, int B, int K, int V, int32_t* draft_tokens,
                                    float* q_tok, double* lse_q, uint16_t* op_rows, void* workspace,
                                    size_t ws_bytes, dspark_stream_t stream) {
  if (op_rows == nullptr) return DSPARK_ERR_INVALID_ARG;
  if (sizes_ok(B, K, V) && r >= 1 && !tc_shape(factor_dtype, r, B, V)) return DSPARK_ERR_UNSUPPORTED;
  return draft_call(base_logits, A, nullptr, Bf, factor_dtype, r, anchor, u_draft, B, K, V, draft_tokens, q_tok,
                    lse_q, nullptr, op_rows, workspace, ws_bytes, stream);
}

dspark_status dspark_rnn_draft_b(const float* base_logits, const void* A, const void* W, const void* Bf,
                                 dspark_dtype factor_dtype, int r, const int32_t* anchor, const float* u_draft,
                                 int B, int K, int V, int32_t* draft_tokens, float* q_tok, double* lse_q,
                                 uint16_t* op_rows, void* workspace, size_t ws_bytes, dspark_stream_t stream) {
  if (W == nullptr || op_rows == nullptr) return DSPARK_ERR_INVALID_ARG;
  if (sizes_ok(B, K, V) && r >= 1 && !tc_shape(factor_dtype, r, B, V)) return DSPARK_ERR_UNSUPPORTED;
  return draft_call(base_logits, A, W, Bf, factor_dtype, r, anchor, u_draft, B, K, V, draft_tokens, q_tok, lse_q,
                    nullptr, op_rows, workspace, ws_bytes, stream);
}

dspark_status dspark_schedule(const float* conf_logits, const float* temps, const float* profile_ms,
                              int n_prof, int B, int K, int32_t* verify_len, float* survival,
                              int64_t* row_start, int32_t* n_tokens, void* workspace, size_t ws_bytes,
                              dspark_stream_t stream) {
  if (B < 1 || B > kMaxB || K < 1 || K > kMaxK || static_cast<long long>(B) * K > kMaxScheduleItems)
    return DSPARK_ERR_INVALID_ARG;
  if (n_prof < B) return DSPARK_ERR_INVALID_ARG;
  const void* ptrs[] = {conf_logits, temps, profile_ms, verify_len, survival, row_start, n_tokens, workspace};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return DSPARK_ERR_INVALID_ARG;
  if (ws_bytes < kScratchOffset + schedule_scratch_bytes(B, K)) return DSPARK_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  ScheduleArgs a{};
  a.conf = conf_logits;
  a.temps = temps;
  a.profile = profile_ms;
  a.n_prof = n_prof;
  a.B = B;
  a.K = K;
  a.verify_len = verify_len;
  a.survival = survival;
  a.row_start = row_start;
  a.n_tokens = n_tokens;
  a.err = reinterpret_cast<unsigned*>(ws + kErrOffset);
  return from_cuda(launch_schedule(a, ws + kScratchOffset, reinterpret_cast<cudaStream_t>(stream)));
}

dspark_status dspark_verify(const float* target_logits, const int64_t* row_start, const float* z,
                            const double* lse_q, const float* q_tok, const int32_t* draft_tokens,
                            const int32_t* verify_len, const float* u_accept, const float* u_resample,
                            int B, int K, int V, int32_t* accepted, int32_t* out_tokens, int32_t* n_out,
                            void* workspace, size_t ws_bytes, dspark_stream_t stream) {
  if (z == nullptr) return DSPARK_ERR_INVALID_ARG;
  return verify_call(target_logits, row_start, z, nullptr, nullptr, nullptr, 0, lse_q, q_tok, draft_tokens,
                     verify_len, u_accept, u_resample, B, K, V, accepted, out_tokens, n_out, workspace, ws_bytes,
                     stream);
}

dspark_status dspark_verify_b(const float* target_logits, const int64_t* row_start, const float* base_logits,
                              const uint16_t* op_rows, const void* Bf, int r, const double* lse_q,
                              const float* q_tok, const int32_t* draft_tokens, const int32_t* verify_len,
                              const float* u_accept, const float* u_resample, int B, int K, int V,
                              int32_t* accepted, int32_t* out_tokens, int32_t* n_out, void* workspace,
                              size_t ws_bytes, dspark_stream_t stream) {
  if (base_logits == nullptr || op_rows == nullptr || Bf == nullptr) return DSPARK_ERR_INVALID_ARG;
  if (!aligned16(base_logits) || !aligned16(op_rows) || !aligned16(Bf)) return DSPARK_ERR_INVALID_ARG;
  if (r < 1 || r > kMaxR) return DSPARK_ERR_INVALID_ARG;
  if (sizes_ok(B, K, V) && !tc_shape(DSPARK_BF16, r, B, V)) return DSPARK_ERR_UNSUPPORTED;
  if (ws_bytes < dspark_workspace_bytes(B, K, V, r)) return DSPARK_ERR_INVALID_ARG;
  return verify_call(target_logits, row_start, nullptr, base_logits, op_rows, Bf, r, lse_q, q_tok, draft_tokens,
                     verify_len, u_accept, u_resample, B, K, V, accepted, out_tokens, n_out, workspace, ws_bytes,
                     stream);
}

dspark_status dspark_set_wait_budget(void* workspace, uint32_t microseconds, dspark_stream_t stream) {
  if (workspace == nullptr || !aligned16(workspace)) return DSPARK_ERR_INVALID_ARG;
  const uint32_t v = microseconds;  // pageable source: staged before the call returns
  return from_cuda(cudaMemcpyAsync(static_cast<char*>(workspace) + kErrOffset + 2 * sizeof(unsigned), &v,
                                   sizeof(v), cudaMemcpyHostToDevice, reinterpret_cast<cudaStream_t>(stream)));
}

dspark_status dspark_inject_stall(void* workspace, dspark_inject where, uint32_t cta, dspark_stream_t stream) {
  if (workspace == nullptr || !aligned16(workspace)) return DSPARK_ERR_INVALID_ARG;
  if (where != DSPARK_INJECT_NONE && where != DSPARK_INJECT_DRAFT_SLICE_SUMS && where != DSPARK_INJECT_VERIFY_BARRIER &&
      where != DSPARK_INJECT_RESIDUAL_SLICE_SUMS)
    return DSPARK_ERR_INVALID_ARG;
  if (cta >= (1u << 24)) return DSPARK_ERR_INVALID_ARG;
  const uint32_t v = where == DSPARK_INJECT_NONE ? 0u : ((static_cast<uint32_t>(where) << 24) | cta);
  return from_cuda(cudaMemcpyAsync(static_cast<char*>(workspace) + kErrOffset + 3 * sizeof(unsigned), &v,
                                   sizeof(v), cudaMemcpyHostToDevice, reinterpret_cast<cudaStream_t>(stream)));
}

dspark_status dspark_read_device_error(void* workspace, dspark_stream_t stream, uint32_t* detail) {
  if (workspace == nullptr || !aligned16(workspace)) return DSPARK_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned host[2] = {0, 0};
  if (cudaMemcpyAsync(host, workspace, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return DSPARK_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DSPARK_ERR_CUDA;
  if (detail) *detail = host[1];
  if (host[0] != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(host), s) != cudaSuccess) return DSPARK_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return DSPARK_ERR_CUDA;
  }
  return static_cast<dspark_status>(host[0]);
}

const char* dspark_status_string(dspark_status status) {
  switch (status) {
    case DSPARK_OK: return "ok";
    case DSPARK_ERR_INVALID_ARG: return "invalid argument";
    case DSPARK_ERR_UNSUPPORTED: return "unsupported";
    case DSPARK_ERR_CUDA: return "CUDA error";
    case DSPARK_ERR_TIMEOUT: return "device-wide wait timed out";
    case DSPARK_ERR_DEVICE_ASSERT: return "device-side check failed";
  }
  return "unknown status";
}

}  // extern "C"
