// dspark_schedule_static: the scheduler with its scratch in a static device
// array, for callers that cannot allocate device memory themselves (a
// runtime whose allocator is owned by another framework, code running inside
// stream capture, or an embedding that forbids cudaMalloc on its hot path).
//
// The scratch lives in g_schedule_scratch below: a file-scope __device__
// array of fixed size, so every GPU that loads libdspark holds it (about
// 192 KB) until the process exits. Host code cannot use the array's name as
// a device address; every call looks the address up with cudaGetSymbolAddress
// on the current device.
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kStaticErrBytes = 256;
constexpr size_t kStaticScratchBytes =
    kStaticErrBytes + static_cast<size_t>(DSPARK_STATIC_SCHEDULE_MAX_ITEMS) * (sizeof(int32_t) + sizeof(double));

static __device__ __align__(256) unsigned char g_schedule_scratch[kStaticScratchBytes];

// Device address of g_schedule_scratch on the current device. It is looked
// up on every call (no allocation, and cheap next to the two launches), so a
// context that was torn down and rebuilt, e.g. after cudaDeviceReset, never
// sees a stale address, and a failed lookup is not remembered.
cudaError_t static_scratch(void** out) {
  *out = nullptr;
  return cudaGetSymbolAddress(out, g_schedule_scratch);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" dspark_status dspark_schedule_static(const float* conf_logits, const float* temps,
                                                const float* profile_ms, int n_prof, int B, int K,
                                                int32_t* verify_len, float* survival, int64_t* row_start,
                                                int32_t* n_tokens, dspark_stream_t stream) {
  if (B < 1 || K < 1 || K > dspark::kMaxK || static_cast<long long>(B) * K > DSPARK_STATIC_SCHEDULE_MAX_ITEMS)
    return DSPARK_ERR_INVALID_ARG;
  if (n_prof < B) return DSPARK_ERR_INVALID_ARG;
  const void* ptrs[] = {conf_logits, temps, profile_ms, verify_len, survival, row_start, n_tokens};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return DSPARK_ERR_INVALID_ARG;
  // the largest layout (B*K at the limit) fills the array exactly
  if (kStaticErrBytes + dspark::schedule_scratch_bytes(B, K) > kStaticScratchBytes) return DSPARK_ERR_INVALID_ARG;
  void* base = nullptr;
  if (static_scratch(&base) != cudaSuccess || base == nullptr) return DSPARK_ERR_CUDA;
  char* scratch = static_cast<char*>(base);
  dspark::ScheduleArgs a{};
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
  a.err = reinterpret_cast<unsigned*>(scratch);
  // rank[] and sorted_P[] are rewritten in full by every call (each item gets
  // a rank, and the ranks are a permutation), so nothing needs clearing.
  const cudaError_t e = dspark::launch_schedule(a, scratch + kStaticErrBytes, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
}
