// Confidence-scheduled verify lengths on the GPU, with no host round trip.
//
// QbitAI article "DSpark: ten concepts are enough", section "variable-length
// drafts and hardware-aware scheduling": a confidence head scores each draft
// position's survival; a pre-measured throughput-vs-batch curve then picks
// each request's verify length, entirely on the GPU. Section "speculation is
// not free" (and the Dzhulgakov thread, item 4): time per token = (draft
// time + verify time) / accepted tokens. Section "online drafter
// calibration": sequential temperature scaling of the confidence.
//
// Two kernels:
//   rank  : every CTA recomputes the survival products P[b,j] in fp64 (cheap,
//           bit-identical in every CTA) and ranks its items among all B*K by
//           (P desc, j asc, b asc). Request b's items are a non-increasing
//           list, so the items of request b' that precede a key form a prefix
//           found by binary search; the rank is the sum over b'.
//   final : one CTA: prefix sums S_m of the ranked values, the smallest m*
//           maximising (B + S_m) / T(B + m), per-request counts, row offsets.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace dspark {

namespace {

constexpr int ST = 256;
constexpr int FT = 1024;

__device__ __forceinline__ bool precedes(double Pa, int ja, int ba, double Pb, int jb, int bb) {
  return Pa > Pb || (Pa == Pb && (ja < jb || (ja == jb && ba < bb)));
}

__global__ void __launch_bounds__(ST) schedule_rank_kernel(ScheduleArgs a, int tpi) {
  extern __shared__ double P[];  // [B*K]
  // launched early (programmatic dependent launch): the previous kernel's
  // writes are visible after the wait; the final kernel may launch meanwhile
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int B = a.B, K = a.K, N = B * K;
  for (int b = threadIdx.x; b < B; b += ST) {
    double prod = 1.0;
    for (int j = 0; j < K; ++j) {
      const double x = static_cast<double>(a.conf[b * K + j]) / static_cast<double>(a.temps[j]);
      const double s = 1.0 / (1.0 + exp(-x));
      prod = __dmul_rn(prod, s);
      P[b * K + j] = prod;
      if (blockIdx.x == 0) a.survival[b * K + j] = static_cast<float>(prod);
    }
  }
  __syncthreads();
  const int lane = threadIdx.x % tpi;
  const int groups_per_cta = ST / tpi;
  // the loop bound depends only on `base`, so every thread of a warp takes the
  // same number of trips and the group shuffles stay converged
  for (int base = blockIdx.x * groups_per_cta; base < N; base += gridDim.x * groups_per_cta) {
    const int item = base + threadIdx.x / tpi;
    const bool valid = item < N;
    const int b = valid ? item / K : 0, j = valid ? item - b * K : 0;
    const double p = valid ? P[item] : 0.0;
    int cnt = 0;
    if (valid) {
      for (int bp = lane; bp < B; bp += tpi) {
        int lo = 0, hi = K;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (precedes(P[bp * K + mid], mid, bp, p, j, b)) lo = mid + 1;
          else hi = mid;
        }
        cnt += lo;
      }
    }
    for (int o = tpi / 2; o > 0; o >>= 1) cnt += __shfl_down_sync(0xffffffffu, cnt, o, tpi);
    if (valid && lane == 0) {
      a.rank[item] = cnt;
      a.sorted_P[cnt] = p;
    }
  }
}

__global__ void __launch_bounds__(FT) schedule_final_kernel(ScheduleArgs a) {
  __shared__ double redd[33];
  __shared__ double s_best[32];
  __shared__ int s_bestm[32];
  __shared__ int s_mstar;
  __shared__ long long redl[33];
  const int B = a.B, K = a.K, N = B * K, tid = threadIdx.x;
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the rank kernel's results
  const int M = min(N, a.n_prof - B);
  // prefix sums S_m over the ranked values, m = 1..N
  const int per = (N + FT - 1) / FT;
  const int lo = min(N, tid * per), hi = min(N, lo + per);
  double local = 0.0;
  for (int k = lo; k < hi; ++k) local += a.sorted_P[k];
  double total;
  const double ex = block_exclusive_scan<FT>(local, redd, &total);
  // objective (B + S_m) / T(B + m); T(n) = profile[n - 1]
  double best = -1.0;
  int best_m = 0x7fffffff;
  if (tid == 0) {
    best = static_cast<double>(B) / static_cast<double>(a.profile[B - 1]);
    best_m = 0;
  }
  double S = ex;
  for (int k = lo; k < hi; ++k) {
    S += a.sorted_P[k];
    const int m = k + 1;
    if (m > M) break;
    const double obj = (static_cast<double>(B) + S) / static_cast<double>(a.profile[B + m - 1]);
    if (obj > best || (obj == best && m < best_m)) {
      best = obj;
      best_m = m;
    }
  }
  // block arg-max, ties to the smaller m
  for (int o = 16; o > 0; o >>= 1) {
    const double ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int om = __shfl_xor_sync(0xffffffffu, best_m, o);
    if (ob > best || (ob == best && om < best_m)) {
      best = ob;
      best_m = om;
    }
  }
  if ((tid & 31) == 0) {
    s_best[tid >> 5] = best;
    s_bestm[tid >> 5] = best_m;
  }
  __syncthreads();
  if (tid < 32) {
    best = s_best[tid];
    best_m = s_bestm[tid];
    for (int o = 16; o > 0; o >>= 1) {
      const double ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int om = __shfl_xor_sync(0xffffffffu, best_m, o);
      if (ob > best || (ob == best && om < best_m)) {
        best = ob;
        best_m = om;
      }
    }
    if (tid == 0) s_mstar = best_m;
  }
  __syncthreads();
  const int mstar = s_mstar;
  // per-request lengths and packed row offsets
  const int perb = (B + FT - 1) / FT;
  const int b_lo = min(B, tid * perb), b_hi = min(B, b_lo + perb);
  long long lcount = 0;
  for (int b = b_lo; b < b_hi; ++b) {
    int L = 0;
    for (int j = 0; j < K; ++j) L += (a.rank[b * K + j] < mstar) ? 1 : 0;
    a.verify_len[b] = L;
    lcount += L + 1;
  }
  // exclusive scan of (L_b + 1) in int64
  {
    const int w = tid >> 5, l = tid & 31;
    long long inc = lcount;
    for (int o = 1; o < 32; o <<= 1) {
      const long long n = __shfl_up_sync(0xffffffffu, inc, o);
      if (l >= o) inc += n;
    }
    if (l == 31) redl[w] = inc;
    __syncthreads();
    if (w == 0) {
      long long s = redl[l];
      long long si = s;
      for (int o = 1; o < 32; o <<= 1) {
        const long long n = __shfl_up_sync(0xffffffffu, si, o);
        if (l >= o) si += n;
      }
      redl[l] = si - s;
      if (l == 31) redl[32] = si;
    }
    __syncthreads();
    long long run = redl[w] + inc - lcount;
    for (int b = b_lo; b < b_hi; ++b) {
      a.row_start[b] = run;
      run += a.verify_len[b] + 1;
    }
    if (tid == 0) a.n_tokens[0] = static_cast<int32_t>(redl[32]);
  }
}

}  // namespace

size_t schedule_scratch_bytes(int B, int K) {
  const size_t N = static_cast<size_t>(B) * K;
  return align_up(N * sizeof(int32_t), 256) + align_up(N * sizeof(double), 256);
}

cudaError_t launch_schedule(ScheduleArgs a, char* scratch, cudaStream_t stream) {
  const size_t N = static_cast<size_t>(a.B) * a.K;
  a.rank = reinterpret_cast<int32_t*>(scratch);
  a.sorted_P = reinterpret_cast<double*>(scratch + align_up(N * sizeof(int32_t), 256));
  int tpi = 1;
  while (tpi < 32 && tpi * 8 < a.B) tpi <<= 1;
  const size_t smem = N * sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(schedule_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const long long threads = static_cast<long long>(N) * tpi;
  const int grid = static_cast<int>(std::max<long long>(1, (threads + ST - 1) / ST));
  // both kernels are launched with programmatic stream serialisation, so that
  // each one's launch overlaps the kernel before it; each waits (griddepcontrol)
  // for its predecessor's results before reading anything
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(ST);
  cfg.dynamicSmemBytes = smem;
  e = cudaLaunchKernelEx(&cfg, schedule_rank_kernel, a, tpi);
  if (e == cudaErrorNotSupported) {  // without the early launch
    (void)cudaGetLastError();
    cfg.numAttrs = 0;
    e = cudaLaunchKernelEx(&cfg, schedule_rank_kernel, a, tpi);
  }
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(FT);
  cfg.dynamicSmemBytes = 0;
  e = cudaLaunchKernelEx(&cfg, schedule_final_kernel, a);
  if (e == cudaErrorNotSupported) {
    (void)cudaGetLastError();
    cfg.numAttrs = 0;
    e = cudaLaunchKernelEx(&cfg, schedule_final_kernel, a);
  }
  return e;
}

}  // namespace dspark
