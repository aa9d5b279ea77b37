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
// One kernel:
//   every CTA recomputes the survival products P[b,j] in fp64 (cheap,
//   bit-identical in every CTA) and ranks its items among all B*K by
//   (P desc, j asc, b asc). Request b's items are a non-increasing list, so
//   the items of request b' that precede a key form a prefix found by binary
//   search; the rank is the sum over b'. The grid is at most two CTAs per SM
//   (the products are recomputed once per CTA), of 1024 threads from 2048
//   items on (more threads for the final step's scans) and of 256 below.
//   The last CTA to finish (a device-wide counter, reset for the next call)
//   runs the final step: prefix sums S_m of the ranked values, the smallest m*
//   maximising (B + S_m) / T(B + m), per-request counts and row offsets.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace dspark {

namespace {


__device__ __forceinline__ bool precedes(double Pa, int ja, int ba, double Pb, int jb, int bb) {
  return Pa > Pb || (Pa == Pb && (ja < jb || (ja == jb && ba < bb)));
}

// The final step, by one CTA of NT threads, after every rank is written.
template <int NT>
__device__ void final_step(const ScheduleArgs& a) {
  __shared__ double redd[33];
  __shared__ double s_best[NT / 32];
  __shared__ int s_bestm[NT / 32];
  __shared__ int s_mstar;
  __shared__ long long redl[33];
  const int B = a.B, K = a.K, N = B * K, tid = threadIdx.x;
  const int M = min(N, a.n_prof - B);
  // prefix sums S_m over the ranked values, m = 1..N (read through L2: other
  // CTAs wrote them)
  const int per = (N + NT - 1) / NT;
  const int lo = min(N, tid * per), hi = min(N, lo + per);
  double local = 0.0;
#pragma unroll 8
  for (int k = lo; k < hi; ++k) local += __ldcg(a.sorted_P + k);
  double total;
  const double ex = block_exclusive_scan<NT>(local, redd, &total);
  // objective (B + S_m) / T(B + m); T(n) = profile[n - 1]
  double best = -1.0;
  int best_m = 0x7fffffff;
  if (tid == 0) {
    best = static_cast<double>(B) / static_cast<double>(a.profile[B - 1]);
    best_m = 0;
  }
  double S = ex;
#pragma unroll 8
  for (int k = lo; k < hi; ++k) {
    S += __ldcg(a.sorted_P + k);
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
    best = tid < NT / 32 ? s_best[tid] : -1.0;
    best_m = tid < NT / 32 ? s_bestm[tid] : 0x7fffffff;
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
  const int perb = (B + NT - 1) / NT;
  const int b_lo = min(B, tid * perb), b_hi = min(B, b_lo + perb);
  long long lcount = 0;
  for (int b = b_lo; b < b_hi; ++b) {
    int L = 0;
#pragma unroll 8
    for (int j = 0; j < K; ++j) L += (__ldcg(a.rank + b * K + j) < mstar) ? 1 : 0;
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
      long long s = l < NT / 32 ? redl[l] : 0;
      long long si = s;
      for (int o = 1; o < 32; o <<= 1) {
        const long long n = __shfl_up_sync(0xffffffffu, si, o);
        if (l >= o) si += n;
      }
      if (l < NT / 32) redl[l] = si - s;
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

template <int ST>
__global__ void __launch_bounds__(ST) schedule_kernel(ScheduleArgs a, int tpi) {
  extern __shared__ double Pt[];  // [K][B]: position-major, so that lanes searching consecutive requests read
                                  // consecutive words
  __shared__ int s_last;
  // launched early (programmatic dependent launch): the previous kernel's
  // writes are visible after the wait; the next kernel may launch meanwhile
  // (it waits for this whole grid, the final step included)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int B = a.B, K = a.K, N = B * K;
  for (int b = threadIdx.x; b < B; b += ST) {
    double prod = 1.0;
    for (int j = 0; j < K; ++j) {
      const double x = static_cast<double>(a.conf[b * K + j]) / static_cast<double>(a.temps[j]);
      const double s = 1.0 / (1.0 + exp(-x));
      prod = __dmul_rn(prod, s);
      Pt[j * B + b] = prod;
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
    const double p = valid ? Pt[j * B + b] : 0.0;
    int cnt = 0;
    if (valid) {
      for (int bp = lane; bp < B; bp += tpi) {
        int lo = 0, hi = K;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (precedes(Pt[mid * B + bp], mid, bp, p, j, b)) lo = mid + 1;
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
  // the last CTA to finish runs the final step (its fence and the counter
  // order every CTA's ranks before it reads them)
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(a.done, 1u) == gridDim.x - 1 ? 1 : 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  final_step<ST>(a);
  if (threadIdx.x == 0) *a.done = 0u;  // ready for the next call
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
  a.done = a.err + 4;  // word 4 of the error region: zero between calls
  int tpi = 1;
  while (tpi < 32 && tpi * 8 < a.B) tpi <<= 1;
  const size_t smem = N * sizeof(double);
  const bool big = N >= 2048;
  const int ST = big ? 1024 : 256;
  const void* fn = big ? reinterpret_cast<const void*>(&schedule_kernel<1024>)
                       : reinterpret_cast<const void*>(&schedule_kernel<256>);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long threads = static_cast<long long>(N) * tpi;
  const int grid = static_cast<int>(std::min<long long>(2LL * sms, std::max<long long>(1, (threads + ST - 1) / ST)));
  // launched with programmatic stream serialisation, so that its launch
  // overlaps the kernel before it; it waits (griddepcontrol) for that
  // kernel's results before reading anything
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
  void* args[] = {&a, &tpi};
  e = cudaLaunchKernelExC(&cfg, fn, args);
  if (e == cudaErrorNotSupported) {  // without the early launch
    (void)cudaGetLastError();
    cfg.numAttrs = 0;
    e = cudaLaunchKernelExC(&cfg, fn, args);
  }
  return e;
}

}  // namespace dspark
