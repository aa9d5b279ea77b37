// Device helpers shared by the draft, schedule and verify kernels:
// the workspace error word, bounded device-wide waits, block reductions and
// scans in fp32/fp64, and the workspace layout.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/dspark.h"

namespace dspark {

// ---------------------------------------------------------------- limits
constexpr int kMaxB = 65536;
constexpr int kMaxK = 32;
constexpr int kMaxV = 1 << 24;
constexpr int kMaxR = 512;
constexpr int kMaxScheduleItems = 16384;
constexpr int kMaxGrid = 256;        // CTAs of the persistent draft kernel (>= SM count)

// -------------------------------------------------------- workspace layout
// [0, 256)      error word: u32 code, u32 detail
// [256, 4352)   counters of the device-wide waits (cleared by every draft launch)
// [4352, ...)   schedule arrays, then the verify arrays, then the draft
//               partials (disjoint, so a round's calls never overwrite each
//               other's data).
constexpr size_t kErrOffset = 0;
constexpr size_t kSyncOffset = 256;
constexpr size_t kSyncBytes = 4096;
constexpr size_t kScratchOffset = kSyncOffset + kSyncBytes;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ------------------------------------------------------------ error word
// Words of the workspace's first 256 bytes: [0] status code, [1] detail,
// [2] wait budget in microseconds (0 = kWaitBudgetNs), [3] stall injection
// (a test hook: DSPARK_INJECT_* << 24 | CTA index, 0 = none).
constexpr unsigned kWaitIterLimit = 1u << 26;           // spins before a wait gives up
constexpr unsigned long long kWaitBudgetNs = 1000000000ull;  // 1 s of device time

__device__ __forceinline__ void set_error(unsigned* err, unsigned code, unsigned detail) {
  if (atomicCAS(err, 0u, code) == 0u) atomicExch(err + 1, detail);
}

__device__ __forceinline__ unsigned error_code(const unsigned* err) {
  return *reinterpret_cast<const volatile unsigned*>(err);
}

// Time after which a device-wide wait of a kernel using this workspace gives up.
__device__ __forceinline__ unsigned long long wait_budget_ns(const unsigned* err) {
  const unsigned us = *reinterpret_cast<const volatile unsigned*>(err + 2);
  return us ? static_cast<unsigned long long>(us) * 1000ull : kWaitBudgetNs;
}

// True when the test hook asks CTA `cta` to skip the publish of kind `kind`.
__device__ __forceinline__ bool injected_stall(const unsigned* err, unsigned kind, unsigned cta) {
  return *reinterpret_cast<const volatile unsigned*>(err + 3) == ((kind << 24) | cta);
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Atomic add with acquire-release semantics at gpu scope; returns the old value.
__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ void red_release_gpu_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Spin (one thread) until *ctr >= target. Gives up when the error word is set
// by anyone, after kWaitIterLimit polls, or after kWaitBudgetNs; in the last
// two cases it records DSPARK_ERR_TIMEOUT with `where`. Returns true on success.
static __device__ __noinline__ bool wait_at_least(const unsigned* ctr, unsigned target, unsigned* err,
                                           unsigned where) {
  const unsigned long long t0 = globaltimer_ns();
  const unsigned long long budget = wait_budget_ns(err);
  for (unsigned it = 0; it < kWaitIterLimit; ++it) {
    if (ld_acquire_gpu(ctr) >= target) return true;
    if ((it & 31u) == 31u) {
      if (error_code(err) != 0u) return false;
      if (globaltimer_ns() - t0 > budget) break;
    }
    __nanosleep(40);
  }
  set_error(err, DSPARK_ERR_TIMEOUT, where);
  return false;
}

// CTA-wide: thread 0 waits, the result is broadcast; all threads then see the
// producers' writes (acquire by thread 0, ordered for the CTA by the barrier).
template <class Sync>
__device__ __forceinline__ bool cta_wait_at_least(const unsigned* ctr, unsigned target, unsigned* err,
                                                  unsigned where, int* s_flag);

// CTA-wide release: every thread's prior global writes become visible before
// the counter moves.
template <class Sync>
__device__ __forceinline__ void cta_release_add(unsigned* ctr, unsigned v);


// ------------------------------------------------------ barrier policies
// Whole-CTA barrier, or a named barrier over the first NT threads (used by
// warp-specialised kernels whose other warps never join).
struct CtaSync {
  __device__ __forceinline__ static void sync() { __syncthreads(); }
};
template <int ID, int NT>
struct NamedSync {
  __device__ __forceinline__ static void sync() { asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(NT) : "memory"); }
};

// ----------------------------------------------------------- reductions
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_min_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ int warp_max_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide reductions; `red` is shared scratch of >= 32 elements. All
// threads of the block must call; every thread gets the result.
template <int NT, class Sync = CtaSync>
__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  Sync::sync();
  if (l == 0) red[w] = v;
  Sync::sync();
  v = (l < NT / 32) ? red[l] : -INFINITY;
  v = warp_max(v);
  return v;
}
template <int NT, class Sync = CtaSync>
__device__ __forceinline__ double block_sum(double v, double* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  Sync::sync();
  if (l == 0) red[w] = v;
  Sync::sync();
  v = (l < NT / 32) ? red[l] : 0.0;
  v = warp_sum(v);
  return v;
}
template <int NT, class Sync = CtaSync>
__device__ __forceinline__ int block_min_int(int v, int* red) {
  v = warp_min_int(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  Sync::sync();
  if (l == 0) red[w] = v;
  Sync::sync();
  v = (l < NT / 32) ? red[l] : 0x7fffffff;
  v = warp_min_int(v);
  return v;
}
template <int NT, class Sync = CtaSync>
__device__ __forceinline__ int block_max_int(int v, int* red) {
  v = warp_max_int(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  Sync::sync();
  if (l == 0) red[w] = v;
  Sync::sync();
  v = (l < NT / 32) ? red[l] : -0x7fffffff;
  v = warp_max_int(v);
  return v;
}

// Inclusive scan of fp64 within a warp.
__device__ __forceinline__ double warp_inclusive_scan(double v) {
  const int l = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    double n = __shfl_up_sync(0xffffffffu, v, o);
    if (l >= o) v += n;
  }
  return v;
}

// Block-wide exclusive scan of fp64 (thread order); returns the exclusive
// prefix, writes the block total to *total. `red` >= 33 doubles of shared.
template <int NT, class Sync = CtaSync>
__device__ __forceinline__ double block_exclusive_scan(double v, double* red, double* total) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  double inc = warp_inclusive_scan(v);
  double exw = __shfl_up_sync(0xffffffffu, inc, 1);
  if (l == 0) exw = 0.0;
  Sync::sync();
  if (l == 31) red[w] = inc;
  Sync::sync();
  if (w == 0) {
    double s = (l < NT / 32) ? red[l] : 0.0;
    double si = warp_inclusive_scan(s);
    double se = __shfl_up_sync(0xffffffffu, si, 1);
    if (l == 0) se = 0.0;
    if (l < NT / 32) red[l] = se;
    if (l == NT / 32 - 1) red[32] = si;
  }
  Sync::sync();
  double ex = red[w] + exw;
  *total = red[32];
  Sync::sync();
  return ex;
}

template <class Sync>
__device__ __forceinline__ bool cta_wait_at_least(const unsigned* ctr, unsigned target, unsigned* err,
                                                  unsigned where, int* s_flag) {
  if (threadIdx.x == 0) {
    bool ok = wait_at_least(ctr, target, err, where);
    __threadfence();
    *s_flag = ok ? 1 : 0;
  }
  Sync::sync();
  bool ok = *s_flag != 0;
  Sync::sync();
  return ok;
}

template <class Sync>
__device__ __forceinline__ void cta_release_add(unsigned* ctr, unsigned v) {
  Sync::sync();
  if (threadIdx.x == 0) {
    __threadfence();
    red_release_gpu_add(ctr, v);
  }
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<unsigned>(b) << 16);
}

// ------------------------------------------------- exponential in fp64
// 2^(j/16), j = 0..15, for exp_fine; fill with fill_exp_table before use.
__device__ __forceinline__ void fill_exp_table(double* t16, int tid) {
  if (tid < 16) t16[tid] = exp2(static_cast<double>(tid) / 16.0);
}

// max / min that return NaN when either input is NaN (PTX .NaN form).
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}
__device__ __forceinline__ float fmin_nan(float a, float b) {
  float d;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// e^(zh + zl) in fp64, for an fp32 value zh and a small fp32 correction zl
// (the rounding error of zh, |zl| <= ulp(zh)). Table-driven, after Tang's
// method: zh = n ln2/16 + r with n the integer nearest zh 16/ln2, so that
// e^(zh+zl) = 2^(n>>4) 2^((n&15)/16) e^(r+zl). r is formed with a two-part
// constant (Cody and Waite): n kC1 is exact since kC1 has 10 significant bits
// and |n| < 2^14, and the remainder costs one rounding (~1e-9 absolute at
// |r| ~ 0.02). e^x - 1 for |x| <= 0.022 is its Taylor series to the fifth
// power (truncation < 2e-13) in fp32, whose rounding moves 1 + p by ~3e-9;
// the last step is one fp64 FMA by the exact 2^(n>>4) 2^((n&15)/16). The
// result's relative error is ~5e-9 for |zh| < 30 (against ~1e-7 for an fp32
// exponential of an fp32-rounded argument). Branch-free: zh is clamped to
// [-708, 709] (so a row far outside fp64's range has a sum outside
// [1e-280, 1e280] and is redrawn by its caller with its own maximum), and a
// NaN zh gives NaN.
__device__ __forceinline__ double exp_fine(float zh, float zl, const double* t16) {
  constexpr float kInvC = 23.083120654223414f;     // 16 / ln 2
  constexpr float kC1 = 0.0433349609375f;          // 710 * 2^-14
  constexpr float kC2 = -1.326215250341961e-05f;   // ln2/16 - kC1
  const float x = fmin_nan(fmax_nan(zh, -708.f), 709.f);
  // n = x 16/ln2 rounded to the nearest integer, by adding 1.5 * 2^23 in one
  // rounding (exact product): the integer lands in the low mantissa bits
  const float tn = fmaf(x, kInvC, 12582912.f);
  const float n = __fsub_rn(tn, 12582912.f);
  const int ni = __float_as_int(tn) - 0x4B400000;
  float r = fmaf(-n, kC1, x);
  r = fmaf(-n, kC2, r);
  r = __fadd_rn(r, zl);
  float q = fmaf(r, 1.f / 120.f, 1.f / 24.f);
  q = fmaf(q, r, 1.f / 6.f);
  q = fmaf(q, r, 0.5f);
  q = fmaf(q, r, 1.f);
  const float p = __fmul_rn(q, r);
  const double t = t16[ni & 15];
  // t is in [1, 2); adding (n >> 4) to its exponent field scales it by
  // 2^(n>>4), within the normal range for |x| <= 709
  const double ts = __hiloint2double(__double2hiint(t) + (ni >> 4) * (1 << 20), __double2loint(t));
  return fma(ts, static_cast<double>(p), ts);
}

// ------------------------------------------- packed fp32 pairs (sm_100)
// Two fp32 values in one 64-bit register, for the .f32x2 forms of add, sub,
// mul and fma (one instruction, two results, each rounded as its scalar form).
struct F2 {
  unsigned long long v;
};
__device__ __forceinline__ F2 f2(float a, float b) {
  F2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r.v) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float f2_lo(F2 x) { return __uint_as_float(static_cast<unsigned>(x.v)); }
__device__ __forceinline__ float f2_hi(F2 x) { return __uint_as_float(static_cast<unsigned>(x.v >> 32)); }
__device__ __forceinline__ F2 add2(F2 a, F2 b) {
  F2 r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
  return r;
}
__device__ __forceinline__ F2 sub2(F2 a, F2 b) {
  F2 r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
  return r;
}
__device__ __forceinline__ F2 mul2(F2 a, F2 b) {
  F2 r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
  return r;
}
__device__ __forceinline__ F2 fma2(F2 a, F2 b, F2 c) {
  F2 r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r.v) : "l"(a.v), "l"(b.v), "l"(c.v));
  return r;
}

// e^(x + y) for two pairs, where zh = fl(x + y) is already formed: the same
// table-driven steps as exp_fine, with the reduced argument built from x and y
// themselves, r = (x - n ln2/16) + y, so that the rounding error of zh never
// enters (x is the base logit, y the small Markov bias). n comes from the
// clamped zh; when zh is clamped the argument is shifted with it.
__device__ __forceinline__ void exp_sum2(F2 x, F2 y, F2 zh, const double* t16, double* w0, double* w1) {
  const F2 kInvC = f2(23.083120654223414f, 23.083120654223414f);
  const F2 kMagic = f2(12582912.f, 12582912.f);
  const F2 kNC1 = f2(-0.0433349609375f, -0.0433349609375f);
  const F2 kNC2 = f2(1.326215250341961e-05f, 1.326215250341961e-05f);
  const F2 zc = f2(fmin_nan(fmax_nan(f2_lo(zh), -708.f), 709.f), fmin_nan(fmax_nan(f2_hi(zh), -708.f), 709.f));
  const F2 xs = add2(x, sub2(zc, zh));   // x itself unless zh was clamped
  const F2 tn = fma2(zc, kInvC, kMagic);
  const F2 n = sub2(tn, kMagic);
  F2 r = fma2(n, kNC1, xs);
  r = fma2(n, kNC2, r);
  r = add2(r, y);
  F2 q = fma2(r, f2(1.f / 120.f, 1.f / 120.f), f2(1.f / 24.f, 1.f / 24.f));
  q = fma2(q, r, f2(1.f / 6.f, 1.f / 6.f));
  q = fma2(q, r, f2(0.5f, 0.5f));
  q = fma2(q, r, f2(1.f, 1.f));
  const F2 p = mul2(q, r);
  const int n0 = __float_as_int(f2_lo(tn)) - 0x4B400000, n1 = __float_as_int(f2_hi(tn)) - 0x4B400000;
  const double t0 = t16[n0 & 15], t1 = t16[n1 & 15];
  const double s0 = __hiloint2double(__double2hiint(t0) + (n0 >> 4) * (1 << 20), __double2loint(t0));
  const double s1 = __hiloint2double(__double2hiint(t1) + (n1 >> 4) * (1 << 20), __double2loint(t1));
  *w0 = fma(s0, static_cast<double>(f2_lo(p)), s0);
  *w1 = fma(s1, static_cast<double>(f2_hi(p)), s1);
}

// Sum over the 32 lanes of a warp of 16 values per lane, v[c] for c = 0..15:
// a halving exchange (lanes split the values at each step and add what their
// partner sends), then one final exchange. Lane l returns the total of
// v[l >> 1] (lanes 2c and 2c + 1 both hold the total of value c). 15 paired
// exchanges and one more: about 7 instructions per value.
__device__ __forceinline__ double warp_transpose_sum16(double (&v)[16], int lane) {
#pragma unroll
  for (int step = 0; step < 4; ++step) {
    const int half = 8 >> step;           // values kept after this step
    const int bit = 16 >> step;           // partner lane distance
    const bool upper = (lane & bit) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const double send = upper ? v[i] : v[i + half];
      const double keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
    }
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

}  // namespace dspark
