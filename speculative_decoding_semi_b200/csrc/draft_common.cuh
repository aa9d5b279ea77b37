// Pieces of the persistent draft kernels that do not depend on how the
// corrected logits were produced: the previous-token lookup and the
// per-request selection (inverse-CDF sampling over vocabulary chunks).
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace dspark {

// Token that conditions the Markov bias at position i (0-based): the anchor
// for i = 0, else the token drawn at i-1 (written by another CTA in this
// launch, read through L2). An out-of-range anchor is recorded and replaced by 0.
__device__ __forceinline__ int previous_token(const DraftArgs& a, int b, int i) {
  int t = (i == 0) ? a.anchor[b] : __ldcg(a.tokens + static_cast<long long>(b) * a.K + i - 1);
  if (t < 0 || t >= a.V) {
    set_error(a.err, DSPARK_ERR_DEVICE_ASSERT, 0x40000000u | static_cast<unsigned>(b));
    t = 0;
  }
  return t;
}

// Vocabulary chunk of CTA c when V is split into `unit`-wide pieces over G CTAs.
__device__ __forceinline__ void chunk_bounds(int V, int unit, int G, int c, int* lo, int* hi) {
  const int U = V / unit;
  *lo = static_cast<int>(static_cast<long long>(c) * U / G) * unit;
  *hi = static_cast<int>(static_cast<long long>(c + 1) * U / G) * unit;
}

// Weight of logit z with shift m and factor f: fp32 exp(z - m) f for a row
// redrawn with its own maximum (m != 0), fp64 exp(z) f otherwise.
__device__ __forceinline__ double shifted_weight(float z, float m, double f, const double* t16) {
  if (m == 0.f) return __dmul_rn(exp_fine(z, 0.f, t16), f);
  return __dmul_rn(static_cast<double>(expf(z - m)), f);
}

// First element k of z[lo,hi) at which the running sum of the weights
// shifted_weight(z_k, m, f) exceeds R (strict '>'), with each thread scanning a
// contiguous stretch; if rounding leaves no such element, the last one with a
// positive weight. Returns the index (>= lo) to every thread.
template <int NT, class Sync>
__device__ __forceinline__ int rescan_range(const float* zrow, int lo, int hi, float m, double f, double R,
                                            const double* t16) {
  __shared__ double redd[33];
  __shared__ int redi[32];
  const int tid = threadIdx.x;
  const int per = (hi - lo + NT - 1) / NT;
  const int e_lo = min(hi, lo + tid * per), e_hi = min(hi, e_lo + per);
  double lw = 0.0;
  int last_pos = -1;
  for (int k = e_lo; k < e_hi; ++k) {
    const double w = shifted_weight(__ldcg(zrow + k), m, f, t16);
    lw += w;
    if (w > 0.0) last_pos = k;
  }
  double tot;
  const double ex = block_exclusive_scan<NT, Sync>(lw, redd, &tot);
  int found = 0x7fffffff;
  if (e_lo < e_hi && ex + lw > R) {
    double cum = ex;
    for (int k = e_lo; k < e_hi; ++k) {
      const double w = shifted_weight(__ldcg(zrow + k), m, f, t16);
      cum += w;
      if (cum > R && w > 0.0) {
        found = k;
        break;
      }
    }
    if (found == 0x7fffffff && last_pos >= 0) found = last_pos;
  }
  int t = block_min_int<NT, Sync>(found, redi);
  if (t == 0x7fffffff) t = block_max_int<NT, Sync>(last_pos, redi);
  return max(t, lo);
}

// Inverse-CDF draw of request b at position i from the G chunk partials
// (m_c, S_c = sum_{v in chunk c} exp(z_v - m_c)); chunk c covers the
// vocabulary slice chunk_bounds(V, unit, G, c). The chunks are combined in
// vocabulary order in fp64 with the common shift M = max m_c; the chunk whose
// inclusive prefix first exceeds u*W is rescanned with the weights
// exp(z - m_c) * exp(m_c - M) of the stored fp32 z (the producer's sums also
// carried z's rounding error; the difference is confined to one chunk), and
// the first element whose running sum exceeds the remainder is the token
// (strict '>', so a zero weight is never drawn). If W leaves [1e-280, 1e280]
// (every weight underflowing or some overflowing fp64), the row is redone with
// its exact maximum as the shift. Writes draft_tokens, q_tok = w_t / W and
// lse_q = M + log W. All NT threads call.
template <int NT, class Sync>
__device__ __noinline__ void select_token(const DraftArgs& a, int b, int i, int G, int unit, const double* t16) {
  __shared__ float redf[32];
  __shared__ double redd[33];
  __shared__ int redi[32];
  __shared__ double s_W, s_exc;
  const int tid = threadIdx.x;
  const long long pb = static_cast<long long>(b) * G;
  const long long o = static_cast<long long>(b) * a.K + i;
  const float* zrow = a.z + o * a.V;
  float mc = -INFINITY;
  double Sc = 0.0;
  if (tid < G) {
    mc = __ldcg(a.part_m + pb + tid);
    Sc = __ldcg(a.part_S + pb + tid);
  }
  float M = block_max<NT, Sync>(mc, redf);
  const double wc = (tid < G) ? __dmul_rn(Sc, exp(static_cast<double>(mc) - static_cast<double>(M))) : 0.0;
  double total;
  const double ex = block_exclusive_scan<NT, Sync>(wc, redd, &total);
  if (tid == G - 1) s_W = ex + wc;
  Sync::sync();
  double W = s_W;
  const double u = static_cast<double>(a.u[o]);
  int t;
  float m_t;
  double f_t;
  if (W >= 1e-280 && W <= 1e280) {
    const double thr = u * W;
    int c = block_min_int<NT, Sync>((tid < G && ex + wc > thr) ? tid : 0x7fffffff, redi);
    if (c == 0x7fffffff) c = G - 1;
    if (tid == c) s_exc = ex;
    Sync::sync();
    const double R = thr - s_exc;
    int lo, hi;
    chunk_bounds(a.V, unit, G, c, &lo, &hi);
    m_t = __ldcg(a.part_m + pb + c);
    f_t = exp(static_cast<double>(m_t) - static_cast<double>(M));
    t = rescan_range<NT, Sync>(zrow, lo, hi, m_t, f_t, R, t16);
  } else {
    // whole row with its exact maximum as the shift
    float mx = -INFINITY;
    for (int k = tid; k < a.V; k += NT) mx = fmaxf(mx, __ldcg(zrow + k));
    M = block_max<NT, Sync>(mx, redf);
    double s = 0.0;
    for (int k = tid; k < a.V; k += NT) s += shifted_weight(__ldcg(zrow + k), M, 1.0, t16);
    W = block_sum<NT, Sync>(s, redd);
    if (!(W > 0.0) || !(W < INFINITY)) {  // non-finite logits
      if (tid == 0) {
        set_error(a.err, DSPARK_ERR_DEVICE_ASSERT, 0x30000000u | static_cast<unsigned>(b));
        a.tokens[o] = 0;
        a.q_tok[o] = 0.f;
        a.lse_q[o] = 0.0;
      }
      Sync::sync();
      return;
    }
    m_t = M;
    f_t = 1.0;
    // the rescan's own running total is the W that u scales
    double Wscan;
    {
      const int per = (a.V + NT - 1) / NT;
      const int e_lo = min(a.V, tid * per), e_hi = min(a.V, e_lo + per);
      double lw = 0.0;
      for (int k = e_lo; k < e_hi; ++k) lw += shifted_weight(__ldcg(zrow + k), M, 1.0, t16);
      double tot;
      const double exs = block_exclusive_scan<NT, Sync>(lw, redd, &tot);
      if (e_hi == a.V && e_lo < e_hi) s_W = exs + lw;
      Sync::sync();
      Wscan = s_W;
      Sync::sync();
    }
    W = Wscan;
    t = rescan_range<NT, Sync>(zrow, 0, a.V, M, 1.0, u * W, t16);
  }
  if (tid == 0) {
    const double w_t = shifted_weight(__ldcg(zrow + t), m_t, f_t, t16);
    a.tokens[o] = t;
    a.q_tok[o] = static_cast<float>(w_t / W);
    a.lse_q[o] = static_cast<double>(M) + log(W);
  }
  Sync::sync();
}

// Among n values x(0..n-1) (read through `get`) laid out in lane-contiguous
// blocks, find the first index whose inclusive prefix exceeds `thr(total)`
// (strict, never a zero entry); returns it, or the last positive index if
// rounding leaves none, with its exclusive prefix in *excl and the sum of all
// n values in *total. `thr` maps the total to the threshold, so one pass both
// sums and searches. Sums run sequentially within a lane's block and in lane
// order across blocks. One warp, all lanes; each lane's loads are issued
// together (up to kSearchRegs values per lane stay in registers).
template <int kSearchRegs, class Get, class Thr>
__device__ __forceinline__ int warp_search(int n, Get get, Thr thr_of, int lane, double* excl, double* total) {
  const int per = (n + 31) / 32;
  const int lo = min(n, lane * per), hi = min(n, lo + per);
  double local = 0.0;
  int last_pos = -1;
  double vals[kSearchRegs];
  const bool in_regs = per <= kSearchRegs;
  if (in_regs) {
#pragma unroll
    for (int j = 0; j < kSearchRegs; ++j) vals[j] = get(min(lo + j, n - 1));  // clamped: the loads issue together
#pragma unroll
    for (int j = 0; j < kSearchRegs; ++j)
      if (lo + j >= hi) vals[j] = 0.0;
#pragma unroll
    for (int j = 0; j < kSearchRegs; ++j) {
      local += vals[j];
      if (vals[j] > 0.0) last_pos = lo + j;
    }
  } else {
    for (int x = lo; x < hi; ++x) {
      const double v = get(x);
      local += v;
      if (v > 0.0) last_pos = x;
    }
  }
  double inc = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double nb = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += nb;
  }
  double mine = __shfl_up_sync(0xffffffffu, inc, 1);
  if (lane == 0) mine = 0.0;
  *total = __shfl_sync(0xffffffffu, inc, 31);
  const double thr = thr_of(*total);
  int found = 0x7fffffff;
  double found_ex = 0.0;
  if (lo < hi && mine + local > thr) {
    double c = mine;
    if (in_regs) {
#pragma unroll
      for (int j = 0; j < kSearchRegs; ++j) {
        if (found == 0x7fffffff && lo + j < hi) {
          if (c + vals[j] > thr && vals[j] > 0.0) {
            found = lo + j;
            found_ex = c;
          }
          c += vals[j];
        }
      }
    } else {
      for (int x = lo; x < hi; ++x) {
        const double v = get(x);
        if (c + v > thr && v > 0.0) {
          found = x;
          found_ex = c;
          break;
        }
        c += v;
      }
    }
  }
  int best = found;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = min(best, __shfl_xor_sync(0xffffffffu, best, o));
  if (best == 0x7fffffff) {
    // rounding: the last positive entry, with its exclusive prefix from its owner
    int lp = last_pos;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lp = max(lp, __shfl_xor_sync(0xffffffffu, lp, o));
    best = max(lp, 0);
    double e = 0.0;
    if (best >= lo && best < hi) {
      e = mine;
      for (int x = lo; x < best; ++x) e += get(x);
    }
    const int owner = per > 0 ? min(31, best / per) : 0;
    *excl = __shfl_sync(0xffffffffu, e, owner);
    return best;
  }
  const int owner = per > 0 ? min(31, best / per) : 0;
  *excl = __shfl_sync(0xffffffffu, found_ex, owner);
  return best;
}


// Sum over the 32 lanes of a warp of 32 values per lane, v[c] for c = 0..31,
// by a halving exchange: lane l returns the total of v[l] (31 exchanges).
__device__ __forceinline__ float warp_transpose_sum32f(float (&v)[32], int lane) {
#pragma unroll
  for (int step = 0; step < 5; ++step) {
    const int half = 16 >> step, bit = 16 >> step;
    const bool upper = (lane & bit) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
    }
  }
  return v[0];
}

// z of row v0 + lane of one row of logits, base + a . Bf, for a 32-row unit
// at v0 (a multiple of 32): a is the operand row (r bf16 values), Bf the
// [r, V] factor (bf16), zbase the row's base logits. fp32 (one warp; lane l
// takes the rank indices l, l + 32, ... and the lanes' 32 partial sums are
// exchanged at the end). For r a multiple of 32.
static __device__ __noinline__ float unit_logit(const uint16_t* a, const uint16_t* Bf, const float* zbase, int r, int V,
                                                long long v0, int lane) {
  float acc[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) acc[e] = 0.f;
#pragma unroll 2
  for (int k = lane; k < r; k += 32) {
    const float ak = __uint_as_float(static_cast<unsigned>(__ldcg(a + k)) << 16);
    const uint4* row = reinterpret_cast<const uint4*>(Bf + static_cast<long long>(k) * V + v0);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = __ldg(row + c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc[8 * c + 2 * j] = fmaf(ak, __uint_as_float(w[j] << 16), acc[8 * c + 2 * j]);
        acc[8 * c + 2 * j + 1] = fmaf(ak, __uint_as_float(w[j] & 0xffff0000u), acc[8 * c + 2 * j + 1]);
      }
    }
  }
  const float bias = warp_transpose_sum32f(acc, lane);
  return __fadd_rn(__ldcg(zbase + v0 + lane), bias);
}

// Stage the 32 columns v0.. of the [r, V] bf16 factor Bf in shared memory as
// [r][32] (64 bytes a row), one warp: 16-byte cp.async copies, r * 4 of them,
// all issued at once so the unit arrives in one memory trip; then
// stage_unit_wait. v0 is a multiple of 32, V of 32; dst 16-byte aligned.
__device__ __forceinline__ void stage_unit_issue(uint8_t* dst, const uint16_t* Bf, int V, int r, long long v0,
                                                 int lane) {
  for (int idx = lane; idx < r * 4; idx += 32) {
    const int k = idx >> 2, c = idx & 3;
    const uint16_t* src = Bf + static_cast<long long>(k) * V + v0 + 8 * c;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(
                     dst + k * 64 + c * 16))),
                 "l"(src)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void stage_unit_wait() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncwarp();  // every lane's copies are visible to the warp
}

// sum_k a_k Bf[k, v0 + lane] over a 32-column unit staged in shared memory:
// bfu [r][32] bf16 (stage_unit_issue), a_s the operand row (r bf16, 16-byte
// aligned). fp32, eight partial sums (k mod 8) added at the end.
__device__ __forceinline__ float staged_unit_dot(const uint16_t* bfu, const uint4* a_s, int r, int lane) {
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  for (int k0 = 0; k0 < r; k0 += 8) {
    const uint4 av = a_s[k0 >> 3];
    const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float b0 = __uint_as_float(static_cast<unsigned>(bfu[(k0 + 2 * j) * 32 + lane]) << 16);
      const float b1 = __uint_as_float(static_cast<unsigned>(bfu[(k0 + 2 * j + 1) * 32 + lane]) << 16);
      acc[2 * j] = fmaf(__uint_as_float(aw[j] << 16), b0, acc[2 * j]);
      acc[2 * j + 1] = fmaf(__uint_as_float(aw[j] & 0xffff0000u), b1, acc[2 * j + 1]);
    }
  }
  return ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
}

}  // namespace dspark
