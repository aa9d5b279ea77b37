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

}  // namespace dspark
