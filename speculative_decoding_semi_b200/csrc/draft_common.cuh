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

// Inverse-CDF draw of request b at position i from the G chunk partials
// (m_c, S_c = sum_{v in chunk c} exp(z_v - m_c)). Chunks are combined in
// vocabulary order in fp64 with the common shift M = max m_c; the chunk whose
// inclusive prefix first exceeds u*W is rescanned with weights exp(z - m_c) *
// exp(m_c - M), and the first element whose running sum exceeds the remainder
// is the token (strict '>', so a zero weight is never drawn). Writes
// draft_tokens, q_tok = w_t / W and lse_q = M + log W. All NT threads call.
template <int NT>
__device__ __noinline__ void select_token(const DraftArgs& a, int b, int i, int G) {
  __shared__ float redf[32];
  __shared__ double redd[33];
  __shared__ int redi[32];
  __shared__ double s_W, s_exc;
  const int tid = threadIdx.x;
  const long long pb = static_cast<long long>(b) * G;
  float mc = -INFINITY;
  double Sc = 0.0;
  if (tid < G) {
    mc = __ldcg(a.part_m + pb + tid);
    Sc = __ldcg(a.part_S + pb + tid);
  }
  const float M = block_max<NT>(mc, redf);
  const double wc = (tid < G) ? __dmul_rn(Sc, exp(static_cast<double>(mc) - static_cast<double>(M))) : 0.0;
  double total;
  const double ex = block_exclusive_scan<NT>(wc, redd, &total);
  if (tid == G - 1) s_W = ex + wc;
  __syncthreads();
  const double W = s_W;
  const long long zrow = (static_cast<long long>(b) * a.K + i) * a.V;
  if (!(W > 0.0) || !(W < INFINITY)) {  // non-finite logits
    if (tid == 0) {
      set_error(a.err, DSPARK_ERR_DEVICE_ASSERT, 0x30000000u | static_cast<unsigned>(b));
      a.tokens[static_cast<long long>(b) * a.K + i] = 0;
      a.q_tok[static_cast<long long>(b) * a.K + i] = 0.f;
      a.lse_q[static_cast<long long>(b) * a.K + i] = 0.0;
    }
    __syncthreads();
    return;
  }
  const double thr = static_cast<double>(a.u[static_cast<long long>(b) * a.K + i]) * W;
  int c = block_min_int<NT>((tid < G && ex + wc > thr) ? tid : 0x7fffffff, redi);
  if (c == 0x7fffffff) c = G - 1;
  if (tid == c) s_exc = ex;
  __syncthreads();
  const double R = thr - s_exc;
  const int NU = a.V / 8;
  const int lo = static_cast<int>(static_cast<long long>(c) * NU / G) * 8;
  const int hi = static_cast<int>(static_cast<long long>(c + 1) * NU / G) * 8;
  const float m_c = __ldcg(a.part_m + pb + c);
  const double f_c = exp(static_cast<double>(m_c) - static_cast<double>(M));
  const int per = (hi - lo + NT - 1) / NT;
  const int e_lo = min(hi, lo + tid * per), e_hi = min(hi, e_lo + per);
  double lw = 0.0;
  int last_pos = -1;
  for (int k = e_lo; k < e_hi; ++k) {
    const double w = __dmul_rn(static_cast<double>(expf(__ldcg(a.z + zrow + k) - m_c)), f_c);
    lw += w;
    if (w > 0.0) last_pos = k;
  }
  double tot2;
  const double ex2 = block_exclusive_scan<NT>(lw, redd, &tot2);
  int found = 0x7fffffff;
  if (e_lo < e_hi && ex2 + lw > R) {
    double cum = ex2;
    for (int k = e_lo; k < e_hi; ++k) {
      const double w = __dmul_rn(static_cast<double>(expf(__ldcg(a.z + zrow + k) - m_c)), f_c);
      cum += w;
      if (cum > R && w > 0.0) {
        found = k;
        break;
      }
    }
    if (found == 0x7fffffff && last_pos >= 0) found = last_pos;
  }
  int t = block_min_int<NT>(found, redi);
  if (t == 0x7fffffff) t = block_max_int<NT>(last_pos, redi);
  if (tid == 0) {
    t = max(t, lo);
    const double w_t = __dmul_rn(static_cast<double>(expf(__ldcg(a.z + zrow + t) - m_c)), f_c);
    const long long o = static_cast<long long>(b) * a.K + i;
    a.tokens[o] = t;
    a.q_tok[o] = static_cast<float>(w_t / W);
    a.lse_q[o] = static_cast<double>(M) + log(W);
  }
  __syncthreads();
}

}  // namespace dspark
