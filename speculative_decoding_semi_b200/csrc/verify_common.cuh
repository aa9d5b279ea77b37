// Structures and warp-level routines shared by the verify kernel and the
// tensor-core residual kernel (internal to libdspark).
#pragma once

#include <cfloat>
#include <climits>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace dspark {
namespace vfy {

using namespace sm100;

constexpr int kSeg = 1024;                // row-pass segment: 32 lanes x 8 float4
constexpr int kRSeg = 512;                // residual segment: 32 lanes x 4 float4
constexpr int kCons = 8;                  // consumer warps per group (one segment each)
constexpr int kGroups = 2;                // consumer groups, taking alternate stages
constexpr int kProdWarp = kCons * kGroups;
constexpr int kWarps = kProdWarp + 4;     // + producer + three more for the warp-per-unit phases
constexpr int kThreads = kWarps * 32;
constexpr int kRowItem = kCons * kSeg;    // logits per row item
constexpr int kResItem = kCons * kRSeg;   // logits (and z values) per residual item
constexpr int kStageBytes = kRowItem * 4;
constexpr int kStages = 6;
constexpr int kPlanThreads = 1024;
constexpr int kRegSeg = 8;                // segment values per lane held in registers (nseg <= 256)
constexpr double kSumLo = 1e-20, kSumHi = 1e30;
constexpr float kLog2e = 1.44269504088896340736f;  // log2(e)
constexpr double kLog2eD = 1.44269504088896340736;

enum : int { kItemRow = 0, kItemRes = 1, kItemExit = 2 };
// kCtlBar..kCtlBar+3: barrier counters
// kCtlRes..kCtlRes+3: slice sums of the residual groups published (variant B)
enum : int { kCtlRows = 0, kCtlListed = 1, kCtlBar = 2, kCtlBonus = 6, kCtlRes = 8, kCtlCount = 12 };

// One target row of the compact numbering.
struct RowInfo {
  int brl;        // b | rho << 16 | L_b << 22
  int tok;        // drafted token tested at this row, -1 at the last row or if invalid
  long long row;  // row index into the target logits
};

struct Desc {
  int type, b, R, g;     // request, compact row, item index
  int n, tok, pad0, pad1;  // logits in the item; drafted token (row items)
  float shift[4], f[4];  // residual: per 1024-segment base-2 shift and p factor
  float mq, fq, pad2[2];  // residual: q = 2^(z log2 e - mq) * fq
};

struct RowStat {
  double M, W;  // base-2 largest shift, sum of 2^(x log2 e - M)
};
struct ResDec {
  int acc, R;
  long long row;  // target row of the rejection
  float mq, fq;
};

// Variant B: one request with a residual, in list order. The residual kernel
// recomputes z of row brow = b K + acc (of the base logits and of the operand
// rows) and weighs max(0, p - q) with p = 2^(x log2 e - mp) fp and
// q = 2^(z log2 e - mq) fq.
struct ResSlot {
  int b, acc;
  long long row;  // target row of the rejection
  int brow, R;    // base / operand row; compact target row (for the fallback draw from p)
  float mq, fq, mp, fp;
  int pad[2];
};

struct Ws {
  RowInfo* rowinfo;  // [B*(K+1)]
  int* rowbase;      // [B] compact index of row 0, -1 for an invalid request
  unsigned* ctl;     // counters, cleared by the plan kernel
  float* part_m;     // [B*(K+1)][nseg] segment base-2 shift h
  double* part_S;    // [B*(K+1)][nseg] segment sum of 2^(x log2 e - h)
  float* x_tok;      // [B*(K+1)] logit at the drafted token (-inf if none)
  RowStat* rstat;    // [B*(K+1)]
  int* accepted;     // [B*(K+1)] accept test of the row's draft
  ResDec* dec;       // [B]
  float2* resfac;    // [B][nseg] residual (shift, p factor) per 1024-segment
  int* list;         // [B] requests with a residual pass
  int* blist;        // [B] requests whose drafts were all accepted (bonus draw)
  unsigned* req_rows;  // [B] rows of the request whose statistics are done (phase 2)
  double* seg_w;     // [B][nrseg] residual segment sums
  ResSlot* slots;    // [B] variant B: the requests with a residual, in list order
};

struct Params {
  VerifyArgs a;
  Ws w;
  int nseg, nrseg, ngrp, nrgrp;
  int recompute;  // variant B: z is not stored; the residual kernel follows
  int res_gsize;  // variant B: requests per residual group (the MMA's N, at most 128)
};

// Requests per residual group: a multiple of 32 up to 128 (the draft's
// request groups, whose operand-image scratch the residual groups reuse).
inline int residual_group_size(int B) { return B >= 128 ? 128 : (B <= 32 ? 32 : (B + 31) & ~31); }

// The tensor-core residual kernel of variant B (residual_tc.cu), launched
// after the verify kernel on the same stream.
cudaError_t launch_residual_tc(const Params& P, cudaStream_t stream);

// ------------------------------------------------------------ weights
// The fp32 weights of the target distribution p and of the residual
// max(0, p - q); explicit rounding intrinsics keep every site bit-identical.
__device__ __forceinline__ float p_w(float x, float h) { return exp2f(__fmaf_rn(x, kLog2e, -h)); }
__device__ __forceinline__ float res_w(float x, float z, float h, float f, float mq, float fq) {
  const float p = __fmul_rn(exp2f(__fmaf_rn(x, kLog2e, -h)), f);
  const float q = __fmul_rn(exp2f(__fmaf_rn(z, kLog2e, -mq)), fq);
  const float d = __fsub_rn(p, q);
  return d > 0.f ? d : 0.f;
}
__device__ __forceinline__ float group4(float w0, float w1, float w2, float w3) {
  return __fadd_rn(__fadd_rn(__fadd_rn(w0, w1), w2), w3);
}
// 2^(h - M): the scale of a segment with base-2 shift h in a row whose largest
// shift is M (exactly 1 in the common case h == M). The rare exponential is
// kept out of line, so the common path carries neither its instructions nor
// their evaluation.
static __device__ __noinline__ double exp2_rare(double x) { return exp2(x); }
__device__ __forceinline__ double seg_scale(float h, double M) {
  if (static_cast<double>(h) == M) return 1.0;
  return exp2_rare(static_cast<double>(h) - M);
}
// (shift, factor) of a 1024-segment in the residual: p = 2^(x log2 e - h) * f.
__device__ __forceinline__ float2 res_factor(float h, double M, double W) {
  if (h == -INFINITY) return make_float2(0.f, 0.f);
  return make_float2(h, static_cast<float>(seg_scale(h, M) / W));
}
// q = exp(z - lse) = 2^(z log2 e - mq) * fq with mq = fp32(lse log2 e).
__device__ __forceinline__ void q_factor(double lse, float* mq, float* fq) {
  const double c = lse * kLog2eD;
  *mq = static_cast<float>(c);
  *fq = static_cast<float>(exp2(static_cast<double>(*mq) - c));
}

// p = exp(x - lse_p) = 2^(x log2 e - mp) * fp for a row with base-2 largest
// shift M and sum W (lse_p log2 e = M + log2 W); a degenerate row gets p = 0.
__device__ __forceinline__ void p_factor(double M, double W, float* mp, float* fp) {
  if (!(W > 0.0) || !(W < INFINITY)) {
    *mp = 0.f;
    *fp = 0.f;
    return;
  }
  const double c = M + log2(W);
  *mp = static_cast<float>(c);
  *fp = static_cast<float>(exp2(static_cast<double>(*mp) - c));
}

__device__ __forceinline__ float4 neg_inf4() { return make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY); }


// ------------------------------------------------------ warp-level helpers
// Inverse CDF over nseg segment weights, one warp; lane l owns the segments
// [l per, l per + per). raw(q) loads what segment q's weight needs and
// value(raw) computes the weight (the same value whenever called); the N <=
// per-lane raw values are loaded before any is used, so their loads issue
// together. Returns the first segment whose inclusive running sum exceeds
// u * total with a positive weight, else (rounding) the last positive one,
// with *rem = u * total minus the weight before it; -1 if total <= 0.
template <int N, class Raw, class Value>
__device__ int pick_segment_n(int nseg, float u, int lane, Raw raw, Value value, double* rem) {
  const int per = (nseg + 31) / 32;
  const int lo = min(nseg, lane * per), hi = min(nseg, lo + per);
  using T = decltype(raw(0));
  T rv[N];
#pragma unroll
  for (int i = 0; i < N; ++i) rv[i] = raw(min(lo + i, nseg - 1));  // clamped: always a valid address
  double wv[N];
  double local = 0.0;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    wv[i] = lo + i < hi ? value(rv[i]) : 0.0;
    local += wv[i];
  }
  const double inc = warp_inclusive_scan(local);
  double ex = __shfl_up_sync(0xffffffffu, inc, 1);
  if (lane == 0) ex = 0.0;
  const double total = __shfl_sync(0xffffffffu, inc, 31);
  if (!(total > 0.0)) return -1;
  const double thr = static_cast<double>(u) * total;
  int cand = INT_MAX, lastq = -1;
  double cand_ex = 0.0, last_ex = 0.0, c = ex;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const double v = wv[i];
    if (v > 0.0) {
      if (cand == INT_MAX && c + v > thr) {
        cand = lo + i;
        cand_ex = c;
      }
      lastq = lo + i;
      last_ex = c;
    }
    c += v;
  }
  int seg = warp_min_int(cand);
  double seg_ex;
  if (seg != INT_MAX) {
    seg_ex = __shfl_sync(0xffffffffu, cand_ex, seg / per);
  } else {
    seg = warp_max_int(lastq);
    if (seg < 0) return -1;
    seg_ex = __shfl_sync(0xffffffffu, last_ex, seg / per);
  }
  *rem = thr - seg_ex;
  return seg;
}

// The same for any nseg: the smallest register block that holds per, or a
// plain loop beyond 32 segments per lane.
template <class Raw, class Value>
__device__ int pick_segment(int nseg, float u, int lane, Raw raw, Value value, double* rem) {
  const int per = (nseg + 31) / 32;
  if (per <= 4) return pick_segment_n<4>(nseg, u, lane, raw, value, rem);
  if (per <= 8) return pick_segment_n<8>(nseg, u, lane, raw, value, rem);
  if (per <= 16) return pick_segment_n<16>(nseg, u, lane, raw, value, rem);
  const int lo = min(nseg, lane * per), hi = min(nseg, lo + per);
  double local = 0.0;
  for (int q = lo; q < hi; ++q) local += value(raw(q));
  const double inc = warp_inclusive_scan(local);
  double ex = __shfl_up_sync(0xffffffffu, inc, 1);
  if (lane == 0) ex = 0.0;
  const double total = __shfl_sync(0xffffffffu, inc, 31);
  if (!(total > 0.0)) return -1;
  const double thr = static_cast<double>(u) * total;
  int cand = INT_MAX, lastq = -1;
  double cand_ex = 0.0, last_ex = 0.0, c = ex;
  for (int q = lo; q < hi; ++q) {
    const double v = value(raw(q));
    if (v > 0.0) {
      if (cand == INT_MAX && c + v > thr) {
        cand = q;
        cand_ex = c;
      }
      lastq = q;
      last_ex = c;
    }
    c += v;
  }
  int seg = warp_min_int(cand);
  double seg_ex;
  if (seg != INT_MAX) {
    seg_ex = __shfl_sync(0xffffffffu, cand_ex, seg / per);
  } else {
    seg = warp_max_int(lastq);
    if (seg < 0) return -1;
    seg_ex = __shfl_sync(0xffffffffu, last_ex, seg / per);
  }
  *rem = thr - seg_ex;
  return seg;
}

// First element of a run of n <= 32 * E elements whose running sum of
// weights exceeds R with a positive weight, or -1 (then *last = the last
// positive one); one warp. Lane l owns elements [E l, E l + E): w[] holds
// their fp32 weights (zero past n). Four consecutive weights form one fp32
// group exactly as in the segment sums; the groups accumulate in fp64, one
// warp-wide scan over the lanes' totals, then a search inside one lane.
template <int E>
__device__ int rescan(int n, int lane, double R, const float (&w)[E], int* last) {
  float c[E];  // inclusive fp32 sums within each group of four
  double lsum = 0.0;
#pragma unroll
  for (int k = 0; k < E / 4; ++k) {
    c[4 * k] = w[4 * k];
    c[4 * k + 1] = __fadd_rn(c[4 * k], w[4 * k + 1]);
    c[4 * k + 2] = __fadd_rn(c[4 * k + 1], w[4 * k + 2]);
    c[4 * k + 3] = __fadd_rn(c[4 * k + 2], w[4 * k + 3]);
    lsum += static_cast<double>(c[4 * k + 3]);
  }
  const double inc = warp_inclusive_scan(lsum);
  double before = __shfl_up_sync(0xffffffffu, inc, 1);
  if (lane == 0) before = 0.0;
  int hit = -1, lp = -1;
  if (before + lsum > R) {
#pragma unroll
    for (int k = 0; k < E / 4; ++k) {
      if (hit < 0) {
#pragma unroll
        for (int j = 3; j >= 0; --j)
          if (w[4 * k + j] > 0.f && before + static_cast<double>(c[4 * k + j]) > R) hit = 4 * k + j;
        before += static_cast<double>(c[4 * k + 3]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (w[e] > 0.f) lp = E * lane + e;
  *last = warp_max_int(lp);
  const unsigned hits = __ballot_sync(0xffffffffu, hit >= 0);
  if (!hits) return -1;
  const int hl = __ffs(hits) - 1;
  return E * hl + __shfl_sync(0xffffffffu, hit, hl);
}


// Draw from p of compact row R (the bonus row, or a rejected row whose
// residual vanished) with the row pass's segment sums; one warp. With `warm`
// set it runs its whole path on whatever the arrays hold, to load its code
// into the SM's instruction cache ahead of the phase that needs it.
static __device__ __noinline__ int sample_p(const Params& P, int R, float u, int lane, bool warm = false) {
  const VerifyArgs& a = P.a;
  const float* pm = P.w.part_m + static_cast<long long>(R) * P.nseg;
  const double* pS = P.w.part_S + static_cast<long long>(R) * P.nseg;
  const double M = __ldcg(&P.w.rstat[R].M);
  const long long row = P.w.rowinfo[R].row;
  // segment weights S 2^(h - M): the row's total W scales them all alike and
  // cancels in the inverse CDF
  double rem = 0.0;
  const int seg = pick_segment(
      P.nseg, u, lane, [&](int q) { return make_double2(__ldcg(pS + q), static_cast<double>(__ldcg(pm + q))); },
      [&](double2 r) { return r.x > 0.0 ? __dmul_rn(r.x, seg_scale(static_cast<float>(r.y), M)) : 0.0; }, &rem);
  if (seg < 0 && !warm) return 0;  // no positive weight: degenerate row
  const int sg = max(seg, 0);
  const float m_s = __ldcg(pm + sg);
  const double Rs = rem / seg_scale(m_s, M);
  const float* x = a.target + row * a.V + static_cast<long long>(sg) * kSeg;
  const int n = min(kSeg, a.V - sg * kSeg);
  constexpr int E = kSeg / 32;
  float w[E];
#pragma unroll
  for (int k = 0; k < E / 4; ++k) {
    const int e = E * lane + 4 * k;
    const float4 v = e < n ? __ldcg(reinterpret_cast<const float4*>(x + e)) : neg_inf4();
    w[4 * k] = p_w(v.x, m_s);
    w[4 * k + 1] = p_w(v.y, m_s);
    w[4 * k + 2] = p_w(v.z, m_s);
    w[4 * k + 3] = p_w(v.w, m_s);
  }
  int last = -1;
  int k = rescan<E>(n, lane, Rs, w, &last);
  if (k < 0) k = max(last, 0);
  return sg * kSeg + k;
}

// Emits request b's accepted drafts and the drawn token.
static __device__ void write_output(const Params& P, int b, int acc, int tok, int lane) {
  const VerifyArgs& a = P.a;
  int32_t* out = a.out_tokens + static_cast<long long>(b) * (a.K + 1);
  // j = 32 (K = 32 only) is never an accepted draft, since acc <= K
  for (int j = lane; j <= a.K; j += 32)
    out[j] = j < acc ? a.tokens[static_cast<long long>(b) * a.K + j] : (j == acc ? tok : -1);
  if (lane == 0) {
    a.accepted[b] = acc;
    a.n_out[b] = acc + 1;
  }
}


}  // namespace vfy
}  // namespace dspark
