// Lossless rejection-sampling verification on the GPU.
//
// QbitAI article "DSpark: ten concepts are enough", section "speculative
// decoding": drafts are checked one by one, the longest accepted prefix is kept
// and one token is resampled at the first divergence, which keeps the target
// distribution exactly. wangjunjian.com tag page, article "Speculative
// Decoding", steps 3-5: compare the two models' probabilities with a random
// number; if every draft passes sample the next token from the target, else
// resample from an adjusted distribution (here max(0, p - q) renormalised).
//
// Two launches (variant B adds the residual kernel of residual_tc.cu).
//   plan    one CTA: checks verify_len and the drafted tokens, numbers the
//           target rows 0..L_b of every request consecutively in request
//           order and clears the counters of the main kernel.
//   main    one persistent cooperative CTA per SM, in four phases separated
//           by device-wide barriers:
//     1 rows      the target rows stream through a ring of shared-memory
//                 stages filled by bulk asynchronous copies (one producer
//                 warp); sixteen consumer warps, in two groups taking alternate
//                 stages, reduce 1024-wide segments: fp64 sum of exp(x) and the
//                 logit at the drafted token;
//     2 row stats one warp per row: (max, sum) from the segment partials and
//                 the accept test u * q(t) < p(t) of the row's draft; the warp
//                 that completes a request's last row (a per-request counter)
//                 finds its first rejection, and the request joins the list
//                 of bonus draws (none) or of residual passes;
//     3 residual  the rejected rows and their z rows stream through the same
//                 ring: sums of max(0, p - q) over 512-wide segments; the
//                 warps outside the stream make the bonus draws meanwhile;
//     4 resample  one warp per listed request draws the resampled token.
// (Variant B ends after phase 2 with the bonus draws: its residual kernel
// recomputes the rejected rows of z and draws the rest.)
// The barriers fall between streaming phases, when no copy is in flight: a
// gpu-scope fence on an SM with bulk copies in flight waits for them to land,
// and a plain store from such an SM takes several microseconds to be seen by
// other SMs, so cross-CTA hand-offs in the middle of a stream cost more than
// the barriers do. Every wait is bounded and reports DSPARK_ERR_TIMEOUT.
//
// Weights. exp(x) is taken as 2^(x log2 e - h), one fused multiply-add and
// one exp2f, with a base-2 shift h = 0 (a segment whose sum leaves
// [1e-20, 1e30] is redone with its own maximum as the shift); four consecutive
// weights are added in fp32 and the groups in fp64. The draws rescan one
// segment with the same fp32 groups, so the segment sums and the rescans
// agree up to the fp64 order of the groups.
#include <algorithm>
#include <cfloat>
#include <climits>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "verify_common.cuh"

namespace dspark {

namespace {

using namespace sm100;
using namespace vfy;

// ------------------------------------------------------------ plan kernel
__device__ int block_exscan_int(int v, int* total, int* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  __syncthreads();
  if (lane == 31) red[w] = inc;
  __syncthreads();
  if (w == 0) {
    const int s = lane < kPlanThreads / 32 ? red[lane] : 0;
    int si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += n;
    }
    if (lane < kPlanThreads / 32) red[lane] = si - s;
    if (lane == 31) red[32] = si;
  }
  __syncthreads();
  const int ex = red[w] + inc - v;
  *total = red[32];
  __syncthreads();
  return ex;
}

__global__ void __launch_bounds__(kPlanThreads) verify_plan_kernel(Params p) {
  __shared__ int red[33];
  // launched early (programmatic dependent launch): the previous kernel's
  // writes (verify lengths, drafts) are visible after the wait; the main
  // kernel may start its prologue now and waits for this grid's results
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const VerifyArgs& a = p.a;
  int carry = 0;
  for (int base = 0; base < a.B; base += kPlanThreads) {
    const int b = base + threadIdx.x;
    int L = -1;
    bool valid = false;
    if (b < a.B) {
      L = a.verify_len[b];
      valid = L >= 0 && L <= a.K;
      if (!valid) set_error(a.err, DSPARK_ERR_DEVICE_ASSERT, 0x10000000u | static_cast<unsigned>(b));
    }
    int total;
    const int ex = block_exscan_int(valid ? L + 1 : 0, &total, red);
    if (b < a.B) {
      const int r0 = carry + ex;
      p.w.rowbase[b] = valid ? r0 : -1;
      p.w.req_rows[b] = 0u;
      if (valid) {
        for (int rho = 0; rho <= L; ++rho) {
          int tok = -1;
          if (rho < L) {
            tok = a.tokens[static_cast<long long>(b) * a.K + rho];
            if (tok < 0 || tok >= a.V) {
              set_error(a.err, DSPARK_ERR_DEVICE_ASSERT, 0x20000000u | static_cast<unsigned>(b));
              tok = -1;  // x_tok stays -inf: p(t) = 0 and the draft is rejected
            }
          }
          RowInfo ri;
          ri.brl = b | (rho << 16) | (L << 22);
          ri.tok = tok;
          ri.row = a.row_start[b] + rho;
          p.w.rowinfo[r0 + rho] = ri;
          p.w.x_tok[r0 + rho] = -INFINITY;
        }
      }
    }
    carry += total;
  }
  if (threadIdx.x < kCtlCount) p.w.ctl[threadIdx.x] = threadIdx.x == kCtlRows ? static_cast<unsigned>(carry) : 0u;
}

// Phase 2, one warp: (M, W) of compact row R from its segment partials, and
// the accept test of the row's draft.
__device__ void row_stats(const Params& P, int R, int lane) {
  const VerifyArgs& a = P.a;
  const RowInfo ri = P.w.rowinfo[R];
  const int b = ri.brl & 0xffff, rho = (ri.brl >> 16) & 63, L = ri.brl >> 22;
  const float* pm = P.w.part_m + static_cast<long long>(R) * P.nseg;
  const double* pS = P.w.part_S + static_cast<long long>(R) * P.nseg;
  float m = -INFINITY;
  double w = 0.0;
  if (P.nseg <= 32 * kRegSeg) {
    float mv[kRegSeg];
    double sv[kRegSeg];
#pragma unroll
    for (int j = 0; j < kRegSeg; ++j) {
      const int s = lane + 32 * j;
      mv[j] = s < P.nseg ? __ldcg(pm + s) : -INFINITY;
      sv[j] = s < P.nseg ? __ldcg(pS + s) : 0.0;
    }
#pragma unroll
    for (int j = 0; j < kRegSeg; ++j) m = fmaxf(m, mv[j]);
    m = warp_max(m);
#pragma unroll
    for (int j = 0; j < kRegSeg; ++j)
      if (sv[j] > 0.0) w += __dmul_rn(sv[j], seg_scale(mv[j], m));
  } else {
    for (int s = lane; s < P.nseg; s += 32) m = fmaxf(m, __ldcg(pm + s));
    m = warp_max(m);
    for (int s = lane; s < P.nseg; s += 32) {
      const double S = __ldcg(pS + s);
      if (S > 0.0) w += __dmul_rn(S, seg_scale(__ldcg(pm + s), m));
    }
  }
  const double W = warp_sum(w);
  if (lane == 0) {
    RowStat st;
    st.M = m;
    st.W = W;
    P.w.rstat[R] = st;
    int accept = 1;
    if (rho < L) {
      const long long idx = static_cast<long long>(b) * a.K + rho;
      const double p_t = exp2(static_cast<double>(__ldcg(P.w.x_tok + R)) * kLog2eD - static_cast<double>(m)) / W;
      const double uq = static_cast<double>(a.u_accept[idx]) * static_cast<double>(a.q_tok[idx]);
      accept = uq < p_t ? 1 : 0;
    }
    P.w.accepted[R] = accept;
  }
}

// Phase 2, one warp: request b's first rejection; a place in the list of
// bonus draws, or the residual pass's inputs and a place in its list.
// With `warm` set it writes nothing: it runs once during phase 1 to load its
// code into the SM's instruction cache ahead of phase 2.
__device__ __noinline__ void decide(const Params& P, int b, int lane, bool warm = false) {
  const VerifyArgs& a = P.a;
  const int r0 = P.w.rowbase[b];
  if (r0 < 0) return;  // invalid request (recorded by the plan kernel)
  const int L = a.verify_len[b];
  // drafted rows are rho < L <= 32: one lane each
  const bool rej = lane < L && __ldcg(P.w.accepted + r0 + lane) == 0;
  const unsigned m = __ballot_sync(0xffffffffu, rej);
  const int acc = m ? __ffs(m) - 1 : L;
  const int R = r0 + acc;
  if (acc == L) {
    // the bonus draw is made during the residual pass, by the warps that
    // pass leaves idle
    if (lane == 0 && !warm) P.w.blist[atomicAdd(P.w.ctl + kCtlBonus, 1u)] = b;
    return;
  }
  const double M = __ldcg(&P.w.rstat[R].M), W = __ldcg(&P.w.rstat[R].W);
  if (P.recompute) {
    // variant B: the residual kernel weighs the row with its own (shift,
    // factor); its operand row goes to the group's image in the MMA's B
    // layout (K-major, 128-byte swizzle, blocks of 64 rank values gsize rows apart)
    if (warm) return;
    unsigned e = 0;
    if (lane == 0) {
      ResSlot s{};
      s.b = b;
      s.acc = acc;
      s.row = P.w.rowinfo[R].row;
      s.brow = b * a.K + acc;
      s.R = R;
      q_factor(a.lse_q[static_cast<long long>(b) * a.K + acc], &s.mq, &s.fq);
      p_factor(M, W, &s.mp, &s.fp);
      e = atomicAdd(P.w.ctl + kCtlListed, 1u);
      P.w.slots[e] = s;
      P.w.list[e] = b;
    }
    e = __shfl_sync(0xffffffffu, e, 0);
    const int gs = P.res_gsize, gr = static_cast<int>(e) / gs, n = static_cast<int>(e) % gs;
    if (lane < a.r / 8) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.op_rows + (static_cast<long long>(b) * a.K + acc) * a.r) + lane);
      const int kb = lane >> 3, c = lane & 7;
      *reinterpret_cast<uint4*>(a.res_image + static_cast<long long>(gr) * gs * a.r * 2 + kb * (gs * 128) + n * 128 +
                                ((c ^ (n & 7)) << 4)) = v;
    }
    return;
  }
  const float* pm = P.w.part_m + static_cast<long long>(R) * P.nseg;
  float2* rf = P.w.resfac + static_cast<long long>(b) * P.nseg;
  for (int q0 = 0; q0 < P.nseg; q0 += 32 * kRegSeg) {
    float mv[kRegSeg];
#pragma unroll
    for (int j = 0; j < kRegSeg; ++j) {
      const int q = q0 + lane + 32 * j;
      mv[j] = q < P.nseg ? __ldcg(pm + q) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < kRegSeg; ++j) {
      const int q = q0 + lane + 32 * j;
      const float2 f = res_factor(mv[j], M, W);
      if (q < P.nseg && !warm) rf[q] = f;
    }
  }
  if (lane == 0) {
    ResDec d;
    d.acc = acc;
    d.R = R;
    d.row = P.w.rowinfo[R].row;
    q_factor(a.lse_q[static_cast<long long>(b) * a.K + acc], &d.mq, &d.fq);
    if (!warm) {
      P.w.dec[b] = d;
      P.w.list[atomicAdd(P.w.ctl + kCtlListed, 1u)] = b;
    }
  }
}

// Phase 4, one warp: the resampled token of listed request b.
// The resampled token of request b from its residual segment sums; `warm`
// as for sample_p.
__device__ __noinline__ int residual_token(const Params& P, int b, const ResDec& d, float u, int lane, bool warm) {
  const VerifyArgs& a = P.a;
  const double* sw = P.w.seg_w + static_cast<long long>(b) * P.nrseg;
  double rem = 0.0;
  int seg = pick_segment(
      P.nrseg, u, lane, [&](int q) { return __ldcg(sw + q); }, [](double v) { return v; }, &rem);
  if (warm) seg = max(seg, 0);
  int tok;
  if (seg < 0) {
    tok = sample_p(P, d.R, u, lane);  // the residual vanished (rounding): draw from p
  } else {
    const float2 sf = __ldcg(P.w.resfac + static_cast<long long>(b) * P.nseg + seg / 2);
    const long long v0 = static_cast<long long>(seg) * kRSeg;
    const float* x = a.target + d.row * a.V + v0;
    const float* zr = a.z + (static_cast<long long>(b) * a.K + d.acc) * a.V + v0;
    const int n = min(kRSeg, a.V - static_cast<int>(v0));
    constexpr int E = kRSeg / 32;
    float w[E];
#pragma unroll
    for (int k = 0; k < E / 4; ++k) {
      const int e = E * lane + 4 * k;
      const float4 xv = e < n ? __ldcg(reinterpret_cast<const float4*>(x + e)) : neg_inf4();
      const float4 zv = e < n ? __ldcg(reinterpret_cast<const float4*>(zr + e)) : neg_inf4();
      w[4 * k] = res_w(xv.x, zv.x, sf.x, sf.y, d.mq, d.fq);
      w[4 * k + 1] = res_w(xv.y, zv.y, sf.x, sf.y, d.mq, d.fq);
      w[4 * k + 2] = res_w(xv.z, zv.z, sf.x, sf.y, d.mq, d.fq);
      w[4 * k + 3] = res_w(xv.w, zv.w, sf.x, sf.y, d.mq, d.fq);
    }
    int last = -1;
    int k = rescan<E>(n, lane, rem, w, &last);
    if (k < 0) k = max(last, 0);
    tok = static_cast<int>(v0) + k;
  }
  return tok;
}

__device__ __noinline__ void resample(const Params& P, int b, int lane) {
  const ResDec d = P.w.dec[b];
  write_output(P, b, d.acc, residual_token(P, b, d, P.a.u_resample[b], lane, false), lane);
}

// -------------------------------------------------------- consumer bodies
// Segment w of a row item: sum of exp(x - shift) and the drafted token's logit.
__device__ void consume_row(const Params& P, const Desc& ds, const float* stage, uint64_t* empty, int w, int lane) {
  const int off_w = w * kSeg;
  const int nw = min(kSeg, ds.n - off_w);  // <= 0 past the end of the row
  const float* sp = stage + off_w;
  float4 x[kSeg / 128];
#pragma unroll
  for (int k = 0; k < kSeg / 128; ++k) {
    const int e = k * 128 + 4 * lane;
    x[k] = e < nw ? reinterpret_cast<const float4*>(sp)[k * 32 + lane] : neg_inf4();
  }
  const int v_w = ds.g * kRowItem + off_w;
  const bool has_tok = nw > 0 && ds.tok >= v_w && ds.tok < v_w + nw;
  float xt = 0.f;
  if (has_tok && lane == 0) xt = sp[ds.tok - v_w];
  const int R = ds.R, g = ds.g;
  __syncwarp();
  if (lane == 0) mbar_arrive(empty);
  if (nw <= 0) return;
  double S = 0.0;
#pragma unroll
  for (int k = 0; k < kSeg / 128; ++k)
    S += static_cast<double>(group4(p_w(x[k].x, 0.f), p_w(x[k].y, 0.f), p_w(x[k].z, 0.f), p_w(x[k].w, 0.f)));
  S = warp_sum(S);
  float m = 0.f;
  if (!(S >= kSumLo && S <= kSumHi)) {
    float mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < kSeg / 128; ++k) mx = fmaxf(fmaxf(mx, fmaxf(x[k].x, x[k].y)), fmaxf(x[k].z, x[k].w));
    mx = warp_max(mx);
    S = 0.0;
    m = -INFINITY;
    if (mx != -INFINITY) {
      m = __fmul_rn(mx, kLog2e);
#pragma unroll
      for (int k = 0; k < kSeg / 128; ++k)
        S += static_cast<double>(group4(p_w(x[k].x, m), p_w(x[k].y, m), p_w(x[k].z, m), p_w(x[k].w, m)));
      S = warp_sum(S);
    }
  }
  if (lane == 0) {
    const long long idx = static_cast<long long>(R) * P.nseg + g * kCons + w;
    P.w.part_m[idx] = m;
    P.w.part_S[idx] = S;
    if (has_tok) P.w.x_tok[R] = xt;
  }
}

// Segment w of a residual item: sum of max(0, p - q).
__device__ void consume_res(const Params& P, const Desc& ds, const float* stage, uint64_t* empty, int w, int lane) {
  const int off_w = w * kRSeg;
  const int nw = min(kRSeg, ds.n - off_w);
  const float* sp = stage + off_w;
  const float* sz = stage + kResItem + off_w;
  float4 x[kRSeg / 128], z[kRSeg / 128];
#pragma unroll
  for (int k = 0; k < kRSeg / 128; ++k) {
    const int e = k * 128 + 4 * lane;
    x[k] = e < nw ? reinterpret_cast<const float4*>(sp)[k * 32 + lane] : neg_inf4();
    z[k] = e < nw ? reinterpret_cast<const float4*>(sz)[k * 32 + lane] : neg_inf4();
  }
  const float sh = ds.shift[w / 2], f = ds.f[w / 2], mq = ds.mq, fq = ds.fq;
  const int b = ds.b, g = ds.g;
  __syncwarp();
  if (lane == 0) mbar_arrive(empty);
  if (nw <= 0) return;
  double S = 0.0;
#pragma unroll
  for (int k = 0; k < kRSeg / 128; ++k)
    S += static_cast<double>(group4(res_w(x[k].x, z[k].x, sh, f, mq, fq), res_w(x[k].y, z[k].y, sh, f, mq, fq),
                                    res_w(x[k].z, z[k].z, sh, f, mq, fq), res_w(x[k].w, z[k].w, sh, f, mq, fq)));
  S = warp_sum(S);
  if (lane == 0) P.w.seg_w[static_cast<long long>(b) * P.nrseg + g * kCons + w] = S;
}

// ------------------------------------------------------------ main kernel
struct Smem {
  uint64_t full[kStages], empty[kStages];
  Desc desc[kStages];
  int abort;
};

// Device-wide barrier k (bounded): every thread's earlier writes are visible
// to every thread after it. Called between streaming phases, with no copy in
// flight.
__device__ bool grid_barrier(const Params& P, int k, int* s_flag) {
  // The CTA barrier orders every thread's writes before thread 0's release
  // reduction (gpu scope), and thread 0's acquire loads before every thread's
  // later reads; separate gpu fences would only add microseconds.
  __syncthreads();
  if (threadIdx.x == 0) {
    // (test hook: one CTA may skip its arrival at the first barrier so that
    // every CTA's wait runs out)
    if (!(k == 0 && injected_stall(P.a.err, DSPARK_INJECT_VERIFY_BARRIER, blockIdx.x)))
      red_release_gpu_add(P.w.ctl + kCtlBar + k, 1u);
    const bool ok = wait_at_least(P.w.ctl + kCtlBar + k, gridDim.x, P.a.err, 0x500u + k);
    *s_flag = ok ? 1 : 0;
  }
  __syncthreads();
  return *s_flag != 0;
}

// kRecompute: variant B (P.recompute), as a template so that variant A's
// kernel carries none of its code
template <bool kRecompute>
__global__ void __launch_bounds__(kThreads, 1) verify_kernel(const __grid_constant__ Params P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  float* stages = reinterpret_cast<float*>(smem);
  Smem& S = *reinterpret_cast<Smem*>(smem + kStages * kStageBytes);
  __shared__ int s_flag;
  __shared__ volatile int s_sink;
  const VerifyArgs& a = P.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;
  // warp-per-unit phases: unit u goes to CTA u % G, warp u / G, so that
  // consecutive units (rows, requests) land on different SMs
  const int gw = warp * G + c, NW = G * kWarps;
  volatile int* abort = &S.abort;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], kCons);
    }
    S.abort = 0;
    fence_mbar_init();
  }
  // the plan kernel's results (programmatic dependent launch; a no-op when
  // launched without it)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __syncthreads();
  const int n_rows = static_cast<int>(P.w.ctl[kCtlRows]);
  // producer: items issued; consumer group g: index of its next item
  uint32_t seq = warp < kProdWarp ? static_cast<uint32_t>(warp / kCons) : 0u;

  // One streaming phase: the producer issues this CTA's items (fill(item,
  // desc, dst, full) fills the descriptor and starts the copies), then one
  // exit marker per consumer group; consumers reduce the items.
  auto stream = [&](long long n_items, auto fill, auto consume) -> bool {
    if (warp == kProdWarp) {
      bool ok = true;
      auto claim = [&](int* s) -> bool {
        *s = seq % kStages;
        return __all_sync(0xffffffffu, mbar_wait(&S.empty[*s], ((seq / kStages) & 1u) ^ 1u, abort, a.err, 0x402u));
      };
      for (long long item = c; ok && item < n_items; item += G) {
        int s;
        ok = claim(&s);
        if (!ok) break;
        if (lane == 0) fill(item, S.desc[s], stages + static_cast<size_t>(s) * kRowItem, &S.full[s]);
        ++seq;
      }
      for (int k = 0; ok && k < kGroups; ++k) {
        int s;
        ok = claim(&s);
        if (!ok) break;
        if (lane == 0) {
          S.desc[s].type = kItemExit;
          mbar_arrive(&S.full[s]);
        }
        ++seq;
      }
      if (!ok && lane == 0) *abort = 1;
      return ok;
    }
    if (warp < kProdWarp) {
      const int w = warp % kCons;
      for (;; seq += kGroups) {
        const int s = seq % kStages;
        // every lane waits: a warp left waiting on one lane runs its next
        // collective code diverged and several times slower
        if (!__all_sync(0xffffffffu, mbar_wait(&S.full[s], (seq / kStages) & 1u, abort, a.err, 0x400u))) return false;
        const Desc& ds = S.desc[s];
        if (ds.type == kItemExit) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.empty[s]);
          seq += kGroups;
          return true;
        }
        consume(ds, stages + static_cast<size_t>(s) * kRowItem, &S.empty[s], w);
      }
    }
    return true;
  };

  // ---- phase 1: target rows
  const long long n_row_items = static_cast<long long>(n_rows) * P.ngrp;
  bool ok = stream(
      n_row_items,
      [&](long long item, Desc& ds, float* dst, uint64_t* full) {
        const int R = static_cast<int>(item / P.ngrp), g = static_cast<int>(item % P.ngrp);
        const RowInfo ri = P.w.rowinfo[R];
        const int v0 = g * kRowItem, n = min(kRowItem, a.V - v0);
        ds.type = kItemRow;
        ds.b = ri.brl & 0xffff;
        ds.R = R;
        ds.g = g;
        ds.n = n;
        ds.tok = ri.tok;
        const uint32_t bytes = static_cast<uint32_t>(n) * 4u;
        mbar_arrive_expect_tx(full, bytes);
        // variant B: evict-first, so that the draft's Bf (evict-last) stays in
        // L2 for the residual kernel that follows
        if (kRecompute) bulk_load_hint(dst, a.target + ri.row * a.V + v0, bytes, full, policy_evict_first());
        else bulk_load(dst, a.target + ri.row * a.V + v0, bytes, full);
      },
      [&](const Desc& ds, const float* stage, uint64_t* empty, int w) { consume_row(P, ds, stage, empty, w, lane); });
  // the spare warps run the later phases' code once while the rows stream, so
  // that those phases do not start on a cold instruction cache
  if (warp > kProdWarp && n_rows > 0) {
    int r = 0;
    if (warp == kProdWarp + 1) r = sample_p(P, 0, 0.5f, lane, true);
    if (warp == kProdWarp + 2 && !kRecompute) {
      ResDec d{};
      d.row = P.w.rowinfo[0].row;
      r = residual_token(P, 0, d, 0.5f, lane, true);
    }
    if (warp == kProdWarp + 3) {
      row_stats(P, 0, lane);  // rewritten in phase 2
      decide(P, 0, lane, true);
    }
    if (lane == 0) s_sink = r;
  }
  ok = __syncthreads_and(ok) && grid_barrier(P, 0, &s_flag);

  // ---- phase 2: row statistics and accept tests; the warp that completes
  // the last row of a request makes its decision (the bonus and residual
  // lists), so no device-wide barrier separates the two
  if (ok)
    for (int R = gw; R < n_rows; R += NW) {
      row_stats(P, R, lane);
      const int brl = P.w.rowinfo[R].brl;
      const int b = brl & 0xffff, L = brl >> 22;
      unsigned done = 0;
      if (lane == 0) done = atom_add_acq_rel_gpu(P.w.req_rows + b, 1u);  // releases this row's results
      if (__shfl_sync(0xffffffffu, done, 0) == static_cast<unsigned>(L)) {
        // every lane acquires the request's other rows before reading them
        (void)ld_acquire_gpu(P.w.req_rows + b);
        decide(P, b, lane);
      }
    }
  ok = ok && grid_barrier(P, 2, &s_flag);

  // variant B: the bonus draws, one warp per request; the residual kernel
  // that follows does the rest
  if (kRecompute) {
    if (ok) {
      const int n_bonus = static_cast<int>(__ldcg(P.w.ctl + kCtlBonus));
      for (int e = gw; e < n_bonus; e += NW) {
        const int b = __ldcg(P.w.blist + e);
        const int L = a.verify_len[b];
        write_output(P, b, L, sample_p(P, P.w.rowbase[b] + L, a.u_resample[b], lane), lane);
      }
    }
  } else {
    // ---- phase 3: residual segment sums of the listed requests
    const int n_listed = ok ? static_cast<int>(__ldcg(P.w.ctl + kCtlListed)) : 0;
    if (ok) {
      const uint64_t pol_first = policy_evict_first();
      ok = stream(
          static_cast<long long>(n_listed) * P.nrgrp,
          [&](long long item, Desc& ds, float* dst, uint64_t* full) {
            const int e = static_cast<int>(item / P.nrgrp), g = static_cast<int>(item % P.nrgrp);
            const int b = __ldcg(P.w.list + e);
            const ResDec d = P.w.dec[b];
            const int v0 = g * kResItem, n = min(kResItem, a.V - v0);
            ds.type = kItemRes;
            ds.b = b;
            ds.R = d.R;
            ds.g = g;
            ds.n = n;
            ds.tok = -1;
  #pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int q = g * 4 + i;
              const float2 f =
                  q < P.nseg ? __ldcg(P.w.resfac + static_cast<long long>(b) * P.nseg + q) : make_float2(0.f, 0.f);
              ds.shift[i] = f.x;
              ds.f[i] = f.y;
            }
            ds.mq = d.mq;
            ds.fq = d.fq;
            const uint32_t bytes = static_cast<uint32_t>(n) * 4u;
            mbar_arrive_expect_tx(full, 2u * bytes);
            bulk_load(dst, a.target + d.row * a.V + v0, bytes, full);
            bulk_load_hint(dst + kResItem, a.z + (static_cast<long long>(b) * a.K + d.acc) * a.V + v0, bytes, full,
                           pol_first);
          },
          [&](const Desc& ds, const float* stage, uint64_t* empty, int w) { consume_res(P, ds, stage, empty, w, lane); });
      // meanwhile the warps outside the stream make the bonus draws
      if (warp > kProdWarp) {
        const int n_bonus = static_cast<int>(__ldcg(P.w.ctl + kCtlBonus));
        const int nsw = (kWarps - kProdWarp - 1) * G;
        for (int e = (warp - kProdWarp - 1) * G + c; e < n_bonus; e += nsw) {
          const int b = __ldcg(P.w.blist + e);
          const int L = a.verify_len[b];
          const int tok = sample_p(P, P.w.rowbase[b] + L, a.u_resample[b], lane);
          write_output(P, b, L, tok, lane);
        }
      }
      ok = __syncthreads_and(ok) && grid_barrier(P, 3, &s_flag);
    }

    // ---- phase 4: resampled tokens
    if (ok)
      for (int e = gw; e < n_listed; e += NW) resample(P, __ldcg(P.w.list + e), lane);
  }

  // copies still in flight (after an abort) land before the CTA exits
  __syncthreads();
  if (warp == kProdWarp && lane == 0)
    for (uint32_t q = seq > kStages ? seq - kStages : 0; q < seq; ++q)
      mbar_drain(&S.full[q % kStages], (q / kStages) & 1u, a.err, 0x405u);
}

struct Layout {
  size_t rowinfo, rowbase, ctl, part_m, part_S, x_tok, rstat, accepted, dec, resfac, list, blist, seg_w, slots, req_rows,
      total;
};

Layout verify_layout(int B, int K, int V) {
  const size_t nseg = (V + kSeg - 1) / kSeg, nrseg = (V + kRSeg - 1) / kRSeg;
  const size_t rows = static_cast<size_t>(B) * (K + 1), nb = static_cast<size_t>(B);
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  L.rowinfo = take(rows * sizeof(RowInfo));
  L.rowbase = take(nb * sizeof(int));
  L.ctl = take(kCtlCount * sizeof(unsigned));
  L.part_m = take(rows * nseg * sizeof(float));
  L.part_S = take(rows * nseg * sizeof(double));
  L.x_tok = take(rows * sizeof(float));
  L.rstat = take(rows * sizeof(RowStat));
  L.accepted = take(rows * sizeof(int));
  L.dec = take(nb * sizeof(ResDec));
  L.resfac = take(nb * nseg * sizeof(float2));
  L.list = take(nb * sizeof(int));
  L.blist = take(nb * sizeof(int));
  L.seg_w = take(nb * nrseg * sizeof(double));
  L.slots = take(nb * sizeof(ResSlot));
  L.req_rows = take(nb * sizeof(unsigned));
  L.total = off;
  return L;
}

}  // namespace

size_t verify_scratch_bytes(int B, int K, int V) { return verify_layout(B, K, V).total; }

cudaError_t launch_verify(VerifyArgs a, char* region, cudaStream_t stream) {
  Params P{};
  P.a = a;
  P.nseg = (a.V + kSeg - 1) / kSeg;
  P.nrseg = (a.V + kRSeg - 1) / kRSeg;
  P.ngrp = (a.V + kRowItem - 1) / kRowItem;
  P.nrgrp = (a.V + kResItem - 1) / kResItem;
  const Layout L = verify_layout(a.B, a.K, a.V);
  P.w.rowinfo = reinterpret_cast<RowInfo*>(region + L.rowinfo);
  P.w.rowbase = reinterpret_cast<int*>(region + L.rowbase);
  P.w.ctl = reinterpret_cast<unsigned*>(region + L.ctl);
  P.w.part_m = reinterpret_cast<float*>(region + L.part_m);
  P.w.part_S = reinterpret_cast<double*>(region + L.part_S);
  P.w.x_tok = reinterpret_cast<float*>(region + L.x_tok);
  P.w.rstat = reinterpret_cast<RowStat*>(region + L.rstat);
  P.w.accepted = reinterpret_cast<int*>(region + L.accepted);
  P.w.dec = reinterpret_cast<ResDec*>(region + L.dec);
  P.w.resfac = reinterpret_cast<float2*>(region + L.resfac);
  P.w.list = reinterpret_cast<int*>(region + L.list);
  P.w.blist = reinterpret_cast<int*>(region + L.blist);
  P.w.seg_w = reinterpret_cast<double*>(region + L.seg_w);
  P.w.slots = reinterpret_cast<ResSlot*>(region + L.slots);
  P.w.req_rows = reinterpret_cast<unsigned*>(region + L.req_rows);
  P.recompute = a.z == nullptr ? 1 : 0;
  P.res_gsize = residual_group_size(a.B);

  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const size_t smem = static_cast<size_t>(kStages) * kStageBytes + sizeof(Smem);
  auto kernel = P.recompute ? verify_kernel<true> : verify_kernel<false>;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  {
    cudaLaunchAttribute pattr[1];
    pattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pattr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t pcfg{};
    pcfg.gridDim = dim3(1);
    pcfg.blockDim = dim3(kPlanThreads);
    pcfg.stream = stream;
    pcfg.attrs = pattr;
    pcfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&pcfg, verify_plan_kernel, P);
    if (e == cudaErrorNotSupported) {  // without the early launch
      (void)cudaGetLastError();
      pcfg.numAttrs = 0;
      e = cudaLaunchKernelEx(&pcfg, verify_plan_kernel, P);
    }
    if (e != cudaSuccess) return e;
  }
  const long long rows = static_cast<long long>(a.B) * (a.K + 1);
  const long long units = std::max(rows * P.ngrp, (rows + kWarps - 1) / kWarps);
  const int G = static_cast<int>(std::min<long long>(sms, std::max<long long>(1, units)));
  // cooperative, and allowed to start while the plan kernel runs
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kernel, P);
  if (e == cudaErrorNotSupported) {  // without the early start
    (void)cudaGetLastError();
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kernel, P);
  }
  if (e != cudaSuccess || !P.recompute) return e;
  return launch_residual_tc(P, stream);
}

}  // namespace dspark
