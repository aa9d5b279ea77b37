// Residual draw of variant B on the 5th-generation tensor cores.
//
// wangjunjian.com tag page, article "Speculative Decoding", steps 3-5, and the
// QbitAI article "DSpark: ten concepts are enough", section "speculative
// decoding": at the first rejected draft the token is drawn from
// max(0, p - q) renormalised. Variant B of the round stores no draft logits,
// so q = softmax(z) of that one row is recomputed here: z = base + a . Bf, with
// a the operand row the draft used at that position (the A row of the previous
// token, or the RNN state rounded to bf16). One pass over Bf with the requests
// that need a residual as the MMA's N dimension (groups of up to 128), fused
// with the residual weights, their fp64 sums over 32-row units and over each
// CTA's slice, and a three-level inverse-CDF draw; the bias GEMM is the
// draft's, on the same tiles, so z is the draft's z up to the order of the
// tensor core's fp32 accumulation.
//
// One persistent cooperative CTA per SM, CTA g owning the vocabulary slice
// chunk_bounds(V, 32, G, g) as in the draft. Warp roles:
//   warps 0-7  epilogue, two per TMEM lane quadrant: stage 16-request boxes of
//              the base and target logits of their rows with cp.async (the
//              rows are scattered, one per request), read the accumulator and
//              weigh w = max(0, p - q) in fp32, with p = 2^(x log2 e - mp) fp
//              and q = 2^(z log2 e - mq) fq as in the verify kernel; w is
//              summed in fp64 over each 32-row unit and over the slice;
//   warp 8     TMA producer of Bf tiles;
//   warp 9     TMEM owner and MMA issuer;
//   warp 10    selector: publishes the slice sums and draws the tokens of the
//              group's requests e (list order) with e mod G == g: the G slice
//              sums, the chosen slice's unit sums, then the unit's 32 weights
//              with its z recomputed (the unit's Bf columns staged in shared
//              memory). A residual that sums to zero falls back to a draw from p.
// At the start of each group the epilogue warps and the selector copy the
// group's operand rows into the MMA's B layout in shared memory. Every wait is
// bounded and reports DSPARK_ERR_TIMEOUT.
#include <algorithm>

#include "common.cuh"
#include "draft_common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "verify_common.cuh"

namespace dspark {
namespace vfy {
namespace {

constexpr int kEpiWarps = 8;                  // two per TMEM lane quadrant
constexpr int kRsProdWarp = kEpiWarps;
constexpr int kRsMmaWarp = kEpiWarps + 1;
constexpr int kRsSelWarp = kEpiWarps + 2;
constexpr int kRsThreads = (kEpiWarps + 3) * 32;
constexpr int kBuildThreads = (kEpiWarps + 1) * 32;  // epilogue warps and the selector
constexpr int kBuildBar = 1;                  // named barrier of the operand build
constexpr int kUnit = 32;
constexpr int kTileRows = 128;                // MMA M
constexpr int kKStage = 64;                   // r per Bf stage
constexpr int kMaxBfStages = 8;
constexpr int kBfBoxBytes = 64 * kKStage * 2;
constexpr int kBfStageBytes = 2 * kBfBoxBytes;
constexpr int kSub = 16;                      // requests per TMEM load and per box
constexpr int kBoxFloats = kSub * kUnit;      // one box of base or of target logits
constexpr int kSlotBytes = 2 * kBoxFloats * 4;
constexpr int kMaxGroup = 128;
constexpr int kMaxGroups = 4;
constexpr int kMaxAccSlots = 8;
constexpr uint32_t kTmemCols = 512;
constexpr int kSubPerWarp = kMaxGroup / kSub / 2;

// Per-request constants of the current group, in shared memory.
struct Col {
  long long base_off;    // (b K + acc) V: the base row
  long long target_off;  // row V: the target row
  float mq, fq, mp, fp;
};

struct RsParams {
  Params P;           // the verify kernel's state: slots, counters, row statistics
  int gsize;          // requests per group (multiple of 32, <= 128)
  int r_stages;
  int slot_stride;    // TMEM columns per accumulator slot
  int nslots;
  int nbf, nbs;       // Bf stages; staging slots per epilogue warp
};

struct RsLayout {
  int bf, img, ring, sel, col, part, bar, misc, total;
};

__host__ __device__ inline RsLayout rs_layout(int nbf, int gsize, int r, int nbs) {
  RsLayout L;
  L.bf = 0;
  L.img = nbf * kBfStageBytes;
  L.ring = L.img + ((gsize * r * 2 + 1023) / 1024) * 1024;
  L.sel = L.ring + kEpiWarps * nbs * kSlotBytes;  // the last search level's unit of Bf and operand row
  L.col = L.sel + ((r * kUnit * 2 + r * 2 + 127) / 128) * 128;
  L.part = L.col + kMaxGroup * static_cast<int>(sizeof(Col));
  L.bar = L.part + 4 * gsize * 8;
  L.misc = L.bar + 64 * 8;
  L.total = L.misc + 64;
  return L;
}

struct RsBars {
  uint64_t* q;
  __device__ uint64_t* bf_full(int s) const { return q + s; }
  __device__ uint64_t* bf_empty(int s) const { return q + kMaxBfStages + s; }
  __device__ uint64_t* acc_full(int s) const { return q + 2 * kMaxBfStages + s; }
  __device__ uint64_t* acc_empty(int s) const { return q + 2 * kMaxBfStages + kMaxAccSlots + s; }
  __device__ uint64_t* img_full() const { return q + 2 * kMaxBfStages + 2 * kMaxAccSlots; }
  __device__ uint64_t* step_done() const { return img_full() + 1; }
  __device__ uint64_t* final_mma() const { return img_full() + 2; }
  __device__ uint64_t* mma_done() const { return img_full() + 3; }
};

__device__ __forceinline__ int rs_round16(int n) { return (n + 15) & ~15; }
__device__ __forceinline__ int group_real(int n_listed, int gsize, int gr) { return min(gsize, n_listed - gr * gsize); }
// sub-chunks s (16 requests) of a group with s % 2 == hh among its ncol columns
__device__ __forceinline__ int chunks_for2(int ncol, int hh) {
  const int nsub = (ncol + kSub - 1) / kSub;
  return nsub > hh ? (nsub - hh + 1) / 2 : 0;
}
// passes over the slice alternate direction, so each group starts on the Bf
// tiles the previous one touched last
__device__ __forceinline__ int rs_tile(int gr, int ntiles, int t) { return (gr & 1) ? ntiles - 1 - t : t; }

__device__ __forceinline__ void bar_build() {
  asm volatile("bar.sync %0, %1;" ::"n"(kBuildBar), "n"(kBuildThreads) : "memory");
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "l"(policy)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait(int pending) {
  switch (pending) {
    case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
  }
}

// The per-request constants of group gr, written by the epilogue warps and
// the selector together (thread index tid < kBuildThreads). Both
// barriers are reached by every participant for every group, also after an
// abort, so that none is left waiting. (The operand rows arrive separately:
// the verify kernel left them in the MMA's layout, which the MMA warp loads.)
__device__ void build_group(const RsParams& rp, int gr, int n_listed, Col* col, int tid, bool ok) {
  const Params& P = rp.P;
  const VerifyArgs& a = P.a;
  bar_build();  // the previous group's accumulators are read out and its sums published
  const int nreal = group_real(n_listed, rp.gsize, gr), N = rs_round16(nreal);
  if (ok)
    for (int n = tid; n < N; n += kBuildThreads) {
      ResSlot S{};
      if (n < nreal) S = P.w.slots[gr * rp.gsize + n];
      Col cl;
      cl.base_off = static_cast<long long>(S.brow) * a.V;
      cl.target_off = S.row * a.V;
      cl.mq = S.mq;
      cl.fq = S.fq;
      cl.mp = S.mp;
      cl.fp = S.fp;
      col[n] = cl;
    }
  bar_build();
}

// The resampled token of list entry e (one warp): slice sums, the chosen
// slice's unit sums, then the chosen unit's 32 weights with z recomputed from
// the unit's Bf columns (staged in `sel` in one memory trip) and the operand row.
// With `warm` set the whole path runs on whatever the arrays hold and its
// result is dropped: it loads the code into the SM's instruction cache while
// the group streams, ahead of the draws.
__device__ __noinline__ int residual_draw(const RsParams& rp, int e, const ResSlot& S, double u, int G, int lane,
                                          uint8_t* sel, bool warm) {
  const Params& P = rp.P;
  const VerifyArgs& a = P.a;
  const double* part = a.res_part + static_cast<long long>(e) * G;
  double ex, W;
  const int c = warp_search<8>(
      G, [&](int cc) { return __ldcg(part + cc); }, [&](double tot) { return u * tot; }, lane, &ex, &W);
  if (!warm && (!(W > 0.0) || !(W < INFINITY))) return sample_p(P, S.R, static_cast<float>(u), lane);  // vanished
  const double R = u * W - ex;
  int lo, hi;
  chunk_bounds(a.V, kUnit, G, c, &lo, &hi);
  const int ulo = lo / kUnit;
  const double* us = a.res_unit + static_cast<long long>(ulo) * a.B + e;
  double ex2, tot2;
  const int ux = ulo + warp_search<2>(
                           (hi - lo) / kUnit, [&](int k) { return __ldcg(us + static_cast<long long>(k) * a.B); },
                           [&](double) { return R; }, lane, &ex2, &tot2);
  const double R2 = R - ex2;
  const long long v0 = static_cast<long long>(ux) * kUnit;
  stage_unit_issue(sel, static_cast<const uint16_t*>(a.Bf), a.V, a.r, v0, lane);
  const float zb = __ldcg(a.base + static_cast<long long>(S.brow) * a.V + v0 + lane);
  const float x = __ldcg(a.target + S.row * a.V + v0 + lane);
  uint4* a_s = reinterpret_cast<uint4*>(sel + a.r * kUnit * 2);
  if (lane < a.r / 8)
    a_s[lane] = __ldcg(reinterpret_cast<const uint4*>(a.op_rows + static_cast<long long>(S.brow) * a.r) + lane);
  stage_unit_wait();
  const float z = __fadd_rn(zb, staged_unit_dot(reinterpret_cast<const uint16_t*>(sel), a_s, a.r, lane));
  __syncwarp();  // every lane has read the staging before the next load
  const double w = static_cast<double>(res_w(x, z, S.mp, S.fp, S.mq, S.fq));
  const double inc = warp_inclusive_scan(w);
  const unsigned hit = __ballot_sync(0xffffffffu, inc > R2 && w > 0.0);
  const unsigned pos = __ballot_sync(0xffffffffu, w > 0.0);
  // rounding: the last positive weight of the unit
  const int k = hit ? __ffs(hit) - 1 : (pos ? 31 - __clz(pos) : 0);
  if (warm) return sample_p(P, S.R, static_cast<float>(u), lane, true);
  return static_cast<int>(v0) + k;
}

__global__ void __launch_bounds__(kRsThreads, 1)
    residual_tc_kernel(const __grid_constant__ RsParams rp, const __grid_constant__ CUtensorMap tm_bf) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Params& P = rp.P;
  const VerifyArgs& a = P.a;
  const RsLayout Ly = rs_layout(rp.nbf, rp.gsize, a.r, rp.nbs);
  RsBars bars{reinterpret_cast<uint64_t*>(smem + Ly.bar)};
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + Ly.misc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + Ly.misc + 4);
  Col* col = reinterpret_cast<Col*>(smem + Ly.col);
  __shared__ volatile int s_sink;
  double* s_part = reinterpret_cast<double*>(smem + Ly.part);  // [quadrant][gsize]
  uint8_t* img = smem + Ly.img;  // the group's operand rows: blocks of 64 rank values, gsize rows apart

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, g = blockIdx.x;
  int lo, hi;
  chunk_bounds(a.V, kUnit, G, g, &lo, &hi);
  const int ntiles = (hi - lo + kTileRows - 1) / kTileRows;
  const int last_rows = (hi - lo) - (ntiles - 1) * kTileRows;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxBfStages; ++s) {
      mbar_init(bars.bf_full(s), 1);
      mbar_init(bars.bf_empty(s), 1);
    }
    for (int s = 0; s < kMaxAccSlots; ++s) {
      mbar_init(bars.acc_full(s), 1);
      mbar_init(bars.acc_empty(s), kEpiWarps);
    }
    mbar_init(bars.img_full(), 1);
    mbar_init(bars.step_done(), kEpiWarps);
    mbar_init(bars.final_mma(), 1);
    mbar_init(bars.mma_done(), 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == kRsMmaWarp) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  // the verify kernel's lists and row statistics (programmatic dependent
  // launch; a no-op when launched without it)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int n_listed = min(static_cast<int>(__ldcg(P.w.ctl + kCtlListed)), a.B);
  const int ngroups = (n_listed + rp.gsize - 1) / rp.gsize;

  if (warp == kRsProdWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_bf);
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_parity[kMaxBfStages];
      bool issued[kMaxBfStages];
      for (int s = 0; s < kMaxBfStages; ++s) issued[s] = false;
      bool ok = true;
      for (int gr = 0; ok && gr < ngroups; ++gr)
        for (int t = 0; ok && t < ntiles; ++t)
          for (int s = 0; s < rp.r_stages; ++s) {
            if (!mbar_wait(bars.bf_empty(stage), phase ^ 1u, s_abort, a.err, 0x800u)) {
              ok = false;
              break;
            }
            uint8_t* dst = smem + Ly.bf + stage * kBfStageBytes;
            const int pt = rs_tile(gr, ntiles, t);
            const int v0 = lo + pt * kTileRows;
            const bool both = (pt == ntiles - 1 ? last_rows : kTileRows) > 64;
            mbar_arrive_expect_tx(bars.bf_full(stage), both ? kBfStageBytes : kBfBoxBytes);
            tma_load_2d(dst, &tm_bf, v0, s * kKStage, bars.bf_full(stage), pol);
            if (both) tma_load_2d(dst + kBfBoxBytes, &tm_bf, v0 + 64, s * kKStage, bars.bf_full(stage), pol);
            issued[stage] = true;
            issued_parity[stage] = phase;
            if (++stage == rp.nbf) {
              stage = 0;
              phase ^= 1u;
            }
          }
      if (!ok) *s_abort = 1;
      for (int s = 0; s < rp.nbf; ++s)
        if (issued[s]) mbar_drain(bars.bf_full(s), issued_parity[s], a.err, 0x801u);
    }
  } else if (warp == kRsMmaWarp) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      int stage = 0, slot = 0;
      uint32_t phase = 0, slot_phase = 0;
      const uint32_t img_addr = smem_u32(img);
      const uint32_t bf_addr = smem_u32(smem + Ly.bf);
      const uint32_t img_bytes = static_cast<uint32_t>(rp.gsize * a.r * 2);
      fence_proxy_async_all();  // the verify kernel wrote the images with ordinary stores
      bool ok = true;
      for (int gr = 0; ok && gr < ngroups; ++gr) {
        const int N = rs_round16(group_real(n_listed, rp.gsize, gr));
        const uint32_t idesc = idesc_bf16_f32(N, 1);
        // the image is free once the previous group's MMAs are done
        if (gr > 0) {
          mma_commit(bars.mma_done());
          if (!mbar_wait(bars.mma_done(), (gr - 1) & 1, s_abort, a.err, 0x814u)) {
            ok = false;
            break;
          }
        }
        mbar_arrive_expect_tx(bars.img_full(), img_bytes);
        bulk_load(img, a.res_image + static_cast<long long>(gr) * img_bytes, img_bytes, bars.img_full());
        if (!mbar_wait(bars.img_full(), gr & 1, s_abort, a.err, 0x810u)) {
          mbar_drain(bars.img_full(), gr & 1, a.err, 0x815u);  // the copy lands before the CTA can exit
          ok = false;
          break;
        }
        tc_fence_after();
        for (int t = 0; ok && t < ntiles; ++t) {
          if (!mbar_wait(bars.acc_empty(slot), slot_phase ^ 1u, s_abort, a.err, 0x811u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dcol = tmem_base + static_cast<uint32_t>(slot * rp.slot_stride);
          for (int s = 0; s < rp.r_stages; ++s) {
            if (!mbar_wait(bars.bf_full(stage), phase, s_abort, a.err, 0x812u)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_base = bf_addr + stage * kBfStageBytes;
            const uint32_t b_base = img_addr + s * (rp.gsize * 128);
#pragma unroll
            for (int kk = 0; kk < kKStage / 16; ++kk) {
              const uint64_t adesc = smem_desc_sw128(a_base + kk * 2048, kBfBoxBytes, 1024);
              const uint64_t bdesc = smem_desc_sw128(b_base + kk * 32, 16, 1024);
              mma_bf16(dcol, adesc, bdesc, idesc, (s | kk) != 0);
            }
            mma_commit(bars.bf_empty(stage));
            if (++stage == rp.nbf) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          mma_commit(bars.acc_full(slot));
          if (++slot == rp.nslots) {
            slot = 0;
            slot_phase ^= 1u;
          }
        }
      }
      if (!ok) *s_abort = 1;
      // all issued MMAs complete before TMEM is released
      mma_commit(bars.final_mma());
      mbar_drain(bars.final_mma(), 0, a.err, 0x813u);
    }
  } else if (warp == kRsSelWarp) {
    // ------------------------------------------------------------ selector
    bool ok = true;
    const int tid = kEpiWarps * 32 + lane;
    // The draws of group gr's requests e (list order) with e mod G == g. What
    // does not depend on the other CTAs (the slot, the uniform, the accepted
    // drafts) is read before the wait for their slice sums.
    auto search = [&](int gr) {
      const int e0 = gr * rp.gsize, nreal = group_real(n_listed, rp.gsize, gr);
      const int first = e0 + ((g - e0) % G + G) % G;
      if (!ok || first >= e0 + nreal) return;
      ResSlot S = P.w.slots[first];
      double u = static_cast<double>(a.u_resample[S.b]);
      int drafted = lane < S.acc ? a.tokens[static_cast<long long>(S.b) * a.K + lane] : 0;
      if (!__all_sync(0xffffffffu, wait_at_least(P.w.ctl + kCtlRes + gr, static_cast<unsigned>(G), a.err,
                                                  0x820u + gr))) {
        ok = false;
        return;
      }
      for (int e = first; e < e0 + nreal; e += G) {
        if (e != first) {
          S = P.w.slots[e];
          u = static_cast<double>(a.u_resample[S.b]);
          drafted = lane < S.acc ? a.tokens[static_cast<long long>(S.b) * a.K + lane] : 0;
        }
        const int tok = residual_draw(rp, e, S, u, G, lane, smem + Ly.sel, false);
        // the accepted drafts (acc < L_b <= K <= 32, one per lane), the token, then -1
        int32_t* out = a.out_tokens + static_cast<long long>(S.b) * (a.K + 1);
        if (lane <= a.K) out[lane] = lane < S.acc ? drafted : (lane == S.acc ? tok : -1);
        if (lane == 0 && a.K == 32) out[32] = -1;
        if (lane == 0) {
          a.accepted[S.b] = S.acc;
          a.n_out[S.b] = S.acc + 1;
        }
      }
    };
    for (int gr = 0; gr < ngroups; ++gr) {
      build_group(rp, gr, n_listed, col, tid, ok);
      // the previous group's draws run while this group streams
      if (gr > 0) search(gr - 1);
      // the draw's code into the instruction cache, on entry 0's real (if
      // stale) sums, while the first group streams
      if (gr == 0 && ok) {
        const ResSlot S0 = P.w.slots[0];
        s_sink = residual_draw(rp, 0, S0, 0.5, G, lane, smem + Ly.sel, true);
      }
      if (ok && !mbar_wait(bars.step_done(), gr & 1, s_abort, a.err, 0x821u)) ok = false;
      if (ok) {
        const int e0 = gr * rp.gsize, nreal = group_real(n_listed, rp.gsize, gr);
        for (int n = lane; n < nreal; n += 32) {
          const double S = s_part[n] + s_part[rp.gsize + n] + s_part[2 * rp.gsize + n] + s_part[3 * rp.gsize + n];
          a.res_part[static_cast<long long>(e0 + n) * G + g] = S;
        }
        // (test hook: one CTA may skip its publish of the first group so that
        // the other CTAs' waits run out)
        __syncwarp();
        if (lane == 0 && !(gr == 0 && injected_stall(a.err, DSPARK_INJECT_RESIDUAL_SLICE_SUMS, g)))
          red_release_gpu_add(P.w.ctl + kCtlRes + gr, 1u);
      }
    }
    if (ngroups > 0) search(ngroups - 1);
    if (!ok) *s_abort = 1;
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3, h = warp >> 2;
    const uint64_t pol_first = policy_evict_first();
    float* ring = reinterpret_cast<float*>(smem + Ly.ring + warp * rp.nbs * kSlotBytes);
    int slot = 0;
    uint32_t slot_phase = 0;
    bool ok = true;
    for (int gr = 0; gr < ngroups; ++gr) {
      build_group(rp, gr, n_listed, col, threadIdx.x, ok && *s_abort == 0);
      if (!ok) continue;
      const int e0 = gr * rp.gsize, nreal = group_real(n_listed, rp.gsize, gr);
      const int hh = (h + gr) & 1;
      const int nk = chunks_for2(nreal, hh);
      // items (tile t, sub-chunk kk) in consumption order; item n's boxes go to
      // staging slot n % nbs, one cp.async group per item
      auto rows_of = [&](int t) { return rs_tile(gr, ntiles, t) == ntiles - 1 ? last_rows : kTileRows; };
      int it_t = 0, it_k = 0;  // next item to load
      auto advance = [&]() {
        while (it_t < ntiles && (it_k >= nk || kUnit * q >= rows_of(it_t))) {
          it_k = 0;
          ++it_t;
        }
      };
      advance();
      int nl = 0;
      auto load_next = [&]() {
        if (it_t < ntiles) {
          float* dst = ring + (nl % rp.nbs) * (2 * kBoxFloats);
          const int v0 = lo + rs_tile(gr, ntiles, it_t) * kTileRows + kUnit * q;
          const int col0 = (2 * it_k + hh) * kSub;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int idx = lane + 32 * j, c = idx >> 3, part = idx & 7;
            if (col0 + c < nreal) {
              const Col& cl = col[col0 + c];
              cp_async16(dst + c * kUnit + part * 4, a.base + cl.base_off + v0 + part * 4, pol_first);
              cp_async16(dst + kBoxFloats + c * kUnit + part * 4, a.target + cl.target_off + v0 + part * 4,
                         pol_first);
            }
          }
          ++it_k;
          advance();
        }
        cp_async_commit();  // possibly empty: one group per item keeps the count
        ++nl;
      };
      for (int n = 0; n < rp.nbs - 1; ++n) load_next();
      double acc[kSubPerWarp];
#pragma unroll
      for (int k = 0; k < kSubPerWarp; ++k) acc[k] = 0.0;
      int nc = 0;
      for (int t = 0; ok && t < ntiles; ++t) {
        const int pt = rs_tile(gr, ntiles, t);
        const int rows = rows_of(t);
        ok = mbar_wait(bars.acc_full(slot), slot_phase, s_abort, a.err, 0x830u);
        if (!ok) break;
        tc_fence_after();
        if (kUnit * q < rows) {
          const int v0 = lo + pt * kTileRows + kUnit * q;
#pragma unroll
          for (int kk = 0; kk < kSubPerWarp; ++kk) {
            if (kk < nk) {
              load_next();
              cp_async_wait(rp.nbs - 1);
              __syncwarp();
              const float* bb = ring + (nc % rp.nbs) * (2 * kBoxFloats);
              const float* tb = bb + kBoxFloats;
              const int col0 = (2 * kk + hh) * kSub;
              uint32_t rg[kSub];
              tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(kUnit * q) << 16) +
                                     static_cast<uint32_t>(slot * rp.slot_stride + col0),
                                 rg);
              tmem_ld_wait();
              double wv[kSub];
#pragma unroll
              for (int c = 0; c < kSub; ++c) {
                const Col& cl = col[col0 + c];
                const float z = __fadd_rn(bb[c * kUnit + lane], __uint_as_float(rg[c]));
                wv[c] = static_cast<double>(res_w(tb[c * kUnit + lane], z, cl.mp, cl.fp, cl.mq, cl.fq));
              }
              // the box's sum over its 32 rows for request cr = lane >> 1
              const int cr = lane >> 1;
              const double us = warp_transpose_sum16(wv, lane);
              if ((lane & 1) == 0 && col0 + cr < nreal) {
                acc[kk] += us;
                a.res_unit[static_cast<long long>(v0 / kUnit) * a.B + e0 + col0 + cr] = us;
              }
              __syncwarp();  // every lane has read the slot before it is refilled
              ++nc;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.acc_empty(slot));
        if (++slot == rp.nslots) {
          slot = 0;
          slot_phase ^= 1u;
        }
      }
      cp_async_wait(0);
      if (!ok) {
        *s_abort = 1;
        continue;
      }
      // this warp's share of the group's slice sums (the two warps of a
      // quadrant own disjoint sub-chunks)
#pragma unroll
      for (int kk = 0; kk < kSubPerWarp; ++kk) {
        const int cl = (2 * kk + hh) * kSub + (lane >> 1);
        if ((lane & 1) == 0 && kk < nk && cl < nreal) s_part[q * rp.gsize + cl] = acc[kk];
      }
      // the unit sums and the slice sums reach the selector through the
      // mbarrier's release; its gpu-scope release reduction publishes them
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.step_done());
    }
  }
  __syncthreads();
  if (warp == kRsMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_residual_tc(const Params& P, cudaStream_t stream) {
  const VerifyArgs& a = P.a;
  RsParams rp{};
  rp.P = P;
  rp.gsize = P.res_gsize;  // the groups the verify kernel laid the operand images out for
  if ((a.B + rp.gsize - 1) / rp.gsize > kMaxGroups) return cudaErrorInvalidValue;
  rp.r_stages = a.r / kKStage;
  rp.slot_stride = (rp.gsize + 31) & ~31;
  rp.nslots = std::min(kMaxAccSlots, static_cast<int>(kTmemCols) / rp.slot_stride);
  int dev = 0, max_smem = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int choices[][2] = {{4, 3}, {4, 2}, {3, 2}, {2, 2}};
  size_t smem = 0;
  for (const auto& c : choices) {
    const size_t need = rs_layout(c[0], rp.gsize, a.r, c[1]).total + 1024;
    if (static_cast<int>(need) <= max_smem) {
      rp.nbf = c[0];
      rp.nbs = c[1];
      smem = need;
      break;
    }
  }
  if (smem == 0) return cudaErrorInvalidConfiguration;
  CUtensorMap tm_bf;
  if (!encode_bf_tiles(&tm_bf, a.Bf, a.V, a.r)) return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(residual_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int G = std::max(1, std::min(std::min(kMaxGrid, sms), a.V / kUnit));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(kRsThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, residual_tc_kernel, rp, tm_bf);
  if (e == cudaErrorNotSupported) {  // without the early start
    (void)cudaGetLastError();
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, residual_tc_kernel, rp, tm_bf);
  }
  return e;
}

}  // namespace vfy
}  // namespace dspark
