// Semi-autoregressive Markov draft on the 5th-generation tensor cores.
//
// QbitAI article "DSpark: ten concepts are enough", sections "DSpark = Eagle +
// DFlash" and "a cheaper sequential module: the Markov head": base logits from
// the parallel backbone are corrected left to right by a rank-256 bias that
// depends only on the previous token. Here the bias of a group of requests at
// position i is one GEMM, bias[v, b] = sum_k Bf[k, v] * A[t_b, k], run on
// tcgen05 with the accumulator in TMEM and fused with the logit correction,
// the write of z and the fp64 sums the inverse-CDF draw needs.
//
// One persistent cooperative kernel, one CTA per SM; CTA g owns the vocabulary
// slice chunk_bounds(V, 32, G, g) for every request. Requests are split into
// groups (of up to 128) that synchronise independently. Warp roles:
//   warps 0-15 epilogue, four per TMEM lane quadrant: read the accumulator
//              (warp w reads TMEM lanes 32*(w%4).. = vocabulary rows; columns
//              = requests, 16 at a time), add the base logits staged by TMA,
//              write z back through TMA, and sum exp(z) in fp64 per request
//              over each 32-row unit and over the CTA's slice;
//   warp 16    TMA producer of Bf tiles (ring of stages, L2 evict-last so the
//              78 MB factor can stay resident across positions);
//   warp 17    TMEM owner and MMA issuer (M = 128 vocabulary rows, N = the
//              group's requests, K = r in steps of 16); it bulk-loads each
//              group's operand (the A rows of the last drawn tokens, already
//              in MMA layout) once the group's tokens are published;
//   warp 18    selector: publishes the slice sums, waits for every CTA, draws
//              the tokens of its requests (b mod G == g) by a three-level
//              inverse-CDF search (the G slice sums, the chosen slice's unit
//              sums, then the chosen unit's 32 weights), writes the A rows of
//              the drawn tokens into the operand image and waits for the
//              group's tokens before releasing the next position.
// The epilogue streams base and z through per-warp TMA rings (L2 evict-first)
// that run ahead across positions, since they do not depend on the tokens.
// Variant B writes no z (the ring carries base only): the selector keeps the
// operand row of every position in op_rows instead, and the last search level
// recomputes its unit's 32 logits from base, that row and Bf. The verify of
// variant B recomputes the one rejected row of z the same way.
// Weights. z = base + bias is rounded to fp32 for the output, but the weight
// is exp(base + bias) in fp64 (exp_sum2: the reduced argument is built from
// base and bias, so z's rounding never enters; relative error ~5e-9) with a
// fixed shift of 0, and the 32 rows of a unit are summed across the warp's
// lanes in fp64 (warp_transpose_sum16). The sums that place the draw then
// differ from exact ones by ~1e-10 of the row's mass instead of the ~3e-9 an
// fp32 exponential of the rounded z would give.
// The last level of the search reads the stored fp32 z; the error there is
// confined to one 32-row unit. A row whose sum leaves [1e-280, 1e280] is
// redone by the selector with its exact maximum as the shift. Every wait is
// bounded and reports DSPARK_ERR_TIMEOUT.
#include <algorithm>
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "draft_common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace dspark {

namespace {

using namespace sm100;

constexpr int kEpiWarps = 16;                   // four per TMEM lane quadrant
constexpr int kProdWarp = kEpiWarps;
constexpr int kMmaWarp = kEpiWarps + 1;
constexpr int kSelWarp = kEpiWarps + 2;
constexpr int kThreads = (kEpiWarps + 3) * 32;
constexpr int kUnit = 32;                       // vocabulary granularity (one TMEM lane quadrant)
constexpr int kTileRows = 128;                  // MMA M
constexpr int kKStage = 64;                     // r per Bf stage (one 128-byte swizzle atom)
constexpr int kMaxBfStages = 8;
constexpr int kBfBoxBytes = 64 * kKStage * 2;   // 64 vocabulary x 64 r, bf16
constexpr int kBfStageBytes = 2 * kBfBoxBytes;  // a 128-row tile
constexpr int kChunk = 32;                      // requests per group granule
constexpr int kSub = 16;                        // requests per TMEM load and per z box
constexpr int kBoxBytes = kSub * kUnit * 4;     // 16 requests x 32 vocabulary, fp32
constexpr int kMaxGroup = 128;                  // requests per MMA (N)
constexpr int kMaxGroups = 4;                   // so B <= 512 on this path
constexpr int kMaxRingSlots = 8;
constexpr int kMaxAccSlots = 8;
constexpr uint32_t kTmemCols = 512;
constexpr int kBarBytes = 2048;
constexpr int kSubPerWarp = kMaxGroup / kSub / 4;  // sub-chunks of a group per epilogue warp
static_assert(kSubPerWarp == 2, "the spread mode's running totals assume two sub-chunks per warp");
constexpr double kSumLo = 1e-280, kSumHi = 1e280;  // row sums handled with the fixed shift


struct TcParams {
  DraftArgs d;
  uint8_t* image;       // [groups][image_stride] A rows of the drawn tokens, MMA layout
  unsigned* sync_part;  // [K][groups] slice sums published
  unsigned* sync_tok;   // [K+1][groups] tokens and operand rows published ([0]: anchors)
  int gsize;            // requests per group (multiple of 16, <= 128)
  int ngroups;
  int r_stages;         // r / 64
  int slot_stride;      // TMEM columns per accumulator slot
  int nslots;
  int nbf;              // Bf ring stages
  int nbs;              // base/z ring slots per epilogue warp
  int image_stride;     // bytes per group in the operand image (and in shared memory)
  double* unit_sum;     // [V/32][B] sums of exp(z) over each 32-row unit, this position
  double* hstate;       // [B][r] RNN head: state h_i of each request (fp64)
  double* ustate;       // [B][r] RNN head: W h_i, formed while position i streams
  uint16_t* op_rows;    // [B][K][r] variant B: the operand row of every position (bf16), or null
  int sel_bytes;        // variant B: shared staging of the last search level (0 in variant A)
  int spread;           // B <= 32: the kernel's kSpread instance (a quadrant's warps take turns over the tiles)
};

struct Layout {
  int bf, brows, ring, sel, part, bar, tab, misc, total;
};

// sel_bytes: variant B's staging of one unit's Bf columns and operand row for
// the last search level (0 in variant A)
__host__ __device__ inline Layout make_layout(int nbf, int brows_bytes, int nbs, int part_bytes, int sel_bytes) {
  Layout L;
  L.bf = 0;
  L.brows = L.bf + nbf * kBfStageBytes;
  L.ring = L.brows + ((brows_bytes + 1023) / 1024) * 1024;
  L.sel = L.ring + kEpiWarps * nbs * kBoxBytes;
  L.part = L.sel + ((sel_bytes + 127) / 128) * 128;
  L.bar = L.part + ((part_bytes + 15) / 16) * 16;
  L.tab = L.bar + kBarBytes;
  L.misc = L.tab + 16 * 8;
  L.total = L.misc + 64;
  return L;
}

// The kernel's mbarriers, addressed from one base pointer (one register
// rather than one per array).
struct Bars {
  uint64_t* q;
  __device__ uint64_t* bf_full(int s) const { return q + s; }
  __device__ uint64_t* bf_empty(int s) const { return q + kMaxBfStages + s; }
  __device__ uint64_t* acc_full(int s) const { return q + 2 * kMaxBfStages + s; }
  __device__ uint64_t* acc_empty(int s) const { return q + 2 * kMaxBfStages + kMaxAccSlots + s; }
  __device__ uint64_t* brows_full() const { return q + 2 * kMaxBfStages + 2 * kMaxAccSlots; }
  __device__ uint64_t* mma_done() const { return brows_full() + 1; }
  __device__ uint64_t* final_mma() const { return brows_full() + 2; }
  __device__ uint64_t* tokens_ready(int g) const { return brows_full() + 3 + g; }
  __device__ uint64_t* step_done(int g) const { return brows_full() + 3 + kMaxGroups + g; }
  __device__ uint64_t* base_full(int s) const { return brows_full() + 3 + 2 * kMaxGroups + s; }
};

__device__ __forceinline__ Bars carve_bars(uint8_t* p) { return Bars{reinterpret_cast<uint64_t*>(p)}; }

__device__ __forceinline__ int group_real(const TcParams& p, int gr) { return min(p.gsize, p.d.B - gr * p.gsize); }
__device__ __forceinline__ int round16(int n) { return (n + 15) & ~15; }
// Epilogue warp h of a quadrant (0..3) takes the group's sub-chunks s (16
// requests each) with s % 4 == (h + gr) % 4: the rotation spreads groups whose
// sub-chunk count is not a multiple of 4 over all four warps.
__device__ __forceinline__ int half_of(int h, int gr) { return (h + gr) & 3; }
// sub-chunks s with s % 4 == hh among the group's real columns
__device__ __forceinline__ int chunks_for(int ncol, int hh) {
  const int nsub = (ncol + kSub - 1) / kSub;
  return nsub > hh ? (nsub - hh + 3) / 4 : 0;
}

// The sub-chunks (16 requests each) that epilogue warp h of a quadrant takes
// in the t-th tile it visits in group gr: normally those with index
// s = 4k + (h + gr) % 4, in every tile (item_count of them). With at most two
// sub-chunks (kSpread, B <= 32) most warps would have none; there the items
// (t, s) are dealt round-robin over the quadrant's four warps instead, item
// t * nsub + s to warp (t * nsub + s) % 4, so each warp takes at most one
// per tile.
__device__ __forceinline__ int spread_sub(int h, int t, int nsub) { return ((h - t * nsub) % 4 + 4) % 4; }
template <bool kSpread>
__device__ __forceinline__ int item_count(const TcParams& p, int gr, int h, int t) {
  const int nreal = group_real(p, gr);
  if (!kSpread) return chunks_for(nreal, half_of(h, gr));
  return spread_sub(h, t, (nreal + kSub - 1) / kSub) < (nreal + kSub - 1) / kSub ? 1 : 0;
}
template <bool kSpread>
__device__ __forceinline__ int item_sub(const TcParams& p, int gr, int h, int t, int k) {
  if (!kSpread) return 4 * k + half_of(h, gr);
  return spread_sub(h, t, (group_real(p, gr) + kSub - 1) / kSub);
}

// Tile visited t-th in pass (i, gr): passes over the slice alternate
// direction, so each pass starts on the Bf tiles the previous one touched last
// (the ones most likely still in L2).
__device__ __forceinline__ int phys_tile(int i, int gr, int ngroups, int ntiles, int t) {
  return ((i * ngroups + gr) & 1) ? ntiles - 1 - t : t;
}

// The sequence of (position, group, tile, chunk) boxes one epilogue warp
// streams, in consumption order; the TMA refill cursor walks it ahead of the
// consumer across positions.
template <bool kSpread>
struct Items {
  const TcParams* p;
  int ntiles, last_rows, q, h;
  int i, gr, t, k;
  bool valid;
  __device__ int ptile() const { return phys_tile(i, gr, p->ngroups, ntiles, t); }
  __device__ bool tile_ok() const { return kUnit * q < (ptile() == ntiles - 1 ? last_rows : kTileRows); }
  __device__ void normalize() {
    while (valid) {
      if (i >= p->d.K) {
        valid = false;
        break;
      }
      if (gr >= p->ngroups) {
        gr = 0;
        ++i;
        continue;
      }
      if (t >= ntiles) {
        t = 0;
        ++gr;
        continue;
      }
      if (!tile_ok() || k >= item_count<kSpread>(*p, gr, h, t)) {
        k = 0;
        ++t;
        continue;
      }
      break;
    }
  }
  __device__ void first() {
    i = gr = t = k = 0;
    valid = true;
    normalize();
  }
  __device__ void next() {
    ++k;
    normalize();
  }
};

// Draw from the whole row z with its exact maximum as the shift, for a row
// whose sum of exp(z) leaves [1e-30, 1e30] (one warp). Non-finite logits are
// recorded as a device error and give token 0.
__device__ __noinline__ int draw_full_row(const float* zrow, int V, double u, int lane, int b, unsigned* err,
                                          double* w_t, float* shift, double* W) {
  float mx = -INFINITY;
  for (int k = lane; k < V; k += 32) mx = fmaxf(mx, __ldcg(zrow + k));
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, s));
  *shift = mx;
  auto wz = [&](int k) { return static_cast<double>(expf(__ldcg(zrow + k) - mx)); };
  double ex;
  int tok = warp_search<8>(V, wz, [&](double tot) { return u * tot; }, lane, &ex, W);
  if (!(*W > 0.0) || !(*W < INFINITY)) {
    if (lane == 0) set_error(err, DSPARK_ERR_DEVICE_ASSERT, 0x30000000u | static_cast<unsigned>(b));
    tok = 0;
    *w_t = 0.0;
    *W = 1.0;
  } else {
    *w_t = wz(tok);
  }
  return tok;
}

// Variant B (z not stored): z of row 32 ux + lane for request b at position
// i, recomputed from the operand row the position used.
__device__ __forceinline__ float unit_z(const TcParams& p, int b, int i, int ux, int lane) {
  const DraftArgs& d = p.d;
  const long long o = static_cast<long long>(b) * d.K + i;
  return unit_logit(p.op_rows + o * d.r, static_cast<const uint16_t*>(d.Bf), d.base + o * d.V, d.r, d.V,
                    static_cast<long long>(ux) * kUnit, lane);
}

// Variant B, for a row whose sum of exp(z) leaves the fixed-shift range: the
// draw of draw_full_row over z recomputed one 32-row unit at a time (three
// passes over the row: its maximum, its sum, the search). Slow, and only for
// rows with logits beyond about +-640.
__device__ __noinline__ int draw_full_row_b(const TcParams& p, int b, int i, double u, int lane, double* w_t,
                                            float* shift, double* W) {
  const DraftArgs& d = p.d;
  const int nu = d.V / kUnit;
  float mx = -INFINITY;
  for (int ux = 0; ux < nu; ++ux) mx = fmaxf(mx, unit_z(p, b, i, ux, lane));
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, s));
  *shift = mx;
  double tot = 0.0;
  for (int ux = 0; ux < nu; ++ux) tot += warp_sum(static_cast<double>(expf(unit_z(p, b, i, ux, lane) - mx)));
  *W = tot;
  if (!(tot > 0.0) || !(tot < INFINITY)) {
    if (lane == 0) set_error(d.err, DSPARK_ERR_DEVICE_ASSERT, 0x30000000u | static_cast<unsigned>(b));
    *w_t = 0.0;
    *W = 1.0;
    return 0;
  }
  const double thr = u * tot;
  double c = 0.0;
  int last = -1, last_ux = 0;
  for (int ux = 0; ux < nu; ++ux) {
    const double w = static_cast<double>(expf(unit_z(p, b, i, ux, lane) - mx));
    const double s = warp_sum(w);
    const unsigned pos = __ballot_sync(0xffffffffu, w > 0.0);
    if (pos) {
      last = 31 - __clz(pos);
      last_ux = ux;
    }
    if (c + s > thr) {
      const double inc = c + warp_inclusive_scan(w);
      const unsigned hit = __ballot_sync(0xffffffffu, inc > thr && w > 0.0);
      if (hit) {
        const int x = __ffs(hit) - 1;
        *w_t = __shfl_sync(0xffffffffu, w, x);
        return ux * kUnit + x;
      }
    }
    c += s;
  }
  // rounding: the last positive weight of the row
  const float zl = unit_z(p, b, i, last_ux, lane);
  *w_t = __shfl_sync(0xffffffffu, static_cast<double>(expf(zl - mx)), max(last, 0));
  return last_ux * kUnit + max(last, 0);
}

// Variant B: z of row 32 ux + lane for request b at position i, from the
// unit's Bf columns staged in shared memory (`sel`: r x 32 bf16, then the
// operand row) and the position's operand row: base + sum_k a_k Bf[k, v].
__device__ __forceinline__ float unit_z_staged(const TcParams& p, int b, int i, int ux, int lane, uint8_t* sel) {
  const DraftArgs& d = p.d;
  const long long o = static_cast<long long>(b) * d.K + i;
  const long long v0 = static_cast<long long>(ux) * kUnit;
  stage_unit_issue(sel, static_cast<const uint16_t*>(d.Bf), d.V, d.r, v0, lane);
  const float zb = __ldcg(d.base + o * d.V + v0 + lane);
  uint4* a_s = reinterpret_cast<uint4*>(sel + d.r * kUnit * 2);
  if (lane < d.r / 8) a_s[lane] = __ldcg(reinterpret_cast<const uint4*>(p.op_rows + o * d.r) + lane);
  stage_unit_wait();
  const float acc = staged_unit_dot(reinterpret_cast<const uint16_t*>(sel), a_s, d.r, lane);
  __syncwarp();  // every lane has read the staging before it is reused
  return __fadd_rn(zb, acc);
}

// Draw request b's token at position i (one warp) by a three-level
// inverse-CDF search over fp64 sums of the weights exp(z): the G slice sums
// (whose total is the W that u scales), the chosen slice's sums over its 32-row
// units, then the chosen unit's 32 weights (from the stored fp32 z). Writes
// draft_tokens, q_tok and lse_q; returns the token.
// Inlined into the kernel: as a called function it measured 13% slower (the
// call kept more of the kernel's registers spilled).
__device__ __forceinline__ int select_warp(const TcParams& p, int b, int i, int G, int lane, const double* t16) {
  const DraftArgs& d = p.d;
  const long long o = static_cast<long long>(b) * d.K + i;
  const float* zrow = d.z + o * d.V;
  const double u = static_cast<double>(d.u[o]);
  const double* part = d.part_S + static_cast<long long>(b) * G;
  double ex, W;
  // level 1: slice sums; their total is the W that u scales
  const int c = warp_search<8>(
      G, [&](int cc) { return __ldcg(part + cc); },
      [&](double tot) { return (tot >= kSumLo && tot <= kSumHi) ? u * tot : INFINITY; }, lane, &ex, &W);
  int tok;
  double w_t;
  float shift = 0.f;
  if (W >= kSumLo && W <= kSumHi) {
    const double R = u * W - ex;
    // level 2: the slice's unit sums, in vocabulary order
    int lo, hi;
    chunk_bounds(d.V, kUnit, G, c, &lo, &hi);
    const int ulo = lo / kUnit;
    const double* us = p.unit_sum + static_cast<long long>(ulo) * d.B + b;
    double ex2, tot2;
    const int ux = ulo + warp_search<2>(
                             (hi - lo) / kUnit, [&](int k) { return __ldcg(us + static_cast<long long>(k) * d.B); },
                             [&](double) { return R; }, lane, &ex2, &tot2);
    const double R2 = R - ex2;
    // level 3: the unit's weights, one per lane
    const double w = exp_fine(__ldcg(zrow + static_cast<long long>(ux) * kUnit + lane), 0.f, t16);
    const double inc = warp_inclusive_scan(w);
    const unsigned hit = __ballot_sync(0xffffffffu, inc > R2 && w > 0.0);
    const unsigned pos = __ballot_sync(0xffffffffu, w > 0.0);
    // rounding: the last positive weight of the unit
    const int x = hit ? __ffs(hit) - 1 : (pos ? 31 - __clz(pos) : 0);
    w_t = __shfl_sync(0xffffffffu, w, x);
    tok = ux * kUnit + x;
  } else {
    tok = draw_full_row(zrow, d.V, u, lane, b, d.err, &w_t, &shift, &W);
  }
  if (lane == 0) {
    d.tokens[o] = tok;
    d.q_tok[o] = static_cast<float>(w_t / W);
    d.lse_q[o] = static_cast<double>(shift) + log(W);
  }
  return tok;
}

// Variant B's draw: select_warp with the last level's 32 logits recomputed
// from the staged unit (`sel`) instead of read from z.
__device__ __forceinline__ int select_warp_b(const TcParams& p, int b, int i, int G, int lane, const double* t16,
                                          uint8_t* sel) {
  const DraftArgs& d = p.d;
  const long long o = static_cast<long long>(b) * d.K + i;
  const double u = static_cast<double>(d.u[o]);
  const double* part = d.part_S + static_cast<long long>(b) * G;
  double ex, W;
  // level 1: slice sums; their total is the W that u scales
  const int c = warp_search<8>(
      G, [&](int cc) { return __ldcg(part + cc); },
      [&](double tot) { return (tot >= kSumLo && tot <= kSumHi) ? u * tot : INFINITY; }, lane, &ex, &W);
  int tok;
  double w_t;
  float shift = 0.f;
  if (W >= kSumLo && W <= kSumHi) {
    const double R = u * W - ex;
    // level 2: the slice's unit sums, in vocabulary order
    int lo, hi;
    chunk_bounds(d.V, kUnit, G, c, &lo, &hi);
    const int ulo = lo / kUnit;
    const double* us = p.unit_sum + static_cast<long long>(ulo) * d.B + b;
    double ex2, tot2;
    const int ux = ulo + warp_search<2>(
                             (hi - lo) / kUnit, [&](int k) { return __ldcg(us + static_cast<long long>(k) * d.B); },
                             [&](double) { return R; }, lane, &ex2, &tot2);
    const double R2 = R - ex2;
    // level 3: the unit's weights, one per lane
    const float zu = unit_z_staged(p, b, i, ux, lane, sel);
    const double w = exp_fine(zu, 0.f, t16);
    const double inc = warp_inclusive_scan(w);
    const unsigned hit = __ballot_sync(0xffffffffu, inc > R2 && w > 0.0);
    const unsigned pos = __ballot_sync(0xffffffffu, w > 0.0);
    // rounding: the last positive weight of the unit
    const int x = hit ? __ffs(hit) - 1 : (pos ? 31 - __clz(pos) : 0);
    w_t = __shfl_sync(0xffffffffu, w, x);
    tok = ux * kUnit + x;
  } else {
    tok = draw_full_row_b(p, b, i, u, lane, &w_t, &shift, &W);
  }
  if (lane == 0) {
    d.tokens[o] = tok;
    d.q_tok[o] = static_cast<float>(w_t / W);
    d.lse_q[o] = static_cast<double>(shift) + log(W);
  }
  return tok;
}

// A row of the MMA's B operand for request b at position pos: A[t, :] into
// the operand image of b's group, K-major with the 128-byte swizzle, and in
// variant B also into op_rows (one warp).
template <bool kOpRows>
__device__ __forceinline__ void write_image_row(const TcParams& p, int b, int t, int pos, int lane) {
  const int gr = b / p.gsize, n = b - gr * p.gsize;
  const int N = round16(group_real(p, gr));
  const int cpr = p.d.r / 8;
  const uint4* A4 = reinterpret_cast<const uint4*>(p.d.A) + static_cast<long long>(t) * cpr;
  uint8_t* img = p.image + static_cast<long long>(gr) * p.image_stride;
  for (int ch = lane; ch < cpr; ch += 32) {
    const uint4 v = __ldg(A4 + ch);
    const int kb = ch >> 3, c = ch & 7;
    *reinterpret_cast<uint4*>(img + kb * (N * 128) + n * 128 + ((c ^ (n & 7)) << 4)) = v;
    if (kOpRows) reinterpret_cast<uint4*>(p.op_rows + (static_cast<long long>(b) * p.d.K + pos) * p.d.r)[ch] = v;
  }
}

// ------------------------------------------------------------- RNN head
// QbitAI article, section "a cheaper sequential module: the Markov head",
// last paragraph (and the 10100.com essay, section "parallel drafts are fast
// ..."): an optional RNN head tracks the prefix of the whole draft block. Here
// h_0 = 0, h_i = tanh(A[t_{i-1}] + W h_{i-1}), and the operand row of request
// b at position i is bf16(h_i) instead of A[t_{i-1}]; the state stays in fp64.
// Lane l owns the state's elements 8l .. 8l+7 (one 16-byte chunk of the
// operand row), for r/8 <= 32 lanes.

// fp64 -> bf16 bits, round to nearest even directly from the fp64 value
// (no fp32 step); values below bf16's normal range round on its subnormal
// grid. For finite inputs of magnitude < 2^128.
__device__ __forceinline__ uint16_t f64_to_bf16_bits(double x) {
  const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(x));
  const unsigned sign = static_cast<unsigned>(u >> 63) << 15;
  const double ax = fabs(x);
  if (ax < 1.1754943508222875e-38) {  // 2^-126: subnormal grid 2^-133
    const double m = rint(ax * 1.0889035741470030e+40);  // * 2^133
    return static_cast<uint16_t>(sign | static_cast<unsigned>(m));
  }
  const int e = static_cast<int>((u >> 52) & 0x7FF) - 1023 + 127;
  unsigned long long m = u & ((1ull << 52) - 1);
  const unsigned long long low = m & ((1ull << 45) - 1), half = 1ull << 44;
  m >>= 45;
  unsigned bits = (static_cast<unsigned>(e) << 7) | static_cast<unsigned>(m);
  if (low > half || (low == half && (m & 1))) ++bits;  // a carry moves into the exponent
  return static_cast<uint16_t>(sign | bits);
}

// U = W h for request b (one warp, fp64): lane l forms U[8l .. 8l+7]; the
// state's chunks are passed between lanes by shuffles.
__device__ __noinline__ void rnn_matvec(const TcParams& p, int b, int lane) {
  const int r = p.d.r, nch = r / 8;
  const uint16_t* W = static_cast<const uint16_t*>(p.d.W);
  const double* h = p.hstate + static_cast<long long>(b) * r;
  double hl[8], u[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    hl[e] = lane < nch ? h[8 * lane + e] : 0.0;
    u[e] = 0.0;
  }
  for (int c = 0; c < nch; ++c) {
    double hm[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) hm[e] = __shfl_sync(0xffffffffu, hl[e], c);
    if (lane < nch) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint4 wv = __ldg(reinterpret_cast<const uint4*>(W + static_cast<long long>(8 * lane + k) * r + 8 * c));
        const uint32_t wp[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          u[k] = fma(static_cast<double>(__uint_as_float(wp[e] << 16)), hm[2 * e], u[k]);
          u[k] = fma(static_cast<double>(__uint_as_float(wp[e] & 0xffff0000u)), hm[2 * e + 1], u[k]);
        }
      }
    }
  }
  if (lane < nch) {
    double* us = p.ustate + static_cast<long long>(b) * r + 8 * lane;
#pragma unroll
    for (int k = 0; k < 8; ++k) us[k] = u[k];
  }
}

// h = tanh(A[t] + U) (U = W h_prev, or 0 at the first position) for request
// b: stored as the new state and written, rounded to bf16, as b's operand row
// of position pos (and in variant B into op_rows).
template <bool kOpRows>
__device__ __noinline__ void rnn_step(const TcParams& p, int b, int t, bool first, int pos, int lane) {
  const int r = p.d.r, nch = r / 8;
  if (lane >= nch) return;
  const int gr = b / p.gsize, n = b - gr * p.gsize;
  const int N = round16(group_real(p, gr));
  const uint4 av = __ldg(reinterpret_cast<const uint4*>(p.d.A) + static_cast<long long>(t) * nch + lane);
  const uint32_t ap[4] = {av.x, av.y, av.z, av.w};
  double* hs = p.hstate + static_cast<long long>(b) * r + 8 * lane;
  const double* us = p.ustate + static_cast<long long>(b) * r + 8 * lane;
  uint32_t out[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const double u0 = first ? 0.0 : us[2 * e], u1 = first ? 0.0 : us[2 * e + 1];
    const double h0 = tanh(static_cast<double>(__uint_as_float(ap[e] << 16)) + u0);
    const double h1 = tanh(static_cast<double>(__uint_as_float(ap[e] & 0xffff0000u)) + u1);
    hs[2 * e] = h0;
    hs[2 * e + 1] = h1;
    out[e] = static_cast<uint32_t>(f64_to_bf16_bits(h0)) | (static_cast<uint32_t>(f64_to_bf16_bits(h1)) << 16);
  }
  uint8_t* img = p.image + static_cast<long long>(gr) * p.image_stride;
  const int kb = lane >> 3, c = lane & 7;
  const uint4 row = make_uint4(out[0], out[1], out[2], out[3]);
  *reinterpret_cast<uint4*>(img + kb * (N * 128) + n * 128 + ((c ^ (n & 7)) << 4)) = row;
  if (kOpRows) reinterpret_cast<uint4*>(p.op_rows + (static_cast<long long>(b) * p.d.K + pos) * p.d.r)[lane] = row;
}

// One warp: every lane waits for *ctr >= target (bounded), so the warp stays
// converged for the collective code that follows. Each lane's own acquire load
// of the counter orders its later reads; no further fence is needed.
__device__ __forceinline__ bool warp_wait_counter(const unsigned* ctr, unsigned target, unsigned* err,
                                                  unsigned where, volatile int* abort, int lane) {
  const bool ok = __all_sync(0xffffffffu, wait_at_least(ctr, target, err, where));
  if (!ok && lane == 0) *abort = 1;
  return ok;
}

// 19 warps: five share a 16K-register SM sub-partition, so at most 96 registers each
template <bool kRnn, bool kStoreZ, bool kSpread>
__global__ void __maxnreg__(96)
    draft_tc_kernel(const __grid_constant__ TcParams p, const __grid_constant__ CUtensorMap tm_bf,
                    const __grid_constant__ CUtensorMap tm_base, const __grid_constant__ CUtensorMap tm_z) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const DraftArgs& d = p.d;
  const Layout Ly = make_layout(p.nbf, p.image_stride, p.nbs, (kSpread ? kEpiWarps : p.ngroups * 4) * p.gsize * 8,
                                kStoreZ ? 0 : p.sel_bytes);
  Bars bars = carve_bars(smem + Ly.bar);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + Ly.misc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + Ly.misc + 4);
  double* s_part = reinterpret_cast<double*>(smem + Ly.part);  // [group][quadrant][gsize]
  double* t16 = reinterpret_cast<double*>(smem + Ly.tab);      // 2^(j/16) for exp_fine

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, g = blockIdx.x;
  int lo, hi;
  chunk_bounds(d.V, kUnit, G, g, &lo, &hi);
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
    mbar_init(bars.brows_full(), 1);
    mbar_init(bars.mma_done(), 1);
    mbar_init(bars.final_mma(), 1);
    for (int s = 0; s < kMaxGroups; ++s) {
      mbar_init(bars.tokens_ready(s), 1);
      mbar_init(bars.step_done(s), kEpiWarps);
    }
    for (int s = 0; s < kEpiWarps * kMaxRingSlots; ++s) mbar_init(bars.base_full(s), 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  fill_exp_table(t16, threadIdx.x);
  if (warp == kMmaWarp) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp == kProdWarp) {
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
      for (int i = 0; ok && i < d.K; ++i)
        for (int gr = 0; ok && gr < p.ngroups; ++gr)
          for (int t = 0; ok && t < ntiles; ++t)
            for (int s = 0; s < p.r_stages; ++s) {
              if (!mbar_wait(bars.bf_empty(stage), phase ^ 1u, s_abort, d.err, 0x100u)) {
                ok = false;
                break;
              }
              uint8_t* dst = smem + Ly.bf + stage * kBfStageBytes;
              const int pt = phys_tile(i, gr, p.ngroups, ntiles, t);
              const int v0 = lo + pt * kTileRows;
              // a last tile of at most 64 rows needs only the first 64-row box:
              // the MMA's rows beyond it are never read by the epilogue
              const bool both = (pt == ntiles - 1 ? last_rows : kTileRows) > 64;
              mbar_arrive_expect_tx(bars.bf_full(stage), both ? kBfStageBytes : kBfBoxBytes);
              tma_load_2d(dst, &tm_bf, v0, s * kKStage, bars.bf_full(stage), pol);
              if (both) tma_load_2d(dst + kBfBoxBytes, &tm_bf, v0 + 64, s * kKStage, bars.bf_full(stage), pol);
              issued[stage] = true;
              issued_parity[stage] = phase;
              if (++stage == p.nbf) {
                stage = 0;
                phase ^= 1u;
              }
            }
      // every load lands before the CTA can exit
      for (int s = 0; s < p.nbf; ++s)
        if (issued[s]) mbar_drain(bars.bf_full(s), issued_parity[s], d.err, 0x101u);
    }
  } else if (warp == kMmaWarp) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      int stage = 0, slot = 0;
      uint32_t phase = 0, slot_phase = 0, brows_phase = 0, done_phase = 0;
      uint32_t tr_phase[kMaxGroups] = {0, 0, 0, 0};
      bool brows_used = false;
      const uint32_t brows_addr = smem_u32(smem + Ly.brows);
      const uint32_t bf_addr = smem_u32(smem + Ly.bf);
      bool ok = true;
      for (int i = 0; ok && i < d.K; ++i)
        for (int gr = 0; ok && gr < p.ngroups; ++gr) {
          const int N = round16(group_real(p, gr));
          const uint32_t idesc = idesc_bf16_f32(N, 1);
          // the operand buffer is free once the previous group's MMAs are done
          if (brows_used) {
            mma_commit(bars.mma_done());
            if (!mbar_wait(bars.mma_done(), done_phase, s_abort, d.err, 0x204u)) {
              ok = false;
              break;
            }
            done_phase ^= 1u;
          }
          if (!mbar_wait(bars.tokens_ready(gr), tr_phase[gr], s_abort, d.err, 0x200u)) {
            ok = false;
            break;
          }
          tr_phase[gr] ^= 1u;
          fence_proxy_async_all();
          const uint32_t bytes = static_cast<uint32_t>(N * d.r * 2);
          mbar_arrive_expect_tx(bars.brows_full(), bytes);
          bulk_load(smem + Ly.brows, p.image + static_cast<long long>(gr) * p.image_stride, bytes,
                    bars.brows_full());
          if (!mbar_wait(bars.brows_full(), brows_phase, s_abort, d.err, 0x205u)) {
            ok = false;
            break;
          }
          brows_phase ^= 1u;
          brows_used = true;
          tc_fence_after();
          for (int t = 0; ok && t < ntiles; ++t) {
            if (!mbar_wait(bars.acc_empty(slot), slot_phase ^ 1u, s_abort, d.err, 0x201u)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t dcol = tmem_base + static_cast<uint32_t>(slot * p.slot_stride);
            for (int s = 0; s < p.r_stages; ++s) {
              if (!mbar_wait(bars.bf_full(stage), phase, s_abort, d.err, 0x202u)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t a_base = bf_addr + stage * kBfStageBytes;
              const uint32_t b_base = brows_addr + s * (N * 128);
#pragma unroll
              for (int kk = 0; kk < kKStage / 16; ++kk) {
                const uint64_t adesc = smem_desc_sw128(a_base + kk * 2048, kBfBoxBytes, 1024);
                const uint64_t bdesc = smem_desc_sw128(b_base + kk * 32, 16, 1024);
                mma_bf16(dcol, adesc, bdesc, idesc, (s | kk) != 0);
              }
              mma_commit(bars.bf_empty(stage));
              if (++stage == p.nbf) {
                stage = 0;
                phase ^= 1u;
              }
            }
            if (!ok) break;
            mma_commit(bars.acc_full(slot));
            if (++slot == p.nslots) {
              slot = 0;
              slot_phase ^= 1u;
            }
          }
        }
      // all issued MMAs complete before TMEM is released
      mma_commit(bars.final_mma());
      mbar_drain(bars.final_mma(), 0, d.err, 0x203u);
    }
  } else if (warp == kSelWarp) {
    // ------------------------------------------------------------ selector
    bool ok = true;
    // position 0's operand: the anchors' rows, and zeros in padded rows
    for (int b = g; b < d.B; b += G) {
      if (kRnn) rnn_step<!kStoreZ>(p, b, previous_token(d, b, 0), true, 0, lane);
      else write_image_row<!kStoreZ>(p, b, previous_token(d, b, 0), 0, lane);
    }
    if (g == 0) {
      for (int gr = 0; gr < p.ngroups; ++gr) {
        const int nreal = group_real(p, gr), N = round16(nreal);
        uint8_t* img = p.image + static_cast<long long>(gr) * p.image_stride;
        for (int n = nreal; n < N; ++n)
          for (int ch = lane; ch < d.r / 8; ch += 32) {
            const int kb = ch >> 3, c = ch & 7;
            *reinterpret_cast<uint4*>(img + kb * (N * 128) + n * 128 + ((c ^ (n & 7)) << 4)) =
                make_uint4(0, 0, 0, 0);
          }
      }
    }
    // Publishing: the warp barrier orders every lane's writes before lane 0's
    // release reduction, which makes them visible at gpu scope (on an SM with
    // copies in flight a separate gpu fence costs microseconds).
    __syncwarp();
    for (int gr = 0; gr < p.ngroups; ++gr) {
      const int gbase = gr * p.gsize, nreal = group_real(p, gr);
      unsigned mine = 0;
      for (int b = g; b < d.B; b += G) mine += (b >= gbase && b < gbase + nreal) ? 1u : 0u;
      if (lane == 0 && mine) red_release_gpu_add(&p.sync_tok[gr], mine);
    }
    for (int gr = 0; ok && gr < p.ngroups; ++gr) {
      ok = warp_wait_counter(&p.sync_tok[gr], static_cast<unsigned>(group_real(p, gr)), d.err, 0x400u + gr,
                             s_abort, lane);
      if (ok && lane == 0) mbar_arrive(bars.tokens_ready(gr));
    }
    for (int i = 0; ok && i < d.K; ++i) {
      for (int gr = 0; ok && gr < p.ngroups; ++gr) {
        const int gbase = gr * p.gsize, nreal = group_real(p, gr);
        // RNN head: W h_i of this CTA's requests, while position i streams
        if (kRnn && i + 1 < d.K)
          for (int b = gbase + ((g - gbase) % G + G) % G; b < gbase + nreal; b += G) rnn_matvec(p, b, lane);
        if (!mbar_wait(bars.step_done(gr), i & 1, s_abort, d.err, 0x500u)) {
          ok = false;
          break;
        }
        // this CTA's slice sums, summed over the four quadrants (spread: the
        // sixteen epilogue warps) in a fixed order
        const double* sp = s_part + gr * 4 * p.gsize;
        for (int n = lane; n < nreal; n += 32) {
          double S = sp[n] + sp[p.gsize + n] + sp[2 * p.gsize + n] + sp[3 * p.gsize + n];
          if (kSpread)
            for (int w = 4; w < kEpiWarps; ++w) S += sp[w * p.gsize + n];
          d.part_S[static_cast<long long>(gbase + n) * G + g] = S;
          d.part_m[static_cast<long long>(gbase + n) * G + g] = 0.f;
        }
        __syncwarp();
        const unsigned slot = static_cast<unsigned>(i * p.ngroups + gr);
        // (test hook: one CTA may skip its publish at position 1 so that the
        // other CTAs' waits run out)
        if (lane == 0 && !(i == 0 && injected_stall(d.err, DSPARK_INJECT_DRAFT_SLICE_SUMS, g)))
          red_release_gpu_add(&p.sync_part[slot], 1u);
        unsigned mine = 0;
        // first request of this group drawn by CTA g: the smallest b >= gbase with b % G == g
        const int first = gbase + ((g - gbase) % G + G) % G;
        if (first < gbase + nreal) {
          ok = warp_wait_counter(&p.sync_part[slot], static_cast<unsigned>(G), d.err, 0x600u + slot, s_abort, lane);
          if (!ok) break;
          for (int b = first; b < gbase + nreal; b += G) {
            const int t = kStoreZ ? select_warp(p, b, i, G, lane, t16)
                                  : select_warp_b(p, b, i, G, lane, t16, smem + Ly.sel);
            if (i + 1 < d.K) {
              if (kRnn) rnn_step<!kStoreZ>(p, b, t, false, i + 1, lane);
              else write_image_row<!kStoreZ>(p, b, t, i + 1, lane);
            }
            ++mine;
          }
        }
        if (i + 1 < d.K) {
          const unsigned nslot = static_cast<unsigned>((i + 1) * p.ngroups + gr);
          __syncwarp();
          if (lane == 0 && mine) red_release_gpu_add(&p.sync_tok[nslot], mine);
          ok = warp_wait_counter(&p.sync_tok[nslot], static_cast<unsigned>(nreal), d.err, 0x700u + nslot, s_abort,
                                 lane);
          if (ok && lane == 0) mbar_arrive(bars.tokens_ready(gr));
        }
      }
    }
    if (!ok) *s_abort = 1;
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3, h = warp >> 2;
    const uint64_t pol_first = policy_evict_first();
    if (lane == 0) {
      prefetch_tmap(&tm_base);
      prefetch_tmap(&tm_z);
    }
    float* ring = reinterpret_cast<float*>(smem + Ly.ring + warp * p.nbs * kBoxBytes);
    uint64_t* rfull = bars.base_full(warp * kMaxRingSlots);
    Items<kSpread> L;
    L.p = &p;
    L.ntiles = ntiles;
    L.last_rows = last_rows;
    L.q = q;
    L.h = h;
    L.first();
    int nl = 0, nc = 0;
    auto issue_load = [&]() {
      const int j = nl % p.nbs;
      mbar_arrive_expect_tx(&rfull[j], kBoxBytes);
      tma_load_3d(ring + j * (kBoxBytes / 4), &tm_base, lo + L.ptile() * kTileRows + kUnit * q, L.i,
                  L.gr * p.gsize + item_sub<kSpread>(p, L.gr, h, L.t, L.k) * kSub, &rfull[j], pol_first);
      L.next();
      ++nl;
    };
    if (lane == 0)
      while (L.valid && nl < p.nbs) issue_load();

    // A group's position is released (step_done) once this warp's z stores
    // for it are complete; the wait is deferred until later stores are in
    // flight, so the warp keeps streaming meanwhile.
    int pending = -1, mark = 0;
    auto release_pending = [&](int newer) {
      if (pending < 0) return;
      if (lane == 0) {
        switch (min(newer, 4)) {
          case 0: bulk_wait<0>(); break;
          case 1: bulk_wait<1>(); break;
          case 2: bulk_wait<2>(); break;
          case 3: bulk_wait<3>(); break;
          default: bulk_wait<4>(); break;
        }
        fence_proxy_async_all();
      }
      // the stores are complete; the warp barrier and the mbarrier's release
      // hand them, with the lanes' unit sums, to the selector, whose gpu-scope
      // release reduction publishes them
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.step_done(pending));
      pending = -1;
    };

    int slot = 0;
    uint32_t slot_phase = 0;
    bool ok = true;
    for (int i = 0; ok && i < d.K; ++i) {
      for (int gr = 0; ok && gr < p.ngroups; ++gr) {
        const int gbase = gr * p.gsize;
        const int nreal = group_real(p, gr);
        const int hh = half_of(h, gr);
        const int nk = kSpread ? 1 : chunks_for(nreal, hh);
        const int nsub = (nreal + kSub - 1) / kSub;
        // lane 2c sums column (request) col0 + c of each sub-chunk over the slice
        double acc[kSubPerWarp];
#pragma unroll
        for (int k = 0; k < kSubPerWarp; ++k) acc[k] = 0.0;
        // no stores of this warp follow in this group: release the last one now
        if (nk == 0) release_pending(0);
        for (int t = 0; ok && t < ntiles; ++t) {
          const int pt = phys_tile(i, gr, p.ngroups, ntiles, t);
          const int rows = (pt == ntiles - 1) ? last_rows : kTileRows;
          ok = mbar_wait(bars.acc_full(slot), slot_phase, s_abort, d.err, 0x300u);
          if (!ok) break;
          tc_fence_after();
          if (kUnit * q < rows) {
            const int v0 = lo + pt * kTileRows + kUnit * q;
            const int nkt = kSpread ? item_count<kSpread>(p, gr, h, t) : nk;
            const int ssub = kSpread ? spread_sub(h, t, nsub) : 0;
#pragma unroll
            for (int kk = 0; kk < kSubPerWarp; ++kk) {
              if (kk < nkt && ok) {
                const int j = nc % p.nbs;
                ok = mbar_wait(&rfull[j], (nc / p.nbs) & 1, s_abort, d.err, 0x301u);
                if (ok) {
                  float* box = ring + j * (kBoxBytes / 4);
                  const int col0 = (kSpread ? ssub : 4 * kk + hh) * kSub;
                  uint32_t rg[kSub];
                  tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(kUnit * q) << 16) +
                                         static_cast<uint32_t>(slot * p.slot_stride + col0),
                                     rg);
                  tmem_ld_wait();
                  // z = base + bias in place (lane = vocabulary row, c = request)
                  // and its weight exp(base + bias) in fp64, with the reduced
                  // argument built from base and bias themselves (exp_sum2),
                  // so that z's fp32 rounding never enters the weight
                  double wv[kSub];
#pragma unroll
                  for (int c = 0; c < kSub; c += 2) {
                    const F2 x = f2(box[c * kUnit + lane], box[(c + 1) * kUnit + lane]);
                    const F2 y = f2(__uint_as_float(rg[c]), __uint_as_float(rg[c + 1]));
                    const F2 zh = add2(x, y);
                    if (kStoreZ) {
                      box[c * kUnit + lane] = f2_lo(zh);
                      box[(c + 1) * kUnit + lane] = f2_hi(zh);
                    }
                    exp_sum2(x, y, zh, t16, &wv[c], &wv[c + 1]);
                  }
                  if (kStoreZ) fence_proxy_async_shared();
                  __syncwarp();
                  ++nc;
                  if (kStoreZ && lane == 0) {
                    tma_store_3d(&tm_z, box, v0, i, gbase + col0, pol_first);
                    bulk_commit();
                  }
                  // the box's sum over its 32 rows for request cr = lane >> 1
                  const int cr = lane >> 1;
                  const double us = warp_transpose_sum16(wv, lane);
                  const int col = gbase + col0 + cr;
                  if ((lane & 1) == 0 && col0 + cr < nreal) {
                    // (spread: the sub-chunk index picks the running total)
                    if (!kSpread || ssub == kk) acc[kk] += us;
                    else acc[kSubPerWarp - 1 - kk] += us;
                    p.unit_sum[static_cast<long long>(v0 / kUnit) * d.B + col] = us;
                  }
                  if (lane == 0) {
                    bulk_wait_read<1>();
                    while (L.valid && nl <= nc + p.nbs - 2) issue_load();
                  }
                }
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bars.acc_empty(slot));
          if (++slot == p.nslots) {
            slot = 0;
            slot_phase ^= 1u;
          }
          if (pending >= 0 && nc - mark > 0) release_pending(nc - mark);
        }
        if (!ok) break;
        // this warp's quadrant of the slice sums of group gr (spread: this
        // warp's share of them, one row of partials per warp)
#pragma unroll
        for (int kk = 0; kk < kSubPerWarp; ++kk) {
          if (kSpread) {
            const int col = kk * kSub + (lane >> 1);
            if ((lane & 1) == 0 && kk < nsub && col < nreal) s_part[warp * p.gsize + col] = acc[kk];
          } else {
            const int col = (4 * kk + hh) * kSub + (lane >> 1);
            if ((lane & 1) == 0 && kk < nk && col < nreal) s_part[(gr * 4 + q) * p.gsize + col] = acc[kk];
          }
        }
        release_pending(0);
        pending = gr;
        mark = nc;
        // with a single group the next position needs this release first; a
        // warp that stored nothing for this group has nothing to wait for
        if (p.ngroups == 1 || nk == 0) release_pending(0);
      }
    }
    if (ok) release_pending(0);
    if (!ok) *s_abort = 1;
    // every copy this warp started completes before the CTA exits
    if (lane == 0) {
      bulk_wait<0>();
      for (int n = nc; n < nl; ++n) mbar_drain(&rfull[n % p.nbs], (n / p.nbs) & 1, d.err, 0x302u);
    }
  }
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Requests per group: up to 128, a multiple of 32 so that a group's z boxes
// never reach into the next group. Batches that fit one group are not split:
// with two groups each group's hand-offs meet the other group's stream on
// every SM, where a signal takes several microseconds to become visible, and
// the qwen3 draft (B = 64) measured 0.389 ms split against 0.341 ms whole.
int group_size(int B) { return std::min(kMaxGroup, std::max(kChunk, (B + 31) & ~31)); }

}  // namespace

bool draft_tc_supported(const DraftArgs& a) {
  return a.bf16 && a.r % kKStage == 0 && a.r <= 256 && a.V % kUnit == 0 && a.V >= kUnit &&
         (a.B + group_size(a.B) - 1) / group_size(a.B) <= kMaxGroups;
}

int draft_tc_grid(int V, int sms) { return std::max(1, std::min(std::min(kMaxGrid, sms), V / kUnit)); }

// Global scratch of the kernel: the operand image, then the unit sums.
size_t image_bytes(int B, int r) {
  const size_t gs = group_size(B);
  const size_t ngroups = (B + gs - 1) / gs;
  return align_up(ngroups * gs * r * 2, 256);
}

size_t unit_sum_bytes(int B, int V) { return align_up(static_cast<size_t>(V / kUnit) * B * sizeof(double), 256); }
size_t rnn_state_bytes(int B, int r) { return align_up(static_cast<size_t>(B) * r * sizeof(double), 256); }

size_t draft_tc_extra_bytes(int B, int V, int r) {
  return image_bytes(B, r) + unit_sum_bytes(B, V) + 2 * rnn_state_bytes(B, r);
}

cudaError_t launch_draft_tc(DraftArgs a, int G, unsigned* sync, char* extra, cudaStream_t stream) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  TcParams p{};
  p.d = a;
  p.gsize = group_size(a.B);
  p.ngroups = (a.B + p.gsize - 1) / p.gsize;
  p.r_stages = a.r / kKStage;
  // 32-column TMEM loads may read past a slot's N columns (masked), so slots
  // are 32-column aligned and the last one ends inside the allocation
  p.slot_stride = (p.gsize + 31) & ~31;
  p.nslots = std::min(kMaxAccSlots, static_cast<int>(kTmemCols) / p.slot_stride);
  p.image_stride = p.gsize * a.r * 2;
  p.image = reinterpret_cast<uint8_t*>(extra);
  p.unit_sum = reinterpret_cast<double*>(extra + image_bytes(a.B, a.r));
  p.hstate = reinterpret_cast<double*>(extra + image_bytes(a.B, a.r) + unit_sum_bytes(a.B, a.V));
  p.ustate = p.hstate + rnn_state_bytes(a.B, a.r) / sizeof(double);
  p.op_rows = a.op_rows;
  p.sync_part = sync;
  p.sync_tok = sync + a.K * p.ngroups;
  int dev = 0, max_smem = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  p.spread = a.B <= 2 * kSub ? 1 : 0;  // one group of at most two sub-chunks
  const int part_bytes = (p.spread ? kEpiWarps : p.ngroups * 4) * p.gsize * 8;
  p.sel_bytes = a.z == nullptr ? a.r * kUnit * 2 + a.r * 2 : 0;
  // deepest Bf and base rings that fit, favouring at least 4 base slots
  const int choices[][2] = {{6, 4}, {4, 4}, {6, 3}, {4, 3}, {4, 2}, {3, 2}, {2, 2}};
  size_t smem = 0;
  for (const auto& c : choices) {
    const size_t need = make_layout(c[0], p.image_stride, c[1], part_bytes, p.sel_bytes).total + 1024;
    if (static_cast<int>(need) <= max_smem) {
      p.nbf = c[0];
      p.nbs = c[1];
      smem = need;
      break;
    }
  }
  if (smem == 0) return cudaErrorInvalidConfiguration;

  CUtensorMap tm_bf, tm_base, tm_z;
  if (!encode_bf_tiles(&tm_bf, a.Bf, a.V, a.r)) return cudaErrorInvalidValue;
  auto enc3 = [&](CUtensorMap* tm, const float* ptr) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(a.V), static_cast<cuuint64_t>(a.K),
                          static_cast<cuuint64_t>(a.B)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(a.V) * 4, static_cast<cuuint64_t>(a.V) * a.K * 4};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(kUnit), 1, static_cast<cuuint32_t>(kSub)};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  // variant B writes no z: its map (never used) describes the base logits
  if (!enc3(&tm_base, a.base) || !enc3(&tm_z, a.z != nullptr ? a.z : a.base)) return cudaErrorInvalidValue;

  // the Markov head's kernel carries no code of the RNN head, and variant A's
  // none of variant B's
  const bool store_z = a.z != nullptr;
  // one instance per (head, variant, small batch)
  using KernelFn = void (*)(const TcParams, const CUtensorMap, const CUtensorMap, const CUtensorMap);
  static const KernelFn kernels[8] = {
      draft_tc_kernel<false, false, false>, draft_tc_kernel<false, false, true>,
      draft_tc_kernel<false, true, false>,  draft_tc_kernel<false, true, true>,
      draft_tc_kernel<true, false, false>,  draft_tc_kernel<true, false, true>,
      draft_tc_kernel<true, true, false>,   draft_tc_kernel<true, true, true>};
  const void* fn = reinterpret_cast<const void*>(
      kernels[(a.W != nullptr ? 4 : 0) + (store_z ? 2 : 0) + (p.spread ? 1 : 0)]);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, smem);
  if (e != cudaSuccess) return e;
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (per_sm < 1 || G > per_sm * sms) return cudaErrorCooperativeLaunchTooLarge;
  void* args[] = {&p, &tm_bf, &tm_base, &tm_z};
  return cudaLaunchCooperativeKernel(fn, dim3(G), dim3(kThreads), args, smem, stream);
}

}  // namespace dspark
