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
// Four stream-ordered kernels, one warp per unit of work:
//   rows    : one warp per (row <= L_b, 1024-wide segment): the segment's max
//             and fp64 sum of exp(x - max), and the logit at the drafted token.
//             Rows are visited from the last (bonus) row down to row 0, so the
//             rows most often rejected are the ones still in L2 afterwards.
//   decide  : one warp per request: each row's (max, sum) from its segments,
//             the accept decisions and the first rejection.
//   segsum  : one warp per (request, segment): the final distribution's sum
//             over the segment; max(0, p - q) re-reads the rejected row and its
//             z row, the bonus reuses the row's partials.
//   final   : one warp per request: finds the segment where u*W falls and
//             rescans it, in coalesced rows of 128, with bit-identical weights.
#include <cfloat>

#include "common.cuh"
#include "kernels.h"

namespace dspark {

namespace {

constexpr int kSeg = 1024;              // segment width (32 lanes x 8 float4)
constexpr int kVec = kSeg / 32 / 4;     // float4 per lane
constexpr int WT = 256;                 // threads per CTA (8 warps)

enum { kResidual = 0, kBonus = 1, kResidualAsP = 2 };

// Probability weights shared by `decide` and `final`, so both produce the same
// bits: p_k = exp(x_k - m_s) * fp_s with fp_s = exp(m_s - M) / W; q_k =
// exp(z_k - mq) * fq with mq = fp32(lse_q), fq = exp(mq - lse_q). Products and
// differences use explicit round-to-nearest intrinsics so that no FMA
// contraction can make the two sites differ.
__device__ __forceinline__ double p_weight(float x, float m_s, double fp_s) {
  return __dmul_rn(static_cast<double>(expf(x - m_s)), fp_s);
}
__device__ __forceinline__ double residual_weight(float x, float m_s, double fp_s, float zq, float mq,
                                                  double fq) {
  const double d = __dsub_rn(p_weight(x, m_s, fp_s), __dmul_rn(static_cast<double>(expf(zq - mq)), fq));
  return d > 0.0 ? d : 0.0;
}

__device__ __forceinline__ float wmax(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double wsum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// (max, sum exp(x - max)) of a row from its segment partials, in a fixed
// order (one warp). Up to 8 partials per lane are loaded at once.
__device__ __forceinline__ void row_stats(const float* rp_m, const double* rp_S, int nseg, int lane, float* Mo,
                                          double* Wo) {
  float mv[8];
  double sv[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int s = lane + 32 * j;
    mv[j] = s < nseg ? __ldcg(rp_m + s) : -INFINITY;
    sv[j] = s < nseg ? __ldcg(rp_S + s) : 0.0;
  }
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < 8; ++j) m = fmaxf(m, mv[j]);
  for (int s = lane + 256; s < nseg; s += 32) m = fmaxf(m, __ldcg(rp_m + s));
  const float M = wmax(m);
  double w = 0.0;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (lane + 32 * j < nseg) w += __dmul_rn(sv[j], exp(static_cast<double>(mv[j]) - M));
  for (int s = lane + 256; s < nseg; s += 32)
    w += __dmul_rn(__ldcg(rp_S + s), exp(static_cast<double>(__ldcg(rp_m + s)) - M));
  *Mo = M;
  *Wo = wsum(w);
}

__global__ void __launch_bounds__(WT) verify_rows_kernel(VerifyArgs a) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (WT / 32) + (threadIdx.x >> 5);
  const int nw = gridDim.x * (WT / 32);
  const long long per_rho = static_cast<long long>(a.B) * a.nseg;
  const long long items = per_rho * (a.K + 1);
  for (long long item = gw; item < items; item += nw) {
    // rows from rho = K down to 0, requests and segments inside
    const int rho = a.K - static_cast<int>(item / per_rho);
    const long long rest = item % per_rho;
    const int b = static_cast<int>(rest / a.nseg);
    const int s = static_cast<int>(rest % a.nseg);
    const int L = a.verify_len[b];
    if (L < 0 || L > a.K) {
      if (rho == 0 && s == 0 && lane == 0) set_error(a.err, DSPARK_ERR_DEVICE_ASSERT, 0x10000000u | b);
      continue;
    }
    if (rho > L) continue;
    const long long rowlocal = static_cast<long long>(b) * (a.K + 1) + rho;
    const float* row = a.target + (a.row_start[b] + rho) * static_cast<long long>(a.V);
    const int v0 = s * kSeg;
    const int n = min(kSeg, a.V - v0);
    float4 x[kVec];
#pragma unroll
    for (int k = 0; k < kVec; ++k) {
      const int off = 4 * (k * 32 + lane);
      x[k] = off < n ? __ldcg(reinterpret_cast<const float4*>(row + v0 + off))
                     : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    }
    float m = -INFINITY;
#pragma unroll
    for (int k = 0; k < kVec; ++k) m = fmaxf(fmaxf(m, fmaxf(x[k].x, x[k].y)), fmaxf(x[k].z, x[k].w));
    m = wmax(m);
    double S = 0.0;
#pragma unroll
    for (int k = 0; k < kVec; ++k) {
      S += static_cast<double>(expf(x[k].x - m));
      S += static_cast<double>(expf(x[k].y - m));
      S += static_cast<double>(expf(x[k].z - m));
      S += static_cast<double>(expf(x[k].w - m));
    }
    S = wsum(S);
    if (lane == 0) {
      a.rp_m[rowlocal * a.nseg + s] = m;
      a.rp_S[rowlocal * a.nseg + s] = S;
      if (rho < L) {
        const int t = a.tokens[b * a.K + rho];
        if (t < 0 || t >= a.V) {
          set_error(a.err, DSPARK_ERR_DEVICE_ASSERT, 0x20000000u | b);
        } else if (t >= v0 && t < v0 + n) {
          a.x_tok[b * a.K + rho] = row[t];
        }
      }
    }
  }
}

// One CTA per request: warps form the (max, sum) of rows 0..L_b in parallel,
// then warp 0 takes the accept decisions.
__global__ void __launch_bounds__(WT) verify_decide_kernel(VerifyArgs a) {
  __shared__ float s_M[kMaxK + 1];
  __shared__ double s_W[kMaxK + 1];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int b = blockIdx.x;
  const int L = a.verify_len[b];
  if (L < 0 || L > a.K) return;  // recorded by the rows kernel
  for (int rho = warp; rho <= L; rho += WT / 32) {
    const long long rl = static_cast<long long>(b) * (a.K + 1) + rho;
    float M;
    double W;
    row_stats(a.rp_m + rl * a.nseg, a.rp_S + rl * a.nseg, a.nseg, lane, &M, &W);
    if (lane == 0) {
      s_M[rho] = M;
      s_W[rho] = W;
    }
  }
  __syncthreads();
  if (warp != 0) return;
  bool reject = false;
  if (lane < L) {
    const int idx = b * a.K + lane;
    const double p_t = exp(static_cast<double>(a.x_tok[idx]) - static_cast<double>(s_M[lane])) / s_W[lane];
    const double uq = static_cast<double>(a.u_accept[idx]) * static_cast<double>(a.q_tok[idx]);
    reject = !(uq < p_t);
  }
  const unsigned rej = __ballot_sync(0xffffffffu, reject);
  const int acc = rej ? (__ffs(rej) - 1) : L;
  const float fM = s_M[acc];
  const double fW = s_W[acc];
  if (lane == 0) {
    VerifyDecision dd;
    dd.acc = acc;
    dd.mode = acc < L ? kResidual : kBonus;
    dd.M = fM;
    dd.W = fW;
    a.dec[b] = dd;
  }
}

__global__ void __launch_bounds__(WT) verify_segsum_kernel(VerifyArgs a) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (WT / 32) + (threadIdx.x >> 5);
  const int nw = gridDim.x * (WT / 32);
  const long long items = static_cast<long long>(a.B) * a.nseg;
  for (long long item = gw; item < items; item += nw) {
    const int b = static_cast<int>(item / a.nseg);
    const int s = static_cast<int>(item % a.nseg);
    const int L = a.verify_len[b];
    if (L < 0 || L > a.K) continue;  // recorded by the rows kernel
    const VerifyDecision dd = a.dec[b];
    const int acc = dd.acc, mode = dd.mode;
    const long long rl = static_cast<long long>(b) * (a.K + 1) + acc;
    const float M = dd.M;
    const double W = dd.W;
    const float m_s = __ldcg(a.rp_m + rl * a.nseg + s);
    const double fp_s = exp(static_cast<double>(m_s) - M) / W;
    if (mode == kBonus) {
      if (lane == 0) a.seg_w[static_cast<long long>(b) * a.nseg + s] = __dmul_rn(__ldcg(a.rp_S + rl * a.nseg + s), fp_s);
      continue;
    }
    const float* row = a.target + (a.row_start[b] + acc) * static_cast<long long>(a.V);
    const float* zrow = a.z + (static_cast<long long>(b) * a.K + acc) * a.V;
    const double lq = a.lse_q[b * a.K + acc];
    const float mq = static_cast<float>(lq);
    const double fq = exp(static_cast<double>(mq) - lq);
    const int v0 = s * kSeg;
    const int n = min(kSeg, a.V - v0);
    float4 x[kVec], zz[kVec];
#pragma unroll
    for (int k = 0; k < kVec; ++k) {
      const int off = 4 * (k * 32 + lane);
      if (off < n) {
        x[k] = __ldcg(reinterpret_cast<const float4*>(row + v0 + off));
        zz[k] = __ldcs(reinterpret_cast<const float4*>(zrow + v0 + off));
      }
    }
    double w = 0.0;
#pragma unroll
    for (int k = 0; k < kVec; ++k) {
      const int off = 4 * (k * 32 + lane);
      if (off < n) {
        w += residual_weight(x[k].x, m_s, fp_s, zz[k].x, mq, fq);
        w += residual_weight(x[k].y, m_s, fp_s, zz[k].y, mq, fq);
        w += residual_weight(x[k].z, m_s, fp_s, zz[k].z, mq, fq);
        w += residual_weight(x[k].w, m_s, fp_s, zz[k].w, mq, fq);
      }
    }
    w = wsum(w);
    if (lane == 0) a.seg_w[static_cast<long long>(b) * a.nseg + s] = w;
  }
}

__global__ void __launch_bounds__(WT) verify_final_kernel(VerifyArgs a) {
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x * (WT / 32) + (threadIdx.x >> 5);
  if (b >= a.B) return;
  const int L = a.verify_len[b];
  if (L < 0 || L > a.K) return;
  const VerifyDecision d = a.dec[b];
  const int acc = d.acc;
  int mode = d.mode;
  const long long rl = static_cast<long long>(b) * (a.K + 1) + acc;
  const float* row = a.target + (a.row_start[b] + acc) * static_cast<long long>(a.V);
  const float* zrow = a.z + (static_cast<long long>(b) * a.K + min(acc, a.K - 1)) * a.V;
  const double lq = a.lse_q[b * a.K + min(acc, a.K - 1)];
  const float mq = static_cast<float>(lq);
  const double fq = exp(static_cast<double>(mq) - lq);
  const int nseg = a.nseg;
  // segment totals of the final distribution in segment order, lane-blocked
  const int per = (nseg + 31) / 32;
  const int s_lo = min(nseg, lane * per), s_hi = min(nseg, s_lo + per);
  auto seg_total = [&](int q) -> double {
    if (mode == kResidual) return __ldcg(a.seg_w + static_cast<long long>(b) * nseg + q);
    const double fp = exp(static_cast<double>(__ldcg(a.rp_m + rl * nseg + q)) - d.M) / d.W;
    return __dmul_rn(__ldcg(a.rp_S + rl * nseg + q), fp);
  };
  double local = 0.0;
  for (int q = s_lo; q < s_hi; ++q) local += seg_total(q);
  double run = 0.0, ex = 0.0;
  for (int l = 0; l < 32; ++l) {
    const double v = __shfl_sync(0xffffffffu, local, l);
    if (l == lane) ex = run;
    run += v;
  }
  if (mode == kResidual && !(run > 0.0)) {
    // max(0, p - q) vanished (only possible through rounding): sample p
    mode = kResidualAsP;
    local = 0.0;
    for (int q = s_lo; q < s_hi; ++q) local += seg_total(q);
    run = 0.0;
    for (int l = 0; l < 32; ++l) {
      const double v = __shfl_sync(0xffffffffu, local, l);
      if (l == lane) ex = run;
      run += v;
    }
  }
  const double thr = static_cast<double>(a.u_resample[b]) * run;
  // first segment whose inclusive prefix exceeds thr
  int cand = 0x7fffffff;
  double cand_ex = 0.0;
  {
    double c = ex;
    for (int q = s_lo; q < s_hi; ++q) {
      const double v = seg_total(q);
      if (c + v > thr && v > 0.0) {
        cand = q;
        cand_ex = c;
        break;
      }
      c += v;
    }
  }
  int seg = cand;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) seg = min(seg, __shfl_xor_sync(0xffffffffu, seg, o));
  double seg_ex;
  if (seg == 0x7fffffff) {
    // rounding: the last segment, with its exclusive prefix
    seg = nseg - 1;
    double e = 0.0;
    if (seg >= s_lo && seg < s_hi) {
      e = ex;
      for (int q = s_lo; q < seg; ++q) e += seg_total(q);
    }
    const int owner = min(31, seg / max(per, 1));
    seg_ex = __shfl_sync(0xffffffffu, e, owner);
  } else {
    const int owner = min(31, seg / max(per, 1));
    seg_ex = __shfl_sync(0xffffffffu, cand_ex, owner);
  }
  const double R = thr - seg_ex;
  // rescan the segment in rows of 128 (lane l: elements 4l..4l+3 of a row),
  // with the weights of the segsum kernel, in vocabulary order
  const int v0 = seg * kSeg;
  const int n = min(kSeg, a.V - v0);
  const float m_s = __ldcg(a.rp_m + rl * nseg + seg);
  const double fp_s = exp(static_cast<double>(m_s) - d.M) / d.W;
  struct XZ {
    float4 x, z;
  };
  int last = -1;
  int k = scan_rows128<kSeg / 128, XZ>(
      n, lane, R,
      [&](int e) {
        XZ v;
        v.x = __ldcg(reinterpret_cast<const float4*>(row + v0 + e));
        v.z = mode == kResidual ? __ldcg(reinterpret_cast<const float4*>(zrow + v0 + e)) : v.x;
        return v;
      },
      [&](const XZ& v, double(&w)[4]) {
        if (mode == kResidual) {
          w[0] = residual_weight(v.x.x, m_s, fp_s, v.z.x, mq, fq);
          w[1] = residual_weight(v.x.y, m_s, fp_s, v.z.y, mq, fq);
          w[2] = residual_weight(v.x.z, m_s, fp_s, v.z.z, mq, fq);
          w[3] = residual_weight(v.x.w, m_s, fp_s, v.z.w, mq, fq);
        } else {
          w[0] = p_weight(v.x.x, m_s, fp_s);
          w[1] = p_weight(v.x.y, m_s, fp_s);
          w[2] = p_weight(v.x.z, m_s, fp_s);
          w[3] = p_weight(v.x.w, m_s, fp_s);
        }
      },
      &last);
  if (k < 0) k = max(last, 0);  // rounding: the last positive weight
  int32_t* out = a.out_tokens + static_cast<long long>(b) * (a.K + 1);
  for (int j = lane; j <= a.K; j += 32) out[j] = j < acc ? a.tokens[b * a.K + j] : (j == acc ? v0 + k : -1);
  if (lane == 0) {
    a.accepted[b] = acc;
    a.n_out[b] = acc + 1;
  }
}

}  // namespace

size_t verify_scratch_bytes(int B, int K, int V) {
  const size_t nseg = (V + kSeg - 1) / kSeg;
  const size_t rows = static_cast<size_t>(B) * (K + 1);
  size_t off = 0;
  off = align_up(off + rows * nseg * sizeof(float), 256);
  off = align_up(off + rows * nseg * sizeof(double), 256);
  off = align_up(off + static_cast<size_t>(B) * K * sizeof(float), 256);
  off = align_up(off + static_cast<size_t>(B) * nseg * sizeof(double), 256);
  off = align_up(off + static_cast<size_t>(B) * sizeof(VerifyDecision), 256);
  return off;
}

cudaError_t launch_verify(VerifyArgs a, char* scratch, cudaStream_t stream) {
  a.nseg = (a.V + kSeg - 1) / kSeg;
  const size_t nseg = a.nseg;
  const size_t rows = static_cast<size_t>(a.B) * (a.K + 1);
  size_t off = 0;
  a.rp_m = reinterpret_cast<float*>(scratch + off);
  off = align_up(off + rows * nseg * sizeof(float), 256);
  a.rp_S = reinterpret_cast<double*>(scratch + off);
  off = align_up(off + rows * nseg * sizeof(double), 256);
  a.x_tok = reinterpret_cast<float*>(scratch + off);
  off = align_up(off + static_cast<size_t>(a.B) * a.K * sizeof(float), 256);
  a.seg_w = reinterpret_cast<double*>(scratch + off);
  off = align_up(off + static_cast<size_t>(a.B) * nseg * sizeof(double), 256);
  a.dec = reinterpret_cast<VerifyDecision*>(scratch + off);

  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int wpc = WT / 32;
  const long long items1 = static_cast<long long>(a.B) * (a.K + 1) * a.nseg;
  const int g1 = static_cast<int>(std::min<long long>((items1 + wpc - 1) / wpc, static_cast<long long>(sms) * 8));
  verify_rows_kernel<<<g1, WT, 0, stream>>>(a);
  verify_decide_kernel<<<a.B, WT, 0, stream>>>(a);
  const long long items2 = static_cast<long long>(a.B) * a.nseg;
  const int g2 = static_cast<int>(std::min<long long>((items2 + wpc - 1) / wpc, static_cast<long long>(sms) * 8));
  verify_segsum_kernel<<<g2, WT, 0, stream>>>(a);
  verify_final_kernel<<<(a.B + wpc - 1) / wpc, WT, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace dspark
