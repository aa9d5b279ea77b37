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
// Three stream-ordered kernels, each reading HBM once where it can:
//   rows    : one CTA per (request, row <= L_b, 4096-wide segment): segment max
//             and fp64 sum of exp(x - max); the logit at the drafted token.
//   decide  : one CTA per (request, segment): combines the row partials,
//             takes the accept decisions (identical in every CTA of the
//             request), and sums the final distribution over its segment
//             (the residual re-reads the rejected row and its z row; the bonus
//             reuses the row partials).
//   final   : one CTA per request: finds the segment where u*W falls and
//             rescans it with bit-identical weights.
#include <cfloat>

#include "common.cuh"
#include "kernels.h"

namespace dspark {

namespace {

constexpr int VT = 256;                  // threads per CTA
constexpr int kPerThread = kVerifySeg / VT;  // 16 elements
static_assert(kPerThread % 4 == 0, "segment must split into float4 per thread");

enum { kResidual = 0, kBonus = 1 };

// Probability weights, shared by `decide` and `final` so that both produce the
// same bits: p_k = exp(x_k - m_s) * fp_s with fp_s = exp(m_s - M) / W, q_k =
// exp(z_k - mq) * fq with mq = fp32(lse_q), fq = exp(mq - lse_q). Products and
// differences use explicit round-to-nearest intrinsics so no FMA contraction
// can make the two sites differ.
__device__ __forceinline__ double p_weight(float x, float m_s, double fp_s) {
  return __dmul_rn(static_cast<double>(expf(x - m_s)), fp_s);
}
__device__ __forceinline__ double residual_weight(float x, float m_s, double fp_s, float zq, float mq,
                                                  double fq) {
  const double p = p_weight(x, m_s, fp_s);
  const double q = __dmul_rn(static_cast<double>(expf(zq - mq)), fq);
  const double d = __dsub_rn(p, q);
  return d > 0.0 ? d : 0.0;
}

__global__ void __launch_bounds__(VT) verify_rows_kernel(VerifyArgs a) {
  __shared__ float redf[32];
  __shared__ double redd[33];
  const int tid = threadIdx.x;
  const long long items = static_cast<long long>(a.B) * (a.K + 1) * a.nseg;
  for (long long item = blockIdx.x; item < items; item += gridDim.x) {
    const int s = static_cast<int>(item % a.nseg);
    const long long rowlocal = item / a.nseg;
    const int rho = static_cast<int>(rowlocal % (a.K + 1));
    const int b = static_cast<int>(rowlocal / (a.K + 1));
    const int L = a.verify_len[b];
    if (L < 0 || L > a.K) {
      if (rho == 0 && s == 0 && tid == 0) set_error(a.err, DSPARK_ERR_DEVICE_ASSERT, 0x10000000u | b);
      continue;
    }
    if (rho > L) continue;
    const float* row = a.target + (a.row_start[b] + rho) * static_cast<long long>(a.V);
    const int v0 = s * kVerifySeg;
    const int n = min(kVerifySeg, a.V - v0);
    float x[kPerThread];
#pragma unroll
    for (int k = 0; k < kPerThread / 4; ++k) {
      const int off = 4 * (tid + VT * k);
      float4 f = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      if (off < n) f = __ldcs(reinterpret_cast<const float4*>(row + v0 + off));
      x[4 * k] = f.x; x[4 * k + 1] = f.y; x[4 * k + 2] = f.z; x[4 * k + 3] = f.w;
    }
    float mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) mx = fmaxf(mx, x[k]);
    const float m = block_max<VT>(mx, redf);
    double S = 0.0;
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) S += static_cast<double>(expf(x[k] - m));
    S = block_sum<VT>(S, redd);
    if (tid == 0) {
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

__global__ void __launch_bounds__(VT) verify_decide_kernel(VerifyArgs a) {
  __shared__ double rowM[kMaxK + 1], rowW[kMaxK + 1];
  __shared__ double redd[33];
  __shared__ int s_acc, s_mode;
  const int tid = threadIdx.x;
  const long long items = static_cast<long long>(a.B) * a.nseg;
  for (long long item = blockIdx.x; item < items; item += gridDim.x) {
    const int s = static_cast<int>(item % a.nseg);
    const int b = static_cast<int>(item / a.nseg);
    const int L = a.verify_len[b];
    if (L < 0 || L > a.K) continue;  // recorded by verify_rows_kernel
    // (M, W) of every row 0..L; sequential over segments, so every CTA of this
    // request computes the same bits.
    if (tid <= L) {
      const long long base = (static_cast<long long>(b) * (a.K + 1) + tid) * a.nseg;
      float M = -INFINITY;
      for (int q = 0; q < a.nseg; ++q) M = fmaxf(M, a.rp_m[base + q]);
      double W = 0.0;
      for (int q = 0; q < a.nseg; ++q)
        W += __dmul_rn(a.rp_S[base + q], exp(static_cast<double>(a.rp_m[base + q]) - M));
      rowM[tid] = M;
      rowW[tid] = W;
    }
    __syncthreads();
    if (tid == 0) {
      int acc = L;
      for (int j = 1; j <= L; ++j) {
        const int idx = b * a.K + j - 1;
        const double p_t = exp(static_cast<double>(a.x_tok[idx]) - rowM[j - 1]) / rowW[j - 1];
        const double uq = static_cast<double>(a.u_accept[idx]) * static_cast<double>(a.q_tok[idx]);
        if (!(uq < p_t)) {
          acc = j - 1;
          break;
        }
      }
      s_acc = acc;
      s_mode = acc < L ? kResidual : kBonus;
      if (s == 0) {
        VerifyDecision d;
        d.acc = acc;
        d.mode = s_mode;
        d.M = rowM[acc];
        d.W = rowW[acc];
        a.dec[b] = d;
      }
    }
    __syncthreads();
    const int acc = s_acc, mode = s_mode;
    const long long rl = static_cast<long long>(b) * (a.K + 1) + acc;
    const float m_s = a.rp_m[rl * a.nseg + s];
    const double fp_s = exp(static_cast<double>(m_s) - rowM[acc]) / rowW[acc];
    if (mode == kBonus) {
      if (tid == 0) a.seg_w[static_cast<long long>(b) * a.nseg + s] = __dmul_rn(a.rp_S[rl * a.nseg + s], fp_s);
    } else {
      const float* row = a.target + (a.row_start[b] + acc) * static_cast<long long>(a.V);
      const float* zrow = a.z + (static_cast<long long>(b) * a.K + acc) * a.V;
      const double lq = a.lse_q[b * a.K + acc];
      const float mq = static_cast<float>(lq);
      const double fq = exp(static_cast<double>(mq) - lq);
      const int v0 = s * kVerifySeg;
      const int n = min(kVerifySeg, a.V - v0);
      double acc_w = 0.0;
#pragma unroll
      for (int k = 0; k < kPerThread / 4; ++k) {
        const int off = 4 * (tid + VT * k);
        if (off < n) {
          const float4 xv = __ldcs(reinterpret_cast<const float4*>(row + v0 + off));
          const float4 zv = __ldcs(reinterpret_cast<const float4*>(zrow + v0 + off));
          acc_w += residual_weight(xv.x, m_s, fp_s, zv.x, mq, fq);
          acc_w += residual_weight(xv.y, m_s, fp_s, zv.y, mq, fq);
          acc_w += residual_weight(xv.z, m_s, fp_s, zv.z, mq, fq);
          acc_w += residual_weight(xv.w, m_s, fp_s, zv.w, mq, fq);
        }
      }
      acc_w = block_sum<VT>(acc_w, redd);
      if (tid == 0) a.seg_w[static_cast<long long>(b) * a.nseg + s] = acc_w;
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(VT) verify_final_kernel(VerifyArgs a) {
  __shared__ double redd[33];
  __shared__ int redi[32];
  __shared__ double s_total;
  const int tid = threadIdx.x;
  const int b = blockIdx.x;
  const int L = a.verify_len[b];
  if (L < 0 || L > a.K) return;
  const VerifyDecision d = a.dec[b];
  int acc = d.acc;
  int mode = d.mode;
  const long long rl = static_cast<long long>(b) * (a.K + 1) + acc;
  const float* row = a.target + (a.row_start[b] + acc) * static_cast<long long>(a.V);
  const float* zrow = a.z + (static_cast<long long>(b) * a.K + acc) * a.V;
  const double lq = a.lse_q[b * a.K + min(acc, a.K - 1)];
  const float mq = static_cast<float>(lq);
  const double fq = exp(static_cast<double>(mq) - lq);

  // segment totals of the final distribution, in segment order
  const int per = (a.nseg + VT - 1) / VT;
  const int s_lo = min(a.nseg, tid * per), s_hi = min(a.nseg, s_lo + per);
  auto seg_total = [&](int q) -> double {
    if (mode == kResidual) return a.seg_w[static_cast<long long>(b) * a.nseg + q];
    // bonus, or residual that summed to zero: the target row itself
    const double fp = exp(static_cast<double>(a.rp_m[rl * a.nseg + q]) - d.M) / d.W;
    return __dmul_rn(a.rp_S[rl * a.nseg + q], fp);
  };
  double local = 0.0;
  for (int q = s_lo; q < s_hi; ++q) local += seg_total(q);
  double total;
  double ex = block_exclusive_scan<VT>(local, redd, &total);
  if (mode == kResidual && !(total > 0.0)) {
    // max(0, p - q) vanished (only possible through rounding): sample p.
    mode = kBonus + 1;
    local = 0.0;
    for (int q = s_lo; q < s_hi; ++q) local += seg_total(q);
    ex = block_exclusive_scan<VT>(local, redd, &total);
  }
  // the inclusive sum of the last segment is the W that u scales
  if (tid == 0) s_total = 0.0;
  __syncthreads();
  if (s_hi == a.nseg && s_lo < s_hi) s_total = ex + local;
  __syncthreads();
  const double Wr = s_total;
  const double thr = static_cast<double>(a.u_resample[b]) * Wr;
  // first segment whose inclusive prefix exceeds thr
  int cand = 0x7fffffff;
  {
    double c = ex;
    for (int q = s_lo; q < s_hi; ++q) {
      c += seg_total(q);
      if (c > thr) {
        cand = q;
        break;
      }
    }
  }
  int seg = block_min_int<VT>(cand, redi);
  if (seg == 0x7fffffff) seg = a.nseg - 1;
  // exclusive prefix of that segment, recomputed by its owner in the same order
  __shared__ double s_segex;
  if (tid == seg / per) {
    double c = ex;
    for (int q = s_lo; q < seg; ++q) c += seg_total(q);
    s_segex = c;
  }
  __syncthreads();
  const double R = thr - s_segex;

  // rescan the segment with bit-identical weights, 16 contiguous per thread
  const int v0 = seg * kVerifySeg;
  const int n = min(kVerifySeg, a.V - v0);
  const float m_s = a.rp_m[rl * a.nseg + seg];
  const double fp_s = exp(static_cast<double>(m_s) - d.M) / d.W;
  const int e_lo = min(n, tid * kPerThread), e_hi = min(n, e_lo + kPerThread);
  auto weight = [&](int k) -> double {
    const float x = row[v0 + k];
    if (mode == kResidual) return residual_weight(x, m_s, fp_s, zrow[v0 + k], mq, fq);
    return p_weight(x, m_s, fp_s);
  };
  double lw = 0.0;
  int last_pos = -1;
  for (int k = e_lo; k < e_hi; ++k) {
    const double w = weight(k);
    lw += w;
    if (w > 0.0) last_pos = k;
  }
  double tot2;
  const double ex2 = block_exclusive_scan<VT>(lw, redd, &tot2);
  int found = 0x7fffffff;
  if (e_lo < e_hi && ex2 + lw > R) {
    double c = ex2;
    for (int k = e_lo; k < e_hi; ++k) {
      const double w = weight(k);
      c += w;
      if (c > R && w > 0.0) {
        found = k;
        break;
      }
    }
    if (found == 0x7fffffff) found = last_pos;  // rounding inside this thread's range
    if (found < 0) found = 0x7fffffff;
  }
  int k = block_min_int<VT>(found, redi);
  if (k == 0x7fffffff) k = block_max_int<VT>(last_pos, redi);  // rounding past the end
  if (tid == 0) {
    const int final_tok = v0 + max(k, 0);
    int32_t* out = a.out_tokens + static_cast<long long>(b) * (a.K + 1);
    for (int j = 0; j < acc; ++j) out[j] = a.tokens[b * a.K + j];
    out[acc] = final_tok;
    for (int j = acc + 1; j <= a.K; ++j) out[j] = -1;
    a.accepted[b] = acc;
    a.n_out[b] = acc + 1;
  }
}

}  // namespace

size_t verify_scratch_bytes(int B, int K, int V) {
  const size_t nseg = (V + kVerifySeg - 1) / kVerifySeg;
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
  a.nseg = (a.V + kVerifySeg - 1) / kVerifySeg;
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
  const long long items1 = static_cast<long long>(a.B) * (a.K + 1) * a.nseg;
  const int g1 = static_cast<int>(std::min<long long>(items1, static_cast<long long>(sms) * 8));
  verify_rows_kernel<<<g1, VT, 0, stream>>>(a);
  const long long items2 = static_cast<long long>(a.B) * a.nseg;
  const int g2 = static_cast<int>(std::min<long long>(items2, static_cast<long long>(sms) * 8));
  verify_decide_kernel<<<g2, VT, 0, stream>>>(a);
  verify_final_kernel<<<a.B, VT, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace dspark
