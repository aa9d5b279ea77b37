/*
 * dspark.h -- C ABI of the per-round hot path of DSpark-style speculative
 * decoding on one B200 (sm_100a): semi-autoregressive Markov draft,
 * confidence-scheduled verify lengths, lossless rejection-sampling verify.
 *
 * Sources (four web pages on DeepSeek's DSpark; titles abbreviated):
 *   [Thread] sina.cn, "Fireworks AI CTO Dzhulgakov explains DSpark", items 1-10
 *   [QbitAI] hzrcw.cc, "DSpark: ten concepts are enough", headed sections
 *   [Essay]  10100.com, "speculative decoding is not making the model think less"
 *   [Tags]   wangjunjian.com, tag page "speculative-decoding"
 *
 * Conventions (all entry points):
 *   - Every array pointer is a DEVICE pointer owned by the caller, 16-byte
 *     aligned, row-major, densely packed. The library allocates nothing and
 *     keeps no state between calls apart from what lives in `workspace`.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns without synchronising.
 *   - Argument errors (NULL pointer, size out of range, misalignment,
 *     workspace too small) return DSPARK_ERR_INVALID_ARG before anything is
 *     launched. Launch failures return DSPARK_ERR_CUDA.
 *   - Errors found on the device (a token id outside [0,V), a verify length
 *     outside [0,K], a device-wide wait that ran out of time) are recorded in
 *     the workspace's error word; read them with dspark_read_device_error.
 *     Kernels that hit such an error stop early and leave outputs undefined.
 *   - One workspace per stream: calls that share a workspace must be ordered
 *     on one stream. Zero a new workspace once with dspark_workspace_init.
 *   - Limits: 1 <= B <= 65536, 1 <= K <= 32, 8 <= V <= 2^24 with V % 8 == 0,
 *     1 <= r <= 512, B*K <= 16384 for dspark_schedule.
 */
#ifndef DSPARK_H_
#define DSPARK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dspark_stream_t; /* same type as cudaStream_t */

typedef enum {
  DSPARK_OK = 0,
  DSPARK_ERR_INVALID_ARG = 1,
  DSPARK_ERR_UNSUPPORTED = 2,
  DSPARK_ERR_CUDA = 3,
  DSPARK_ERR_TIMEOUT = 4,       /* a device-wide wait gave up (device error word) */
  DSPARK_ERR_DEVICE_ASSERT = 5  /* an index check failed on the device (device error word) */
} dspark_status;

typedef enum { DSPARK_F32 = 0, DSPARK_BF16 = 1 } dspark_dtype;

/* Bytes of workspace that dspark_markov_draft, dspark_schedule and
 * dspark_verify need for these sizes (the maximum of the three, so one
 * workspace serves a whole round). Returns 0 if the sizes are out of range. */
size_t dspark_workspace_bytes(int B, int K, int V, int r);

/* Zero `ws_bytes` bytes of a fresh workspace on `stream` (clears the error word
 * and the device-wide counters the kernels keep in it; a workspace must be
 * initialised once before its first use). */
dspark_status dspark_workspace_init(void* workspace, size_t ws_bytes, dspark_stream_t stream);

/*
 * Semi-autoregressive draft with the low-rank Markov head.
 * [QbitAI] sections "DSpark = Eagle + DFlash" and "a cheaper sequential
 * module: the Markov head"; [Essay] section "parallel drafts are fast ...";
 * [Tags] DSpark summary, "semi-autoregressive generation".
 *
 * For i = 1..K in order, for every request b:
 *   z[b,i,:]  = base_logits[b,i,:] + A[t_{b,i-1},:] . Bf        (t_{b,0} = anchor[b])
 *   q         = softmax(z[b,i,:])
 *   t_{b,i}   = smallest v with sum_{v'<=v} q_{v'} > u_draft[b,i]*sum(q)
 *   q_tok     = q(t_{b,i}),  lse_q = log sum exp z[b,i,:]
 *
 * base_logits [B,K,V] f32; A [V,r] and Bf [r,V] of factor_dtype (bf16 is
 * IEEE bfloat16 bits); anchor [B] i32 in [0,V); u_draft [B,K] f32 in [0,1).
 * Outputs: draft_tokens [B,K] i32; q_tok [B,K] f32; lse_q [B,K] f64 (the
 * normaliser is kept in fp64 because verification forms max(0, p - q), which a
 * common fp32 rounding of the normaliser would shift); z [B,K,V] f32.
 * The weights exp(z) that place the draw and their sums over the vocabulary
 * are taken in fp64.
 */
dspark_status dspark_markov_draft(const float* base_logits, const void* A, const void* Bf,
                                  dspark_dtype factor_dtype, int r, const int32_t* anchor,
                                  const float* u_draft, int B, int K, int V,
                                  int32_t* draft_tokens, float* q_tok, double* lse_q, float* z,
                                  void* workspace, size_t ws_bytes, dspark_stream_t stream);

/*
 * The same draft with the RNN sequential head in place of the Markov head.
 * [QbitAI] section "a cheaper sequential module: the Markov head", last
 * paragraph, and [Essay] section "parallel drafts are fast ...": the paper
 * offers an RNN head that tracks the prefix of the whole draft block (off by
 * default). The pages give no equations; the head here is an Elman recurrence
 * over the drafted tokens with the Markov factors as embedding and projection:
 *   h_0 = 0,  h_i = tanh(A[t_{i-1},:] + W h_{i-1}),
 *   z[b,i,:] = base_logits[b,i,:] + bf16(h_i) . Bf     (t_0 = anchor[b])
 * with h in fp64 and rounded to bfloat16 (to nearest, ties to even) where it
 * meets the bf16 projection. W [r,r] is bf16, row-major (W[k][m] multiplies
 * h_{i-1}[m] into h_i[k]). Sampling, outputs and conventions are those of
 * dspark_markov_draft. Needs bf16 factors, r a multiple of 64 up to 256 and
 * V % 32 == 0 (the tensor-core kernel); other shapes return
 * DSPARK_ERR_UNSUPPORTED.
 */
dspark_status dspark_rnn_draft(const float* base_logits, const void* A, const void* W, const void* Bf,
                               dspark_dtype factor_dtype, int r, const int32_t* anchor, const float* u_draft,
                               int B, int K, int V, int32_t* draft_tokens, float* q_tok, double* lse_q,
                               float* z, void* workspace, size_t ws_bytes, dspark_stream_t stream);

/*
 * Confidence-scheduled verify lengths.
 * [QbitAI] section "variable-length drafts and hardware-aware scheduling"
 * (a confidence head scores each position's survival; a pre-measured
 * throughput curve picks each request's verify length, all on the GPU) and
 * section "online drafter calibration" (sequential temperature scaling);
 * [Thread] items 4 and 9 (time per token; load-dependent draft length).
 *
 *   s[b,j] = 1/(1+exp(-conf_logits[b,j]/temps[j])),  P[b,j] = prod_{k<=j} s[b,k]
 *   Rank items (b,j) by P descending, then j ascending, then b ascending; S_m =
 *   sum of the first m; choose the smallest m* maximising (B + S_m)/T(B+m) over
 *   0 <= m <= min(B*K, n_prof-B), where T(n) = profile_ms[n-1];
 *   verify_len[b] = number of request b's items among the first m*.
 *
 * conf_logits [B,K] f32; temps [K] f32 > 0; profile_ms [n_prof] f32 (n_prof >= B).
 * Outputs: verify_len [B] i32 in [0,K]; survival [B,K] f32 (P);
 * row_start [B] i64 (exclusive scan of verify_len+1: packed target-row
 * offsets); n_tokens [1] i32 (sum of verify_len+1).
 */
dspark_status dspark_schedule(const float* conf_logits, const float* temps, const float* profile_ms,
                              int n_prof, int B, int K, int32_t* verify_len, float* survival,
                              int64_t* row_start, int32_t* n_tokens, void* workspace,
                              size_t ws_bytes, dspark_stream_t stream);

/*
 * Lossless rejection-sampling verification.
 * [QbitAI] section "speculative decoding" (check candidates one by one,
 * keep the longest accepted prefix, resample at the first divergence, output
 * distributed exactly as the target); [Tags] "Speculative Decoding" steps
 * 3-5 (compare probabilities with a random number; sample from the target if
 * all pass, else from an adjusted distribution).
 *
 * Request b's target rows are target_logits[row_start[b] + rho], rho = 0..L_b
 * (L_b = verify_len[b]); p_j = softmax(row j-1). Draft j <= L_b is accepted iff
 * u_accept[b,j]*q_tok[b,j] < p_j(t_j); j* = first rejection. If j* exists the
 * final token is drawn with u_resample[b] from max(0, p_j* - q_j*) renormalised
 * (q_j* = exp(z[b,j*] - lse_q[b,j*])), else from p_{L_b+1} (row L_b, bonus).
 *
 * target_logits [*,V] f32 (dense [B,K+1,V] is row_start[b] = b*(K+1));
 * z, lse_q, q_tok, draft_tokens as produced by dspark_markov_draft;
 * verify_len [B] i32; u_accept [B,K] and u_resample [B] f32 in [0,1).
 * Outputs: accepted [B] i32 (accepted drafts); out_tokens [B,K+1] i32
 * (accepted drafts, then the final token, then -1); n_out [B] i32 (accepted+1).
 */
dspark_status dspark_verify(const float* target_logits, const int64_t* row_start, const float* z,
                            const double* lse_q, const float* q_tok, const int32_t* draft_tokens,
                            const int32_t* verify_len, const float* u_accept,
                            const float* u_resample, int B, int K, int V, int32_t* accepted,
                            int32_t* out_tokens, int32_t* n_out, void* workspace, size_t ws_bytes,
                            dspark_stream_t stream);

/*
 * Variant B of the round: the draft stores no z (B*K*V*4 bytes, the largest
 * write of the round) and verification recomputes the one row of z it needs.
 * [QbitAI] section "speculative decoding" (the residual at the first
 * divergence needs q of that position only) and section "variable-length
 * drafts and hardware-aware scheduling" (the whole round stays on the GPU).
 *
 * dspark_markov_draft_b, dspark_rnn_draft_b: the draws and the outputs
 * draft_tokens, q_tok and lse_q of dspark_markov_draft / dspark_rnn_draft
 * (same definition and arguments); instead of z they write op_rows [B,K,r]
 * (bf16 bits): the operand row position i used, A[t_{b,i-1},:] for the
 * Markov head or bf16(h_i) for the RNN head, so that
 *   z[b,i,:] = base_logits[b,i,:] + op_rows[b,i,:] . Bf.
 * dspark_verify_b: dspark_verify with z replaced by (base_logits, op_rows,
 * Bf, r): the rejected row's z is recomputed on the tensor cores. Same
 * outputs and conventions.
 * All three need bf16 factors, r a multiple of 64 up to 256, V % 32 == 0 and
 * B <= 512 (the tensor-core kernels); other shapes return
 * DSPARK_ERR_UNSUPPORTED. The workspace is the one dspark_workspace_bytes sizes;
 * dspark_verify_b uses the draft's part of it, so a draft and a verify_b on the
 * same workspace must be ordered (one stream).
 */
dspark_status dspark_markov_draft_b(const float* base_logits, const void* A, const void* Bf,
                                    dspark_dtype factor_dtype, int r, const int32_t* anchor,
                                    const float* u_draft, int B, int K, int V, int32_t* draft_tokens,
                                    float* q_tok, double* lse_q, uint16_t* op_rows, void* workspace,
                                    size_t ws_bytes, dspark_stream_t stream);
dspark_status dspark_rnn_draft_b(const float* base_logits, const void* A, const void* W, const void* Bf,
                                 dspark_dtype factor_dtype, int r, const int32_t* anchor, const float* u_draft,
                                 int B, int K, int V, int32_t* draft_tokens, float* q_tok, double* lse_q,
                                 uint16_t* op_rows, void* workspace, size_t ws_bytes, dspark_stream_t stream);
dspark_status dspark_verify_b(const float* target_logits, const int64_t* row_start, const float* base_logits,
                              const uint16_t* op_rows, const void* Bf, int r, const double* lse_q,
                              const float* q_tok, const int32_t* draft_tokens, const int32_t* verify_len,
                              const float* u_accept, const float* u_resample, int B, int K, int V,
                              int32_t* accepted, int32_t* out_tokens, int32_t* n_out, void* workspace,
                              size_t ws_bytes, dspark_stream_t stream);

/*
 * Online calibration of the sequential temperatures from one round's outcome.
 * [QbitAI] section "online drafter calibration" (the confidence scores are
 * post-processed by sequential temperature scaling, and the calibration runs
 * online from the acceptance observed on the workload); [Thread] item 10;
 * [Essay] section "the hard step ..." (survival given that earlier drafts passed).
 *
 * Position j's temperature is the scale of the logistic survival model
 * sigmoid(c / T_j). The observations of position j are the requests with
 * accepted[b] >= j-1 (they reached it) and verify_len[b] >= j (they verified
 * it), with outcome y = (accepted[b] >= j). One step on theta_j = 1 / T_j:
 *   g_j = (1/n_j) sum_b (sigmoid(conf[b,j] theta_j) - y_bj) conf[b,j]
 *   theta_j -= eta g_j;  temps[j] = clamp(1 / theta_j, t_min, t_max)
 * (a non-positive theta_j gives t_max); positions nobody reached keep their
 * temperature. Sums in fp64 in a fixed order.
 *
 * conf_logits [B,K] f32; verify_len, accepted [B] i32 (as dspark_schedule and
 * dspark_verify produced them); temps [K] f32, updated in place, so the next
 * dspark_schedule on the stream uses the calibrated values. eta >= 0,
 * 0 < t_min <= t_max. The workspace is used for its error word only (a
 * verify_len outside [0,K] or an accepted count outside [0,L_b] is recorded
 * and that request skipped).
 */
dspark_status dspark_calibrate(const float* conf_logits, const int32_t* verify_len, const int32_t* accepted,
                               int B, int K, float eta, float t_min, float t_max, float* temps,
                               void* workspace, size_t ws_bytes, dspark_stream_t stream);

/*
 * The next round's anchors from this round's output: anchor[b] becomes the
 * last token request b emitted, out_tokens[b, n_out[b]-1] (the token the next
 * draft block follows). With dspark_calibrate this lets rounds follow one
 * another on the device with no host round trip ([QbitAI] section
 * "variable-length drafts and hardware-aware scheduling": the whole logic on
 * the GPU). out_tokens [B,K+1], n_out [B] i32 as dspark_verify wrote them;
 * anchor [B] i32 is overwritten. An n_out outside [1,K+1] is recorded in the
 * workspace's error word and leaves that anchor unchanged.
 */
dspark_status dspark_advance_anchor(const int32_t* out_tokens, const int32_t* n_out, int B, int K,
                                    int32_t* anchor, void* workspace, size_t ws_bytes,
                                    dspark_stream_t stream);

/*
 * dspark_schedule without a workspace, for callers that cannot allocate
 * device memory (their allocator belongs to another framework, they run inside
 * stream capture, or their hot path forbids cudaMalloc). The pages describe no
 * such variant; it computes exactly what dspark_schedule computes, with the
 * same kernels, and allocates nothing.
 *
 * Its scratch is one static device array of fixed size inside libdspark
 * (room for DSPARK_STATIC_SCHEDULE_MAX_ITEMS items, about 192 KB), which every
 * GPU that loads the library holds until the process exits. B*K above that
 * limit returns DSPARK_ERR_INVALID_ARG; other argument rules are those of
 * dspark_schedule. Every call looks up the array's device address on the
 * current device (cudaGetSymbolAddress, which allocates nothing); the first
 * call on a device may load the library's device code, so make it before any
 * stream capture. All calls share the one
 * array, and each call fully rewrites what it reads back (its one counter
 * returns to zero at the end of the call), so no state carries over between
 * calls; calls that overlap on the GPU (two streams, or two threads) race on
 * the array and must be serialised by the caller.
 */
#define DSPARK_STATIC_SCHEDULE_MAX_ITEMS 16384
dspark_status dspark_schedule_static(const float* conf_logits, const float* temps,
                                     const float* profile_ms, int n_prof, int B, int K,
                                     int32_t* verify_len, float* survival, int64_t* row_start,
                                     int32_t* n_tokens, dspark_stream_t stream);

/* Bound, in microseconds, on every device-wide wait of the kernels that use
 * this workspace (0 restores the default of one second). A wait that runs
 * out records DSPARK_ERR_TIMEOUT in the workspace's error word; the kernel
 * then lets its copies in flight land, frees its tensor memory and returns,
 * leaving its outputs undefined. The setting is kept in the workspace (word 2
 * of its first 256 bytes) until changed or dspark_workspace_init clears it;
 * it is written on `stream`, ordered with the calls that follow there. */
dspark_status dspark_set_wait_budget(void* workspace, uint32_t microseconds, dspark_stream_t stream);

/* Test hook for failure detection without a GPU fault: make CTA `cta` of the
 * next kernels that use this workspace skip one publish, so that the other
 * CTAs' bounded waits run out and report DSPARK_ERR_TIMEOUT.
 *   DSPARK_INJECT_DRAFT_SLICE_SUMS  the draft skips its slice-sum publish at
 *                                   position 1;
 *   DSPARK_INJECT_VERIFY_BARRIER    verify skips its arrival at the first
 *                                   device-wide barrier;
 *   DSPARK_INJECT_RESIDUAL_SLICE_SUMS  dspark_verify_b's residual kernel
 *                                   skips its slice-sum publish of the first
 *                                   group of requests;
 *   DSPARK_INJECT_NONE              clears the hook.
 * Pair it with a short dspark_set_wait_budget. Kept in the workspace (word 3)
 * until cleared; written on `stream`. */
typedef enum {
  DSPARK_INJECT_NONE = 0,
  DSPARK_INJECT_DRAFT_SLICE_SUMS = 1,
  DSPARK_INJECT_VERIFY_BARRIER = 2,
  DSPARK_INJECT_RESIDUAL_SLICE_SUMS = 3
} dspark_inject;
dspark_status dspark_inject_stall(void* workspace, dspark_inject where, uint32_t cta, dspark_stream_t stream);

/* Synchronise `stream`, return the status recorded in the workspace's error
 * word (DSPARK_OK if none) and clear it; *detail (if non-NULL) receives the
 * offending value or the index of the wait that timed out. */
dspark_status dspark_read_device_error(void* workspace, dspark_stream_t stream, uint32_t* detail);

/* Static, human-readable name of a status. */
const char* dspark_status_string(dspark_status status);

#ifdef __cplusplus
}
#endif

#endif /* DSPARK_H_ */
