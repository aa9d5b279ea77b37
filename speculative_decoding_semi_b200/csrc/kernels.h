// Launchers of the draft, schedule and verify kernels (internal to libdspark).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/dspark.h"

namespace dspark {

struct DraftArgs {
  const float* base;
  const void* A;
  const void* Bf;
  int bf16;
  int r;
  const int32_t* anchor;
  const float* u;
  int B, K, V;
  int32_t* tokens;
  float* q_tok;
  double* lse_q;
  float* z;
  unsigned* err;
  unsigned* sync;   // 2*K counters
  float* part_m;    // [B][G]
  double* part_S;   // [B][G]
  const void* W;    // RNN head's recurrent weight [r,r] (bf16), or null for the Markov head
  uint16_t* op_rows;  // variant B (z == null): [B,K,r] bf16 operand row of every position
};

struct VerifyArgs {
  const float* target;
  const int64_t* row_start;
  const float* z;             // variant A: the draft logits; null in variant B
  // variant B: z of a rejected row is recomputed as base + op_rows . Bf
  const float* base;          // [B,K,V]
  const uint16_t* op_rows;    // [B,K,r] bf16 bits
  const void* Bf;             // [r,V] bf16
  int r;
  double* res_unit;           // scratch [V/32][B]: residual sums over 32-row units
  double* res_part;           // scratch [B][grid]: residual sums over each CTA's slice
  uint8_t* res_image;         // scratch: the residual groups' operand rows in the MMA's B layout
  const double* lse_q;
  const float* q_tok;
  const int32_t* tokens;
  const int32_t* verify_len;
  const float* u_accept;
  const float* u_resample;
  int B, K, V;
  int32_t* accepted;
  int32_t* out_tokens;
  int32_t* n_out;
  unsigned* err;
};

struct ScheduleArgs {
  const float* conf;
  const float* temps;
  const float* profile;
  int n_prof, B, K;
  int32_t* verify_len;
  float* survival;
  int64_t* row_start;
  int32_t* n_tokens;
  unsigned* err;
  int32_t* rank;        // [B*K]
  double* sorted_P;     // [B*K]
  unsigned* done;       // CTAs finished (the last one runs the final step); zero between calls
};

size_t draft_scratch_bytes(int B, int K, int V, int r);
size_t verify_scratch_bytes(int B, int K, int V);
size_t schedule_scratch_bytes(int B, int K);

cudaError_t launch_draft(DraftArgs a, char* scratch, cudaStream_t stream);
// `region`: the verify part of the workspace (verify_scratch_bytes bytes).
cudaError_t launch_verify(VerifyArgs a, char* region, cudaStream_t stream);
cudaError_t launch_schedule(ScheduleArgs a, char* scratch, cudaStream_t stream);

}  // namespace dspark
