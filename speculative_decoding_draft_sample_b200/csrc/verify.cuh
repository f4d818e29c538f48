// Internal interface of the verification kernel.
#pragma once

#include "common.cuh"

namespace dspark {

struct VerifyArgs {
  const void* target;     // [B, K+1, V]
  const void* d;          // [B, K, V]
  const int32_t* x;       // [B, K]
  const float* q_tok;     // [B, K]
  const float2* q_norm;   // [B, K] draft-row normalisers (max z, sum 2^(z - max)) or null
  const int32_t* cut;     // [B] or null
  const float* temp;      // [B]
  int B, K, V, dtype;
  uint64_t seed, round_id;
  int32_t* accepted;      // [B]
  int32_t* out;           // [B, K+1]
  int32_t* n_emit;        // [B]
  Status* status;
  int slice;              // vocabulary entries per CTA (multiple of 8)
};

// CTAs per request (the cluster size) for this batch shape.
int verify_cluster_size(int B, int V, int dtype, int num_sms);
cudaError_t verify_launch(VerifyArgs a, int C, cudaStream_t s);

}  // namespace dspark
