// Internal interface of the verification kernel.
#pragma once

#include "common.cuh"

namespace dspark {

// Bytes of a target row per softmax partial of the row statistics
// (1024 bf16 or 512 fp32 entries).
constexpr int kStatChunkBytes = 2048;

// Statistics of the target rows 0..cut[b] of every request (target_stats.cu).
struct StatsArgs {
  const void* target;        // [B, K+1, V]
  const int32_t* cut;        // [B] or null (every request verifies K)
  const float* temp;         // [B]
  int B, K, V, dtype;
  float2* partials;          // [B, K+1, nchunk] chunk partials (rows past the cut untouched)
  int nchunk;                // stats_chunks(V, dtype)
  unsigned long long* next;  // work counter, zeroed by the launcher
  int32_t* order;            // [B] out: the verification order (cut descending, index ascending)
  Status* status;
};

// 2 KB chunks per target row.
int stats_chunks(int V, int dtype);
cudaError_t target_stats_launch(const StatsArgs& a, int num_sms, cudaStream_t s);

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
  const float2* stats;    // [B, K+1, nstat] target-row partials from target_stats
  int nstat;              // stats_chunks(V, dtype)
  const int32_t* order;   // [B] from target_stats, or null (index order)
};

// CTAs per request (the cluster size) for this batch shape.
int verify_cluster_size(int B, int V, int dtype, int num_sms);
cudaError_t verify_launch(VerifyArgs a, int C, cudaStream_t s);

}  // namespace dspark
