// Internal interface of the draft-stage kernels.
#pragma once

#include "common.cuh"

namespace dspark {

// Vocabulary entries per chunk partial (one online-softmax partial per
// (request, chunk)); the sampler rescans one chunk to place its draw.
constexpr int kChunk = 256;

struct DraftArgs {
  const void* base;        // [B, K, V]
  const void* U;           // [V, r]
  const void* W;           // [r, V]
  const float* bias_scale; // [B] or null
  const int32_t* last_tok; // [B]
  const float* temp;       // [B]
  int B, K, V, r, dtype;
  uint64_t seed, round_id;
  int32_t* x;              // [B, K]
  void* d;                 // [B, K, V]
  float* q_lse;            // [B, K]
  float* q_tok;            // [B, K]
  float2* q_norm;          // [B, K] (max z, sum 2^(z - max)) of z = d log2(e) / temp, or null
  float2* partials;        // [B, nchunk] in the workspace
  int nchunk;
  Status* status;
  const void* R;           // [r, r] recurrent head's state matrix, or null (Markov head)
  void* H;                 // [B, K, r] recurrent states h_1..h_K (out; with R)
};

// Row of the bias GEMM's A operand of request b at draft position k (1-based):
// U[x_{k-1}] for the Markov head and for the recurrent head's first position
// (h_1 = U[x_0] + tanh(0)), else the recurrent state h_k (row k-1 of H).
template <typename T>
__device__ __forceinline__ const T* a_row(const DraftArgs& a, int b, int k, int prev_tok) {
  if (a.R && k >= 2) return static_cast<const T*>(a.H) + ((long long)b * a.K + (k - 1)) * a.r;
  return static_cast<const T*>(a.U) + (long long)prev_tok * a.r;
}

cudaError_t draft_logits_simt_launch(const DraftArgs& a, int k, cudaStream_t s);
cudaError_t draft_sample_launch(const DraftArgs& a, int k, cudaStream_t s);

}  // namespace dspark
