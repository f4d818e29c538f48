// Draft stage of the speculative round: Markov-biased draft logits and
// position-by-position sampling.
//
// "DSpark turns speculation into a scheduler", "DSpark's semi-autoregressive
// compromise": the parallel backbone gives base logits for the whole block and
// a lightweight sequential head adds a prefix-dependent bias before each token
// is sampled; the Markov head's bias is a low-rank transition signal from the
// previous sampled token. "DSpark LLM inference speedup", "The Semi-Autoregressive
// Trick": rank 256, only the immediately preceding token.
//
// Per position k the work is two launches:
//   draft_logits_*  d = round(base + scale * U[x_{k-1}] @ W) for a tile of
//                   requests x 256 vocabulary entries, written to HBM, plus each
//                   tile row's online-softmax partial (max, sum exp2) of d/temp
//   draft_sample    one warp per request: combine the chunk partials, locate
//                   the chunk holding the inverse-CDF crossing, rescan that
//                   chunk (L2-hot); see sample_warp.cuh
#include "draft.cuh"
#include "sample_warp.cuh"

namespace dspark {

// ---------------------------------------------------------------------------
// CUDA-core (FFMA) version: fp32 inputs (no TF32 anywhere) and the reference
// schedule for bf16 before the tensor-core kernel takes over.
// Block: 256 threads, one vocabulary column each; BT requests per block.
// ---------------------------------------------------------------------------
template <int DT, int BT>
__global__ void __launch_bounds__(256) draft_logits_simt(DraftArgs a, int k) {
  using E = Elem<DT>;
  using T = typename E::T;
  extern __shared__ float smem[];
  float* us = smem;                              // [BT][r] gathered U rows
  __shared__ float red_m[8][BT];
  __shared__ float red_s[8][BT];
  __shared__ int red_i[8][BT];
  __shared__ int red_bad[BT];
  __shared__ float cm[BT];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = blockIdx.x;
  const int b0 = blockIdx.y * BT;
  const int v = chunk * kChunk + tid;
  const bool col_ok = v < a.V;
  const T* W = static_cast<const T*>(a.W);

  // gather U rows of the previous tokens (or the recurrent head's states);
  // the recurrent head's first states h_1 = U[x_0] are written out once
  for (int i = tid; i < BT * a.r; i += 256) {
    const int bb = i / a.r, j = i - bb * a.r;
    const int b = b0 + bb;
    float val = 0.f;
    if (b < a.B) {
      int prev = (k == 1) ? a.last_tok[b] : a.x[(long long)b * a.K + (k - 2)];
      if (prev < 0 || prev >= a.V) prev = 0;  // reported by draft_sample / host checks
      const T* row = a_row<T>(a, b, k, prev);
      val = E::load(row, j);
      if (a.R && k == 1 && blockIdx.x == 0) static_cast<T*>(a.H)[(long long)b * a.K * a.r + j] = row[j];
    }
    us[i] = val;
  }
  if (tid < BT) red_bad[tid] = 0;
  __syncthreads();

  float acc[BT];
#pragma unroll
  for (int bb = 0; bb < BT; ++bb) acc[bb] = 0.f;
  if (col_ok) {
    for (int j = 0; j < a.r; ++j) {
      const float w = E::load(W, (long long)j * a.V + v);
#pragma unroll
      for (int bb = 0; bb < BT; ++bb) acc[bb] = fmaf(us[bb * a.r + j], w, acc[bb]);
    }
  }

  const T* base = static_cast<const T*>(a.base);
  T* d = static_cast<T*>(a.d);
  float z[BT];
#pragma unroll
  for (int bb = 0; bb < BT; ++bb) {
    const int b = b0 + bb;
    z[bb] = -INFINITY;
    if (b < a.B && col_ok) {
      const long long off = ((long long)b * a.K + (k - 1)) * a.V + v;
      const float sc = a.bias_scale ? a.bias_scale[b] : 1.f;
      const T dv = E::store_round(fmaf(sc, acc[bb], E::load(base, off)));
      d[off] = dv;
      z[bb] = E::to_float(dv);  // raw stored logit; scaled below per request
    }
  }

  // chunk partials: sampled rows (max, sum exp2) of d * log2e / temp,
  // greedy rows (max d, argmax)
#pragma unroll
  for (int bb = 0; bb < BT; ++bb) {
    const int b = b0 + bb;
    const float tau = (b < a.B) ? a.temp[b] : 1.f;
    const bool greedy = !(tau > 0.f);
    const bool bad = col_ok && bad_logit(z[bb]);
    if (__any_sync(0xffffffffu, bad) && lane == 0) red_bad[bb] = 1;
    if (greedy) {
      float mv = z[bb];
      int mi = col_ok ? v : 0x7fffffff;
      if (!col_ok) mv = -INFINITY;
      warp_argmax(mv, mi);
      if (lane == 0) {
        red_m[warp][bb] = mv;
        red_i[warp][bb] = mi;
      }
    } else {
      const float c = kLog2e / tau;
      z[bb] = z[bb] * c;
      const float mv = warp_max(z[bb]);
      if (lane == 0) red_m[warp][bb] = mv;
    }
  }
  __syncthreads();
  if (tid < BT) {
    const int b = b0 + tid;
    const float tau = (b < a.B) ? a.temp[b] : 1.f;
    if (!(tau > 0.f)) {
      float mv = red_m[0][tid];
      int mi = red_i[0][tid];
      for (int w = 1; w < 8; ++w) argmax_merge(mv, mi, red_m[w][tid], red_i[w][tid]);
      if (b < a.B) {
        float2 p;
        p.x = red_bad[tid] ? NAN : mv;
        p.y = __int_as_float(mi);
        a.partials[(long long)b * a.nchunk + chunk] = p;
      }
    } else {
      float mv = red_m[0][tid];
      for (int w = 1; w < 8; ++w) mv = fmaxf(mv, red_m[w][tid]);
      cm[tid] = mv;
    }
  }
  __syncthreads();
#pragma unroll
  for (int bb = 0; bb < BT; ++bb) {
    const int b = b0 + bb;
    const float tau = (b < a.B) ? a.temp[b] : 1.f;
    if (tau > 0.f) {
      const float e = (col_ok && cm[bb] != -INFINITY) ? ex2(z[bb] - cm[bb]) : 0.f;
      const float s = warp_sum(e);
      if (lane == 0) red_s[warp][bb] = s;
    }
  }
  __syncthreads();
  if (tid < BT) {
    const int b = b0 + tid;
    if (b < a.B && a.temp[b] > 0.f) {
      float s = 0.f;
      for (int w = 0; w < 8; ++w) s += red_s[w][tid];
      float2 p;
      p.x = cm[tid];
      p.y = red_bad[tid] ? NAN : s;
      a.partials[(long long)b * a.nchunk + chunk] = p;
    }
  }
}

// ---------------------------------------------------------------------------
// draft_sample: one warp per request, eight requests per block.
// ---------------------------------------------------------------------------
template <int DT>
__global__ void __launch_bounds__(256) draft_sample(DraftArgs a, int k) {
  const int b = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (b < a.B) {
    sample_row_warp<DT>(a, b, k);
    if (a.R && k < a.K) rnn_step<DT>(a, b, k);  // the recurrent head's next state
  }
}

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------
template <int DT, int BT>
static cudaError_t launch_simt(const DraftArgs& a, int k, cudaStream_t s) {
  dim3 grid(a.nchunk, (a.B + BT - 1) / BT);
  const size_t sm = (size_t)BT * a.r * sizeof(float);
  if (sm > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(draft_logits_simt<DT, BT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
  }
  draft_logits_simt<DT, BT><<<grid, 256, sm, s>>>(a, k);
  return cudaGetLastError();
}

cudaError_t draft_logits_simt_launch(const DraftArgs& a, int k, cudaStream_t s) {
  if (a.dtype == DSPARK_F32) return launch_simt<DSPARK_F32, 8>(a, k, s);
  return launch_simt<DSPARK_BF16, 16>(a, k, s);
}

cudaError_t draft_sample_launch(const DraftArgs& a, int k, cudaStream_t s) {
  if (a.dtype == DSPARK_F32)
    draft_sample<DSPARK_F32><<<(a.B + 7) / 8, 256, 0, s>>>(a, k);
  else
    draft_sample<DSPARK_BF16><<<(a.B + 7) / 8, 256, 0, s>>>(a, k);
  return cudaGetLastError();
}

}  // namespace dspark
