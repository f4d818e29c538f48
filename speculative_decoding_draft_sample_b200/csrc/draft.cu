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
//   draft_sample    per request: combine the chunk partials, locate the chunk
//                   holding the inverse-CDF crossing, rescan that chunk (L2-hot)
#include "draft.cuh"

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
  const T* U = static_cast<const T*>(a.U);
  const T* W = static_cast<const T*>(a.W);

  // gather U rows of the previous tokens
  for (int i = tid; i < BT * a.r; i += 256) {
    const int bb = i / a.r, j = i - bb * a.r;
    const int b = b0 + bb;
    float val = 0.f;
    if (b < a.B) {
      int prev = (k == 1) ? a.last_tok[b] : a.x[(long long)b * a.K + (k - 2)];
      if (prev < 0 || prev >= a.V) prev = 0;  // reported by draft_sample / host checks
      val = E::load(U, (long long)prev * a.r + j);
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
// draft_sample: one block of 256 threads per request.
// ---------------------------------------------------------------------------
template <int DT>
__global__ void __launch_bounds__(256) draft_sample(DraftArgs a, int k) {
  using E = Elem<DT>;
  using T = typename E::T;
  __shared__ float wsum[8];
  __shared__ float wmax[8];
  __shared__ int wint[8];
  __shared__ int s_owner;
  __shared__ int s_chunk;
  __shared__ float s_rem;
  __shared__ int s_tok;
  __shared__ int s_last;

  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nch = a.nchunk;
  const float2* P = a.partials + (long long)b * nch;
  const float tau = a.temp[b];
  const long long out_i = (long long)b * a.K + (k - 1);
  Status* st = a.status;
  if (tid == 0) {
    if (tau != tau || tau < 0.f) report(st, DSPARK_STATUS_BAD_TEMP, b);
    if (k == 1) {
      const int lt = a.last_tok[b];
      if (lt < 0 || lt >= a.V) report(st, DSPARK_STATUS_BAD_TOKEN, b);
    }
  }

  if (!(tau > 0.f)) {
    // greedy: argmax over the chunk partials
    float mv = -INFINITY;
    int mi = 0x7fffffff;
    for (int c = tid; c < nch; c += 256) argmax_merge(mv, mi, P[c].x, __float_as_int(P[c].y));
    bool bad = false;
    for (int c = tid; c < nch; c += 256) bad |= (P[c].x != P[c].x);
    warp_argmax(mv, mi);
    const int anybad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      wmax[warp] = mv;
      wint[warp] = mi | (anybad ? 0x80000000 : 0);
    }
    __syncthreads();
    if (tid == 0) {
      float m = wmax[0];
      int i = wint[0] & 0x7fffffff;
      bool bb = wint[0] < 0;
      for (int w = 1; w < 8; ++w) {
        argmax_merge(m, i, wmax[w], wint[w] & 0x7fffffff);
        bb |= wint[w] < 0;
      }
      if (bb || m == -INFINITY || i >= a.V) {
        report(st, DSPARK_STATUS_BAD_ROW, b);
        i = 0;
      }
      a.x[out_i] = i;
      a.q_tok[out_i] = 1.f;
      a.q_lse[out_i] = m;
    }
    return;
  }

  // contiguous range of chunks per thread (index order matters for the CDF)
  const int per = (nch + 255) / 256;
  const int c0 = min(tid * per, nch), c1 = min(c0 + per, nch);
  float m = -INFINITY;
  for (int c = c0; c < c1; ++c) m = fmaxf(m, P[c].x);
  m = warp_max(m);
  if (lane == 0) wmax[warp] = m;
  __syncthreads();
  float M = wmax[0];
  for (int w = 1; w < 8; ++w) M = fmaxf(M, wmax[w]);

  float s = 0.f;
  for (int c = c0; c < c1; ++c) s += (P[c].x == -INFINITY) ? 0.f : P[c].y * ex2(P[c].x - M);
  const float incl_w = warp_inclusive_scan(s);
  if (lane == 31) wsum[warp] = incl_w;
  __syncthreads();
  float wpre = 0.f, Z = 0.f;
  for (int w = 0; w < 8; ++w) {
    if (w < warp) wpre += wsum[w];
    Z += wsum[w];
  }
  const float excl = wpre + incl_w - s;

  const bool badrow = !(Z > 0.f) || Z == INFINITY || M != M;
  const float u = uniform24(a.seed, a.round_id, (uint32_t)b, (uint32_t)k, kDraft);
  const float thr = u * Z;
  if (tid == 0) s_owner = 0x7fffffff;
  __syncthreads();
  if (!badrow && s > 0.f && thr < excl + s) atomicMin(&s_owner, tid);
  __syncthreads();
  const int owner = s_owner;
  if (!badrow && owner != 0x7fffffff && tid == owner) {
    // walk the owner's chunks in index order: first chunk whose mass exceeds
    // what is left of u*Z
    float rem = thr - excl;
    int found = -1, lastpos = -1;
    for (int c = c0; c < c1; ++c) {
      const float vc = (P[c].x == -INFINITY) ? 0.f : P[c].y * ex2(P[c].x - M);
      if (vc > 0.f) lastpos = c;
      if (rem < vc) {
        found = c;
        break;
      }
      rem -= vc;
    }
    if (found < 0) {  // rounding: take the last positive element of the range
      found = lastpos;
      rem = INFINITY;
    }
    s_chunk = found;
    s_rem = rem;
  }
  if (!badrow && owner == 0x7fffffff && tid == 0) {
    // rounding: u*Z at or past the total; take the last positive element
    int lastpos = -1;
    for (int c = nch - 1; c >= 0; --c)
      if (P[c].x != -INFINITY && P[c].y * ex2(P[c].x - M) > 0.f) {
        lastpos = c;
        break;
      }
    s_chunk = lastpos;
    s_rem = INFINITY;
  }
  __syncthreads();
  if (badrow) {
    if (tid == 0) {
      report(st, DSPARK_STATUS_BAD_ROW, b);
      a.x[out_i] = 0;
      a.q_tok[out_i] = 0.f;
      a.q_lse[out_i] = NAN;
    }
    return;
  }

  // rescan the crossing chunk: one element per thread, block inclusive scan
  const int ch = s_chunk;
  const float rem = s_rem;
  const float c = kLog2e / tau;
  const int vi = ch * kChunk + tid;
  const T* d = static_cast<const T*>(a.d);
  float w = 0.f;
  if (ch >= 0 && tid < kChunk && vi < a.V)
    w = ex2(fmaf(E::load(d, ((long long)b * a.K + (k - 1)) * a.V + vi), c, -M));
  const float iw = warp_inclusive_scan(w);
  __syncthreads();
  if (lane == 31) wsum[warp] = iw;
  if (tid == 0) s_tok = 0x7fffffff;
  __syncthreads();
  float pre = 0.f;
  for (int ww = 0; ww < warp; ++ww) pre += wsum[ww];
  const float incl = pre + iw;
  if (w > 0.f && rem < incl) atomicMin(&s_tok, tid);
  __syncthreads();
  int tok = s_tok;
  if (tok == 0x7fffffff) {
    // rounding fallback: last positive element of the chunk (a second
    // variable: other threads may still be reading s_tok)
    if (tid == 0) s_last = -1;
    __syncthreads();
    if (w > 0.f) atomicMax(&s_last, tid);
    __syncthreads();
    tok = s_last;
  }
  if (tid == (tok < 0 ? 0 : tok)) {
    const int xi = (tok < 0) ? 0 : ch * kChunk + tok;
    a.x[out_i] = xi;
    a.q_tok[out_i] = w / Z;
    a.q_lse[out_i] = M * 0.69314718055994530942f + logf(Z);
    if (tok < 0) report(st, DSPARK_STATUS_BAD_ROW, b);
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
    draft_sample<DSPARK_F32><<<a.B, 256, 0, s>>>(a, k);
  else
    draft_sample<DSPARK_BF16><<<a.B, 256, 0, s>>>(a, k);
  return cudaGetLastError();
}

}  // namespace dspark
