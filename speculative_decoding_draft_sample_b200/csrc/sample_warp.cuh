// Inverse-CDF draw of one draft position of one request by one warp, from the
// per-(request, 256-entry chunk) online-softmax partials that the draft-logit
// kernels leave in the workspace.
//
// "DSpark turns speculation into a scheduler", "DSpark's semi-autoregressive
// compromise": each drafted token is sampled from the biased draft
// distribution before the next position's bias is formed. The draw walks the
// vocabulary in index order: lane l owns a contiguous run of chunks, the warp
// scan of the runs' masses locates the run, the run's owner locates the chunk,
// and the chunk (256 stored logits, L2-hot) is weighed again to place the
// token. Greedy requests (temperature 0) take the argmax, lowest index on ties.
#pragma once

#include "draft.cuh"

namespace dspark {

// The next position gathers U[x] for the token just drawn: start pulling that
// row into L2 (a hint; skipped when the call has no U, as in the pick-only
// entry point, and after the last position).
template <int DT>
__device__ __forceinline__ void prefetch_u_row(const DraftArgs& a, int tok, int k) {
  if (a.U == nullptr || k >= a.K) return;
  const char* urow = static_cast<const char*>(a.U) + (long long)tok * a.r * Elem<DT>::kBytes;
  for (int off = 0; off < a.r * Elem<DT>::kBytes; off += 128)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(urow + off));
}

template <int DT>
__device__ __forceinline__ void sample_row_warp(const DraftArgs& a, int b, int k) {
  using E = Elem<DT>;
  using T = typename E::T;
  constexpr unsigned kFull = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const int nch = a.nchunk;
  const float2* P = a.partials + (long long)b * nch;
  const float tau = a.temp[b];
  const long long out_i = (long long)b * a.K + (k - 1);
  Status* st = a.status;
  if (lane == 0) {
    if (tau != tau || tau < 0.f) report(st, DSPARK_STATUS_BAD_TEMP, b);
    if (k == 1) {
      const int lt = a.last_tok[b];
      if (lt < 0 || lt >= a.V) report(st, DSPARK_STATUS_BAD_TOKEN, b);
    }
  }

  if (!(tau > 0.f)) {
    // greedy: argmax over the chunk partials (max, argmax)
    float mv = -INFINITY;
    int mi = 0x7fffffff;
    bool bad = false;
    for (int c = lane; c < nch; c += 32) {
      const float2 q = P[c];
      argmax_merge(mv, mi, q.x, __float_as_int(q.y));
      bad |= (q.x != q.x);
    }
    warp_argmax(mv, mi);
    bad = __any_sync(kFull, bad);
    if (lane == 0) {
      int i = mi;
      if (bad || mv == -INFINITY || i >= a.V) {
        report(st, DSPARK_STATUS_BAD_ROW, b);
        i = 0;
      }
      a.x[out_i] = i;
      a.q_tok[out_i] = 1.f;
      a.q_lse[out_i] = mv;
      if (a.q_norm) a.q_norm[out_i] = make_float2(mv, 1.f);
      prefetch_u_row<DT>(a, i, k);
    }
    return;
  }

  // lane l: chunks [c0, c1), contiguous (index order matters for the CDF);
  // up to kRun of them sit in registers after one round of loads
  constexpr int kRun = 24;
  const int per = (nch + 31) / 32;
  const int c0 = min(lane * per, nch), c1 = min(c0 + per, nch);
  const bool in_regs = per <= kRun;
  float2 q[kRun];
  float m = -INFINITY;
  if (in_regs) {
#pragma unroll
    for (int j = 0; j < kRun; ++j) q[j] = (c0 + j < c1) ? P[c0 + j] : make_float2(-INFINITY, 0.f);
#pragma unroll
    for (int j = 0; j < kRun; ++j) m = fmaxf(m, q[j].x);
  } else {
    for (int c = c0; c < c1; ++c) m = fmaxf(m, P[c].x);
  }
  const float M = warp_max(m);
  // mass of chunk c0 + j (or of chunk c in the long-run case)
  auto mass = [&](float2 v) { return (v.x == -INFINITY) ? 0.f : v.y * ex2(v.x - M); };
  float s = 0.f;
  if (in_regs) {
#pragma unroll
    for (int j = 0; j < kRun; ++j) s += mass(q[j]);
  } else {
    for (int c = c0; c < c1; ++c) s += mass(P[c]);
  }
  const float incl = warp_inclusive_scan(s);
  const float Z = __shfl_sync(kFull, incl, 31);
  const float excl = incl - s;
  if (!(Z > 0.f) || Z == INFINITY || M != M) {  // NaN, +inf or all -inf logits
    if (lane == 0) {
      report(st, DSPARK_STATUS_BAD_ROW, b);
      a.x[out_i] = 0;
      a.q_tok[out_i] = 0.f;
      a.q_lse[out_i] = NAN;
      if (a.q_norm) a.q_norm[out_i] = make_float2(NAN, 0.f);
    }
    return;
  }
  const float u = uniform24(a.seed, a.round_id, (uint32_t)b, (uint32_t)k, kDraft);
  const float thr = u * Z;

  // the chunk holding thr and what is left of thr at its start
  const unsigned own = __ballot_sync(kFull, s > 0.f && thr < excl + s);
  int fc = -1;
  float frem = INFINITY;
  int src;
  if (own) {
    src = __ffs(own) - 1;
    if (lane == src) {
      float rem = thr - excl;
      int lastpos = -1;
      if (in_regs) {
#pragma unroll
        for (int j = 0; j < kRun; ++j) {
          const float vc = mass(q[j]);
          if (fc < 0) {
            if (vc > 0.f) lastpos = c0 + j;
            if (vc > 0.f && rem < vc) fc = c0 + j;
            else rem -= vc;
          }
        }
      } else {
        for (int c = c0; c < c1; ++c) {
          const float vc = mass(P[c]);
          if (vc > 0.f) lastpos = c;
          if (vc > 0.f && rem < vc) {
            fc = c;
            break;
          }
          rem -= vc;
        }
      }
      if (fc < 0) {  // rounding: the last positive chunk of the run
        fc = lastpos;
        rem = INFINITY;
      }
      frem = rem;
    }
  } else {
    // rounding: thr at or past the total; the last chunk of positive mass
    src = 31 - __clz(__ballot_sync(kFull, s > 0.f));
    if (lane == src) {
      if (in_regs) {
#pragma unroll
        for (int j = 0; j < kRun; ++j)
          if (mass(q[j]) > 0.f) fc = c0 + j;
      } else {
        for (int c = c1 - 1; c >= c0; --c)
          if (mass(P[c]) > 0.f) {
            fc = c;
            break;
          }
      }
    }
  }
  const int ch = __shfl_sync(kFull, fc, src);
  const float rem = __shfl_sync(kFull, frem, src);

  // weigh the chunk again: lane l takes entries [l * 8, l * 8 + 8) of it
  const float cs = kLog2e / tau;
  const T* drow = static_cast<const T*>(a.d) + ((long long)b * a.K + (k - 1)) * a.V;
  const int v0 = ch * kChunk + lane * 8;
  float w[8];
  float ts = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int vi = v0 + j;
    w[j] = (ch >= 0 && vi < a.V) ? ex2(fmaf(E::load(drow, vi), cs, -M)) : 0.f;
    ts += w[j];
  }
  const float incl2 = warp_inclusive_scan(ts);
  const float excl2 = incl2 - ts;
  const unsigned hit = __ballot_sync(kFull, ts > 0.f && rem < excl2 + ts);
  // the lane that holds the token and its index inside the lane's 8 entries
  int tl, tj = -1;
  if (hit) {
    tl = __ffs(hit) - 1;
    float r2 = rem - excl2;
    int lp = -1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (w[j] > 0.f) lp = j;
      if (tj < 0 && w[j] > 0.f && r2 < w[j]) tj = j;
      if (tj < 0) r2 -= w[j];
    }
    if (tj < 0) tj = lp;
  } else {  // rounding: the last entry of positive weight in the chunk
    const unsigned pos = __ballot_sync(kFull, ts > 0.f);
    tl = pos ? 31 - __clz(pos) : 0;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (w[j] > 0.f) tj = j;
  }
  if (lane == tl) {
    float wt = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j == tj) wt = w[j];
    if (tj < 0 || ch < 0) {
      report(st, DSPARK_STATUS_BAD_ROW, b);
      a.x[out_i] = 0;
      a.q_tok[out_i] = 0.f;
      a.q_lse[out_i] = NAN;
      if (a.q_norm) a.q_norm[out_i] = make_float2(NAN, 0.f);
    } else {
      a.x[out_i] = v0 + tj;
      a.q_tok[out_i] = wt / Z;
      a.q_lse[out_i] = M * 0.69314718055994530942f + logf(Z);
      if (a.q_norm) a.q_norm[out_i] = make_float2(M, Z);
      prefetch_u_row<DT>(a, v0 + tj, k);
    }
  }
}

// The recurrent head's next state, by the warp that drew x_k of request b
// ("DSpark turns speculation into a scheduler", "DSpark's semi-autoregressive
// compromise": recurrent head machinery beside the Markov head; "DSpark LLM
// inference speedup", "The Semi-Autoregressive Trick": a head that tracks the
// whole block prefix): h_{k+1} = round(U[x_k] + tanh(h_k @ R)), read from row
// k-1 and written to row k of H. Lane l computes the eight outputs
// i0 + 8l .. i0 + 8l + 7 with fp32 fused multiply-adds in ascending j (r % 8 == 0).
template <int DT>
__device__ void rnn_step(const DraftArgs& a, int b, int k) {
  using E = Elem<DT>;
  using T = typename E::T;
  const int lane = threadIdx.x & 31;
  __syncwarp();  // x_k was written by one lane of this warp
  int tok = a.x[(long long)b * a.K + (k - 1)];
  if (tok < 0 || tok >= a.V) tok = 0;  // reported by the draw
  const int r = a.r;
  const T* hp = static_cast<const T*>(a.H) + ((long long)b * a.K + (k - 1)) * r;
  const T* Rm = static_cast<const T*>(a.R);
  const T* u = static_cast<const T*>(a.U) + (long long)tok * r;
  T* hn = static_cast<T*>(a.H) + ((long long)b * a.K + k) * r;
  for (int i0 = 0; i0 < r; i0 += 256) {
    const int i = i0 + 8 * lane;
    const bool on = i < r;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < r; ++j) {
      const float hj = E::load(hp, j);  // the same address in every lane
      if (on) {
        float rv[8];
        Vec16<DT>::load(Rm + (long long)j * r + i, rv);
        if (DT == DSPARK_F32) Vec16<DT>::load(Rm + (long long)j * r + i + 4, rv + 4);
#pragma unroll
        for (int m = 0; m < 8; ++m) acc[m] = fmaf(hj, rv[m], acc[m]);
      }
    }
    if (on) {
      float uv[8];
      Vec16<DT>::load(u + i, uv);
      if (DT == DSPARK_F32) Vec16<DT>::load(u + i + 4, uv + 4);
      T out[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) out[m] = E::store_round(uv[m] + tanhf(acc[m]));
#pragma unroll
      for (int m = 0; m < 8; ++m) hn[i + m] = out[m];
    }
  }
}

}  // namespace dspark
