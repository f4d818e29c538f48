// Lossless rejection-sampling verification, residual / bonus draw and emission.
//
// "DSpark turns speculation into a scheduler" (intro, "Caveats"): accept the
// longest prefix the target agrees with, correct at the first rejection, and
// only the proper acceptance rule keeps the target distribution. The rule is
// the one of "Fast Inference from Transformers via Speculative Decoding"
// (cited on "notes/dspark-deepseek", "Sources"): accept x with probability
// min(1, p(x)/q(x)); on rejection draw from norm(max(0, p - q)). "DSpark LLM
// inference speedup", "Speculative Decoding in Two Sentences": one bonus token
// is appended when the whole verified block is accepted.
//
// Design (B200): one thread-block cluster of C small CTAs (128 threads) per
// request; CTA `rank` owns vocabulary slice [rank*slice, rank*slice + slice).
// Clusters take requests in descending order of their cut, so that the
// longest chains of rows start in the first wave of resident clusters.
// A request's target rows are walked in order and the walk stops at the first
// rejection, so HBM sees only rows 0..a and one draft row. Each slice streams
// through a ring of 8 KB shared-memory slots filled by bulk asynchronous copies
// (cp.async.bulk; a "full" mbarrier per slot completes with the bytes, a
// per-warp "empty" arrival hands the slot back): no row is kept resident, so a
// CTA needs 35 KB of shared memory and every request of the batch is in flight
// at once. One online (max, sum 2^z) pass per row and one exchange over
// distributed shared memory give the row's normaliser. Every pass also leaves
// per-step, per-warp partial sums ("records"), so an inverse-CDF placement
// rescans one 8 KB step of one CTA (from L2) instead of its whole slice.
#include <algorithm>

#include "common.cuh"
#include "verify.cuh"

namespace dspark {

constexpr int kVThreads = 128;
constexpr int kVWarps = kVThreads / 32;
constexpr int kVBlocksPerSM = 6;  // 35 KB of shared memory each
constexpr int kSlotBytes = 8192;
constexpr int kRing = 4;
constexpr int kThreadBytes = kSlotBytes / kVThreads;  // contiguous bytes per thread per step
constexpr int kVecs = kThreadBytes / 16;              // 16-byte vectors per thread per step
constexpr int kMaxRec = 64;                           // placement records per CTA
constexpr int kMaxCluster = 16;

// One value each CTA publishes to its cluster per exchange.
struct __align__(16) Exch {
  float f0, f1, f2;
  int i0;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// --- thread-block cluster primitives (PTX) ---
__device__ __forceinline__ int cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return (int)r;
}
__device__ __forceinline__ int cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return (int)r;
}
// All threads of all CTAs of the cluster; release/acquire orders shared memory.
// The barrier instructions are warp-aligned, so the warp reconverges first.
__device__ __forceinline__ void cluster_sync() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Reads 16 bytes at the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint4 dsmem_load16(const void* local, int rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(remote)
               : "memory");
  return v;
}

// Combines the online pair (m2, s2) into (m, s); NaN propagates.
__device__ __forceinline__ void online_merge(float& m, float& s, float m2, float s2) {
  const float mm = fmaxf(m, m2);
  const float a = (m == -INFINITY) ? 0.f : s * ex2(m - mm);
  const float b = (m2 == -INFINITY) ? 0.f : s2 * ex2(m2 - mm);
  s = (s != s || s2 != s2) ? NAN : a + b;
  m = mm;
}

// NaN-propagating maximum over a warp.
__device__ __forceinline__ float warp_max_nan(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = max_nan(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

template <int DT>
struct VerifyCta {
  using E = Elem<DT>;
  using T = typename E::T;
  static constexpr int N = Vec16<DT>::N;                    // elements per 16-byte vector
  static constexpr int kStepElems = kSlotBytes / E::kBytes;
  static constexpr int kThreadElems = kThreadBytes / E::kBytes;

  int C, rank, tid, lane, warp;
  int lo, n;               // slice [lo, lo + n) of the vocabulary
  int G, nrec;             // ring steps per record, records in use
  unsigned char* ring;     // kRing slots of kSlotBytes
  uint64_t* bars;          // kRing "full" mbarriers (bytes landed)
  uint64_t* empty;         // kRing "empty" mbarriers (one arrival per warp)
  Exch* ex;                // [2] published slots (double buffered)
  Exch* got;               // [kMaxCluster] gathered copies (read-only after a gather)
  float2* rec;             // [kMaxRec][kVWarps] per record and warp: (reference max, sum)
  float* red;              // [32] scratch
  int* sint;               // [4] scratch
  int* dead;               // set once a wait gave up
  Status* st;
  int request;
  int parity;
  uint32_t issued, consumed;  // ring slot counters (identical in every thread)

  // ---------------- streaming through the ring ----------------
  __device__ void issue(const T* src, uint32_t bytes) {
    const uint32_t r = issued % kRing;
    const uint32_t use = issued / kRing;
    if (threadIdx.x == 0 && !*(volatile int*)dead) {
      // the slot's previous contents must have been read by every warp
      if (use > 0 && !mbar_wait_bounded(smem_u32(&empty[r]), (use - 1) & 1u)) {
        report_wait(st, kWhereVerifyLoad, request);
        *(volatile int*)dead = 1;
      }
    }
    if (threadIdx.x == 0 && !*(volatile int*)dead) {
      const uint32_t b = smem_u32(&bars[r]);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(b), "r"(bytes)
                   : "memory");
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              smem_u32(ring + r * kSlotBytes)),
          "l"(src), "r"(bytes), "r"(b)
          : "memory");
    }
    ++issued;
  }
  // every warp hands slot r back once it is done with it
  __device__ void release(uint32_t r) {
    __syncwarp();
    if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&empty[r])) : "memory");
  }
  __device__ const unsigned char* wait() {
    const uint32_t r = consumed % kRing;
    const uint32_t ph = (consumed / kRing) & 1u;
    if (!*(volatile int*)dead && !mbar_wait_bounded(smem_u32(&bars[r]), ph)) {
      if (threadIdx.x == 0) report_wait(st, kWhereVerifyLoad, request);
      mbar_wait_bounded(smem_u32(&bars[r]), ph);  // a last chance for an in-flight copy
      *(volatile int*)dead = 1;
    }
    __syncwarp();
    ++consumed;
    return ring + r * kSlotBytes;
  }
  __device__ int steps() const { return (n + kStepElems - 1) / kStepElems; }
  __device__ uint32_t step_bytes(int s) const {
    return (uint32_t)min(kStepElems, n - s * kStepElems) * E::kBytes;
  }
  __device__ bool record_end(int s) const { return (s + 1) % G == 0 || s + 1 == steps(); }

  // One pass over `nrow` (1 or 2) row slices, step by step, with no block
  // barrier inside: warps move through the ring independently and hand slots
  // back by arrivals. f(step, slot0, slot1) runs in every thread once the
  // step's slots have landed and must be done with them when it returns.
  template <class F>
  __device__ void pass(const T* r0, const T* r1, int nrow, F f) {
    const int ns = steps();
    const int ahead = kRing / nrow;
    int next = 0;
    for (; next < ns && next < ahead; ++next) {
      issue(r0 + next * kStepElems, step_bytes(next));
      if (nrow == 2) issue(r1 + next * kStepElems, step_bytes(next));
    }
    for (int s = 0; s < ns; ++s) {
      const uint32_t ra = consumed % kRing;
      const unsigned char* a = wait();
      const uint32_t rb = consumed % kRing;
      const unsigned char* b = (nrow == 2) ? wait() : nullptr;
      f(s, a, b);
      release(ra);
      if (nrow == 2) release(rb);
      if (next < ns) {
        issue(r0 + next * kStepElems, step_bytes(next));
        if (nrow == 2) issue(r1 + next * kStepElems, step_bytes(next));
        ++next;
      }
    }
    __syncthreads();
  }

  // A step gives thread t the 64 contiguous bytes [64 t, 64 t + 64) of its
  // slot. The thread reads its four 16-byte vectors in the rotated order
  // q ^ ((t >> 1) & 3), which spreads every 8-thread phase of a 128-bit
  // shared-memory load over all 32 banks.
  __device__ __forceinline__ int rot(int q) const { return q ^ ((tid >> 1) & 3); }
  __device__ __forceinline__ int vec_elem(int s, int q) const {
    return s * kStepElems + tid * kThreadElems + rot(q) * N;
  }
  __device__ __forceinline__ const unsigned char* vec_ptr(const unsigned char* slot, int q) const {
    return slot + tid * kThreadBytes + (rot(q) << 4);
  }

  // Publishes this CTA's value and gathers every CTA's (one cluster barrier).
  __device__ void gather(const Exch& mine) {
    if (tid == 0) ex[parity] = mine;
    cluster_sync();
    if (tid < C) {
      const uint4 v = dsmem_load16(&ex[parity], tid);
      got[tid] = Exch{__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), (int)v.w};
    }
    __syncthreads();
    parity ^= 1;
  }

  // CTA-wide online (max, sum) of the per-thread pairs
  __device__ float2 block_online(float m, float s) {
#pragma unroll
    for (int o = 16; o; o >>= 1)
      online_merge(m, s, __shfl_xor_sync(0xffffffffu, m, o), __shfl_xor_sync(0xffffffffu, s, o));
    if (lane == 0) {
      red[warp] = m;
      red[8 + warp] = s;
    }
    __syncthreads();
    float M = red[0], S = red[8];
    for (int w = 1; w < kVWarps; ++w) online_merge(M, S, red[w], red[8 + w]);
    __syncthreads();
    return make_float2(M, S);
  }
  __device__ float block_sum(float v) {
    v = warp_sum(v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = 0.f;
    for (int w = 0; w < kVWarps; ++w) t += red[w];
    __syncthreads();
    return t;
  }

  // CTA-wide online (max, sum 2^(z - max)) of z = v * cs over the slice of
  // `row`. The reference maximum moves per warp and step (warp-uniform), and
  // every record keeps its warp's (maximum, sum) for a later placement.
  __device__ float2 row_stats(const T* row, float cs) {
    float m = -INFINITY, sum = 0.f, rs = 0.f;
    pass(row, nullptr, 1, [&](int s, const unsigned char* a, const unsigned char*) {
      float v[kVecs][N];
      float vm = -INFINITY;
#pragma unroll
      for (int q = 0; q < kVecs; ++q) {
        if (vec_elem(s, q) < n) {
          Vec16<DT>::load(vec_ptr(a, q), v[q]);
        } else {
#pragma unroll
          for (int j = 0; j < N; ++j) v[q][j] = -INFINITY;
        }
#pragma unroll
        for (int j = 0; j < N; ++j) vm = max_nan(vm, v[q][j]);
      }
      const float zm = warp_max_nan(vm) * cs;
      if (zm != zm) {  // a NaN in this step: the sums stay NaN from here on
        sum = NAN;
        rs = NAN;
      } else {
        if (zm > m) {
          const float sc = (m == -INFINITY) ? 0.f : ex2(m - zm);
          sum *= sc;
          rs *= sc;
          m = zm;
        }
        if (m != -INFINITY) {  // entries at -inf weigh nothing; +inf makes the sum NaN
          const float neg = -m;
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int q = 0; q < kVecs; ++q)
#pragma unroll
            for (int j = 0; j < N; ++j) acc[j & 3] += ex2(fmaf(v[q][j], cs, neg));
          const float t = (acc[0] + acc[1]) + (acc[2] + acc[3]);
          sum += t;
          rs += t;
        }
      }
      if (record_end(s)) {
        const float t = warp_sum(rs);
        if (lane == 0) rec[(s / G) * kVWarps + warp] = make_float2(m, t);
        rs = 0.f;
      }
    });
    return block_online(m, sum);
  }

  // A target row's normaliser (max z, sum 2^(z - max z)) from its chunk
  // partials, combined in the same order in every CTA.
  __device__ float2 stats_norm(const float2* P, int nst) {
    float m = -INFINITY, sum = 0.f;
    for (int c = tid; c < nst; c += kVThreads) {
      const float2 q = P[c];
      online_merge(m, sum, q.x, q.y);
    }
    return block_online(m, sum);
  }

  // A greedy row's (max, lowest argmax) from its chunk partials; bad when a
  // chunk reported NaN or +inf (its maximum is NaN).
  __device__ void stats_argmax(const float2* P, int nst, float& mv, int& mi, bool& bad) {
    float m = -INFINITY;
    int i = 0x7fffffff;
    bool b = false;
    for (int c = tid; c < nst; c += kVThreads) {
      const float2 q = P[c];
      b |= (q.x != q.x);
      argmax_merge(m, i, q.x, __float_as_int(q.y));
    }
    warp_argmax(m, i);
    b = __any_sync(0xffffffffu, b);
    if (lane == 0) {
      red[warp] = m;
      reinterpret_cast<int*>(red)[8 + warp] = i;
      reinterpret_cast<int*>(red)[16 + warp] = b;
    }
    __syncthreads();
    mv = red[0];
    mi = reinterpret_cast<int*>(red)[8];
    bad = reinterpret_cast<int*>(red)[16] != 0;
    for (int w = 1; w < kVWarps; ++w) {
      argmax_merge(mv, mi, red[w], reinterpret_cast<int*>(red)[8 + w]);
      bad |= reinterpret_cast<int*>(red)[16 + w] != 0;
    }
    __syncthreads();
  }

  // Inclusive scan of one value per thread over the CTA (thread order); also
  // returns the CTA total. Uses red[0..kVWarps).
  __device__ float block_scan(float v, float& total) {
    const float incl = warp_inclusive_scan(v);
    if (lane == 31) red[warp] = incl;
    __syncthreads();
    float before = 0.f, tot = 0.f;
    for (int w = 0; w < kVWarps; ++w) {
      if (w < warp) before += red[w];
      tot += red[w];
    }
    __syncthreads();
    total = tot;
    return before + incl;
  }

  // Inverse-CDF draw from the weights 2^(t cs - M) of a whole target row
  // (index order, strict ">"; past the end: the last positive entry), with
  // thr = u * Z. The crossing chunk is located from the row's chunk partials
  // P (their masses rescaled to M), then only that chunk of the row is read
  // again. Runs in one CTA; returns the token in every thread, -2 when no
  // entry has positive weight.
  __device__ int place_row(const T* row, const float2* P, int nst, int V, float thr, float cs, float M) {
    int* found = sint;  // [0] crossing chunk, [1] last positive chunk
    if (tid == 0) {
      found[0] = 0x7fffffff;
      found[1] = -1;
    }
    __syncthreads();
    float before = 0.f;  // mass of the chunks of earlier rounds
    float rem = -1.f;
    for (int c0 = 0; c0 < nst; c0 += kVThreads) {
      const int c = c0 + tid;
      float w = 0.f;
      if (c < nst) {
        const float2 q = P[c];
        w = (q.x == -INFINITY) ? 0.f : q.y * ex2(q.x - M);
      }
      float tot;
      const float incl = block_scan(w, tot);
      if (w > 0.f) {
        atomicMax(&found[1], c);
        if (thr < before + incl) atomicMin(&found[0], c);
      }
      __syncthreads();
      if (found[0] != 0x7fffffff) {
        // this thread's exclusive prefix is read by the owner below
        if (c == found[0]) red[16] = thr - (before + incl - w);
        __syncthreads();
        rem = red[16];
        break;
      }
      before += tot;
    }
    int ch = found[0];
    if (ch == 0x7fffffff) {  // rounding: past the total, the last positive chunk
      ch = found[1];
      rem = INFINITY;
    }
    __syncthreads();
    if (ch < 0) return -2;
    // rescan chunk ch: thread t weighs 16 bytes (N entries) in index order
    constexpr int CE = kStatChunkBytes / E::kBytes;
    const int e0 = ch * CE + tid * N;
    float w[N];
    float ts = 0.f;
    const bool ok = e0 < V;
    float v[N];
    if (ok) Vec16<DT>::load(row + e0, v);
#pragma unroll
    for (int j = 0; j < N; ++j) {
      w[j] = ok ? ex2(fmaf(v[j], cs, -M)) : 0.f;
      ts += w[j];
    }
    float tot;
    const float incl = block_scan(ts, tot);
    if (tid == 0) {
      sint[2] = 0x7fffffff;
      sint[3] = -1;
    }
    __syncthreads();
    if (ts > 0.f) {
      atomicMax(&sint[3], tid);
      if (rem < incl) atomicMin(&sint[2], tid);
    }
    __syncthreads();
    int tt = sint[2];
    const bool fallback = tt == 0x7fffffff;
    if (fallback) tt = sint[3];
    int tok = -2;
    if (tid == tt) {
      float r2 = rem - (incl - ts);
      int f = -1, lp = -1;
#pragma unroll
      for (int j = 0; j < N; ++j) {
        if (w[j] > 0.f) lp = j;
        if (f < 0 && !fallback && w[j] > 0.f && r2 < w[j]) f = j;
        if (f < 0) r2 -= w[j];
      }
      red[17] = __int_as_float(e0 + (f < 0 ? lp : f));
    }
    __syncthreads();
    if (tt >= 0) tok = __float_as_int(red[17]);
    __syncthreads();
    return tok;
  }

  // Inverse-CDF placement of `thr` on the weights wfun(t_value, d_value) of
  // the cluster's slices, in index order. rw[r] are the per-rank totals
  // (identical in every CTA). The owning CTA finds the record holding the
  // crossing from the last pass's records (recw gives a record's weight), then
  // rescans only that record's steps, straight from global memory. It returns
  // the token in every thread; the other CTAs return -1, and -2 means that no
  // rank holds positive mass. No cluster exchange happens here.
  template <class F, class R>
  __device__ int place(float thr, const float* rw, const T* r0, const T* r1, F wfun, R recw) {
    int owner = -1, lastpos = -1;
    float P = 0.f, Pown = 0.f;
    for (int r = 0; r < C; ++r) {
      const float sr = rw[r];
      if (sr > 0.f) {
        lastpos = r;
        if (owner < 0 && thr < P + sr) {
          owner = r;
          Pown = P;
        }
      }
      P += sr;
    }
    bool fallback = false;
    if (owner < 0) {
      owner = lastpos;
      fallback = true;
    }
    if (owner < 0) return -2;
    if (owner != rank) return -1;
    float rem = fallback ? INFINITY : thr - Pown;
    // the record holding the crossing (the same walk in every thread)
    int g0 = -1, glast = -1;
    for (int g = 0; g < nrec; ++g) {
      float wg = 0.f;
      for (int w = 0; w < kVWarps; ++w) wg += recw(rec[g * kVWarps + w]);
      if (wg > 0.f) {
        glast = g;
        if (g0 < 0 && rem < wg) g0 = g;
      }
      if (g0 < 0) rem -= wg;
    }
    if (g0 < 0) {  // rounding: past the last record; its last positive element
      g0 = max(glast, 0);
      rem = INFINITY;
    }
    // rescan the record's steps: thread t weighs its kThreadElems contiguous
    // elements of each step in index order
    const int s_end = min(steps(), (g0 + 1) * G);
    int found = -1, lastp = -1;
    for (int s = g0 * G; s < s_end && found < 0; ++s) {
      const int e0 = s * kStepElems + tid * kThreadElems;
      float w[kThreadElems];
      float ts = 0.f;
#pragma unroll
      for (int q = 0; q < kVecs; ++q) {
        float tv[N], dv[N];
        const bool ok = e0 + q * N < n;
        if (ok) {
          Vec16<DT>::load(r0 + e0 + q * N, tv);
          if (r1) Vec16<DT>::load(r1 + e0 + q * N, dv);
        }
#pragma unroll
        for (int j = 0; j < N; ++j) {
          w[q * N + j] = ok ? wfun(tv[j], r1 ? dv[j] : 0.f) : 0.f;
          ts += w[q * N + j];
          if (w[q * N + j] > 0.f) lastp = e0 + q * N + j;
        }
      }
      // exclusive prefix of the thread sums over the step (thread order is index order)
      const float incl_w = warp_inclusive_scan(ts);
      if (lane == 31) red[warp] = incl_w;
      if (tid == 0) sint[1] = 0x7fffffff;
      __syncthreads();
      float excl = incl_w - ts, tot = 0.f;
      for (int k = 0; k < kVWarps; ++k) {
        if (k < warp) excl += red[k];
        tot += red[k];
      }
      if (rem < tot && ts > 0.f && rem < excl + ts) atomicMin(&sint[1], tid);
      __syncthreads();
      const int kt = sint[1];
      if (rem < tot && kt != 0x7fffffff) {
        if (tid == kt) {
          float r2 = rem - excl;
          int f = -1, lp = -1;
#pragma unroll
          for (int j = 0; j < kThreadElems; ++j) {
            if (w[j] > 0.f) lp = j;
            if (f < 0 && w[j] > 0.f && r2 < w[j]) f = j;
            if (f < 0) r2 -= w[j];
          }
          sint[0] = e0 + (f < 0 ? lp : f);
        }
        __syncthreads();
        found = sint[0];
      }
      if (found < 0) rem -= tot;
      __syncthreads();  // red and sint are free again
    }
    if (found < 0) {  // no crossing (rounding only): the last element of positive weight
      if (tid == 0) sint[2] = -1;
      __syncthreads();
      atomicMax(&sint[2], lastp);
      __syncthreads();
      found = max(sint[2], 0);
    }
    return lo + found;
  }
};

// Combined (max, sum) of the gathered per-CTA online pairs (f0, f1), in rank order.
__device__ __forceinline__ float2 combine_ranks(const Exch* got, int C) {
  float M = -INFINITY;
  for (int r = 0; r < C; ++r) M = fmaxf(M, got[r].f0);
  float Z = 0.f;
  for (int r = 0; r < C; ++r) {
    const float s = got[r].f1;
    if (s != s) return make_float2(M, NAN);
    Z += (got[r].f0 == -INFINITY) ? 0.f : s * ex2(got[r].f0 - M);
  }
  return make_float2(M, Z);
}

// Cluster q verifies the request of rank q in the order (cut descending,
// index ascending): the longest chains of rows start in the first wave of
// clusters and the requests that verify a single row take the slots that free
// up last. The statistics pass writes this order once (a.order); without it
// every CTA of the cluster computes the same answer: a histogram of the
// (clamped) cuts, the cut value whose range holds q, then the position of the
// request among those with that cut, in index order.
__device__ int request_of(const VerifyArgs& a, int q, int* cnt, int* s_req) {
  if (!a.cut) return q;
  if (a.order) return a.order[q];  // the same order, made once by the statistics pass
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = a.K;
  for (int v = tid; v <= K; v += kVThreads) cnt[v] = 0;
  __syncthreads();
  for (int i = tid; i < a.B; i += kVThreads) {
    const int L = min(max(a.cut[i], 0), K);
    atomicAdd(&cnt[L], 1);
  }
  __syncthreads();
  if (tid < 32) {
    // the cut value v whose rank range [base, base + cnt[v]) holds q
    int base = 0, v = K;
    for (; v > 0 && q >= base + cnt[v]; --v) base += cnt[v];
    // the (q - base)-th request with cut v, in index order
    int want = q - base, found = -1;
    for (int i0 = 0; i0 < a.B && found < 0; i0 += 32) {
      const int i = i0 + lane;
      const bool hit = i < a.B && min(max(a.cut[i], 0), K) == v;
      const unsigned m = __ballot_sync(0xffffffffu, hit);
      const int n = __popc(m);
      if (want < n) {
        unsigned mm = m;
        for (int k = 0; k < want; ++k) mm &= mm - 1;
        found = i0 + __ffs(mm) - 1;
      } else {
        want -= n;
      }
    }
    if (lane == 0) *s_req = found < 0 ? q : found;
  }
  (void)warp;
  __syncthreads();
  return *s_req;
}

template <int DT>
__global__ void __launch_bounds__(kVThreads, kVBlocksPerSM) verify_kernel(VerifyArgs a) {
  using E = Elem<DT>;
  using T = typename E::T;
  __shared__ __align__(128) unsigned char ring[kRing * kSlotBytes];
  __shared__ __align__(8) uint64_t bars[kRing];
  __shared__ __align__(8) uint64_t empty[kRing];
  __shared__ Exch ex[2];
  __shared__ Exch got[kMaxCluster];
  __shared__ float rw[kMaxCluster];
  __shared__ float2 rec[kMaxRec * kVWarps];
  __shared__ float red[32];
  __shared__ int sint[4];
  __shared__ int dead;
  __shared__ int cnt_by_cut[65];
  __shared__ int s_req;

  VerifyCta<DT> c;
  c.C = cluster_size();
  c.rank = cluster_rank();
  c.tid = threadIdx.x;
  c.lane = c.tid & 31;
  c.warp = c.tid >> 5;
  c.ring = ring;
  c.bars = bars;
  c.empty = empty;
  c.ex = ex;
  c.got = got;
  c.rec = rec;
  c.red = red;
  c.sint = sint;
  c.dead = &dead;
  c.st = a.status;
  c.parity = 0;
  c.issued = 0;
  c.consumed = 0;
  const int b = request_of(a, blockIdx.x / c.C, cnt_by_cut, &s_req);
  c.request = b;
  c.lo = c.rank * a.slice;
  c.n = max(0, min(a.slice, a.V - c.lo));
  c.G = max(1, (c.steps() + kMaxRec - 1) / kMaxRec);
  c.nrec = (c.steps() + c.G - 1) / c.G;
  Status* st = a.status;
  const int tid = c.tid;

  if (tid == 0) {
    dead = 0;
    for (int i = 0; i < kRing; ++i) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars[i])) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(&empty[i])), "r"(kVThreads / 32)
                   : "memory");
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  const int K = a.K, V = a.V;
  int L = a.cut ? a.cut[b] : K;
  if (L < 0 || L > K) {
    if (tid == 0 && c.rank == 0) report(st, DSPARK_STATUS_BAD_CUT, b);
    L = L < 0 ? 0 : K;
  }
  const float tau = a.temp[b];
  if (tau != tau || tau < 0.f) {
    if (tid == 0 && c.rank == 0) report(st, DSPARK_STATUS_BAD_TEMP, b);
  }
  const bool greedy = !(tau > 0.f);
  const float cs = greedy ? 1.f : kLog2e / tau;
  const T* target = static_cast<const T*>(a.target) + (long long)b * (K + 1) * V;
  const T* drow0 = static_cast<const T*>(a.d) + (long long)b * K * V;

  int acc = 0;
  bool rejected = false;
  bool badrow = false;
  float M = 0.f, Z = 0.f;  // current target row's max (z units) and sum
  int y = -1;
  const float2* stat_b = a.stats + (long long)b * (K + 1) * a.nstat;

  // The walk needs no pass over the rows: their normalisers come from the
  // target statistics, and every CTA of the cluster takes the same decisions
  // from the same partials.
  for (int j = 0; j <= L; ++j) {
    const T* row = target + (long long)j * V;
    const float2* P = stat_b + (long long)j * a.nstat;
    const int xk = (j < L) ? a.x[(long long)b * K + j] : -1;
    if (j < L && (xk < 0 || xk >= V) && tid == 0 && c.rank == 0) report(st, DSPARK_STATUS_BAD_TOKEN, b);
    if (greedy) {
      float gm;
      int gi;
      bool gbad;
      c.stats_argmax(P, a.nstat, gm, gi, gbad);
      if (gbad || gm == -INFINITY) {
        badrow = true;
        gi = 0;
      }
      if (j == L || badrow || xk != gi) {
        rejected = (j < L);
        y = gi;
        break;
      }
      ++acc;
      continue;
    }
    const float2 MZ = c.stats_norm(P, a.nstat);
    M = MZ.x;
    Z = MZ.y;
    if (!(Z > 0.f) || Z == INFINITY || M == -INFINITY || M == INFINITY) {
      badrow = true;
      rejected = (j < L);
      y = 0;
      break;
    }
    if (j == L) {  // every verified draft accepted: bonus token from p of row L (rank 0 draws it)
      if (c.rank == 0) {
        const float u = uniform24(a.seed, a.round_id, (uint32_t)b, (uint32_t)(acc + 1), kBonus);
        y = c.place_row(row, P, a.nstat, V, u * Z, cs, M);
      }
      break;
    }
    const float tx = (xk >= 0 && xk < V) ? E::load(row, xk) * cs : -INFINITY;
    const float p = ex2(tx - M) / Z;
    const float u = uniform24(a.seed, a.round_id, (uint32_t)b, (uint32_t)(j + 1), kAccept);
    if (!(u < p / a.q_tok[(long long)b * K + j])) {
      rejected = true;
      break;
    }
    ++acc;
  }

  if (rejected && !greedy && !badrow) {
    // residual norm(max(0, p - q)) over target row acc and draft row acc: the
    // one streaming pass of the kernel
    const T* trow = target + (long long)acc * V + c.lo;
    const T* drow = drow0 + (long long)acc * V + c.lo;
    // the draft row's normaliser: from the draw that produced it when the
    // caller passes it on, else one more pass over the draft row
    float2 MZq;
    if (a.q_norm) {
      MZq = a.q_norm[(long long)b * K + acc];
    } else {
      const float2 mq = c.row_stats(drow, cs);
      c.gather(Exch{mq.x, mq.y, 0.f, 0});
      MZq = combine_ranks(got, c.C);
    }
    const float Mq = MZq.x, iZ = 1.f / Z, iZq = 1.f / MZq.y;
    auto resid = [&](float tv, float dv) {
      const float pp = ex2(fmaf(tv, cs, -M)) * iZ;
      const float qq = ex2(fmaf(dv, cs, -Mq)) * iZq;
      return fmaxf(0.f, pp - qq);
    };
    float sr = 0.f, rs = 0.f;
    c.pass(trow, drow, 2, [&](int s, const unsigned char* ta, const unsigned char* da) {
      constexpr int N = Vec16<DT>::N;
      float acc2[2] = {0.f, 0.f};
#pragma unroll
      for (int q = 0; q < kVecs; ++q) {
        if (c.vec_elem(s, q) >= c.n) continue;
        float tv[N], dv[N];
        Vec16<DT>::load(c.vec_ptr(ta, q), tv);
        Vec16<DT>::load(c.vec_ptr(da, q), dv);
#pragma unroll
        for (int jj = 0; jj < N; ++jj) acc2[jj & 1] += resid(tv[jj], dv[jj]);
      }
      sr += acc2[0] + acc2[1];
      rs += acc2[0] + acc2[1];
      if (c.record_end(s)) {
        const float t = warp_sum(rs);
        if (c.lane == 0) rec[(s / c.G) * kVWarps + c.warp] = make_float2(0.f, t);
        rs = 0.f;
      }
    });
    const float totr = c.block_sum(sr);
    c.gather(Exch{0.f, totr, 0.f, 0});
    float R = 0.f;
    for (int r = 0; r < c.C; ++r) R += got[r].f1;
    if (tid < c.C) rw[tid] = got[tid].f1;
    __syncthreads();
    const float u = uniform24(a.seed, a.round_id, (uint32_t)b, (uint32_t)(acc + 1), kResidual);
    if (R > 0.f) {
      y = c.place(u * R, rw, trow, drow, resid, [](float2 r) { return r.y; });
    } else if (c.rank == 0) {
      // exact-zero residual (floating point only): draw from p instead
      y = c.place_row(target + (long long)acc * V, stat_b + (long long)acc * a.nstat, a.nstat, V,
                      u * Z, cs, M);
    }
  }

  // emission: rank 0 writes the request's header and drafts; the CTA that
  // placed the final token (any rank for sampled rows) writes it
  if (y == -2) badrow = true;  // no positive mass anywhere (cannot happen with Z > 0)
  const bool y_here = (greedy || badrow) ? (c.rank == 0) : (y >= 0);
  if (badrow && tid == 0 && c.rank == 0) report(st, DSPARK_STATUS_BAD_ROW, b);
  if (c.rank == 0) {
    for (int i = tid; i <= K; i += kVThreads) {
      int v = -1;
      if (i < acc) v = a.x[(long long)b * K + i];
      if (i != acc) a.out[(long long)b * (K + 1) + i] = v;
    }
    if (tid == 0) {
      a.accepted[b] = acc;
      a.n_emit[b] = acc + 1;
    }
  }
  if (y_here && tid == 0) a.out[(long long)b * (K + 1) + acc] = (greedy || !badrow) ? max(y, 0) : 0;
  cluster_sync();  // no CTA leaves while a peer may still read its shared memory
}

int verify_cluster_size(int B, int V, int dtype, int num_sms) {
  // Enough CTAs in flight to keep HBM busy (kVBlocksPerSM 128-thread CTAs per
  // SM), at most 16 per request, and at least one ring step per CTA. Measured
  // on B200 at B = 256, V = 129280: C = 4 (about 1.15 waves) beats 3 (one
  // wave), 2, 6, 8 and 16.
  const int es = dtype == DSPARK_F32 ? 4 : 2;
  const long long slots = (long long)kVBlocksPerSM * num_sms;
  int C = 1;
  while (C < kMaxCluster && (long long)B * C * 2 * 5 <= slots * 6 &&
         (long long)V * es / (2 * C) >= kSlotBytes)
    C <<= 1;
  return C;
}

// Vocabulary entries per CTA: an equal share, rounded up to a multiple of 8
// (every slice starts on a 16-byte boundary).
static int verify_slice(int V, int C) { return ((V + C - 1) / C + 7) & ~7; }

cudaError_t verify_launch(VerifyArgs a, int C, cudaStream_t s) {
  a.slice = verify_slice(a.V, C);
  auto kern = (a.dtype == DSPARK_F32) ? verify_kernel<DSPARK_F32> : verify_kernel<DSPARK_BF16>;
  if (C > 8) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.B * C));
  cfg.blockDim = dim3(kVThreads);
  cfg.dynamicSmemBytes = 0;  // the ring and the bookkeeping are static shared memory
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace dspark
