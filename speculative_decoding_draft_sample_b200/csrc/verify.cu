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
// Design (B200): one thread-block cluster of C CTAs per request; CTA `rank`
// owns vocabulary slice [rank*slice, rank*slice + slice). The request's target
// rows are walked in order and the walk stops at the first rejection, so only
// rows 0..a and one draft row are ever read. Each row slice lands in shared
// memory with one bulk asynchronous copy (cp.async.bulk, completion on an
// mbarrier); every reduction across the cluster goes through distributed
// shared memory. The residual pass re-reads the target row from shared memory,
// so HBM sees every byte once.
#include "common.cuh"
#include "verify.cuh"

namespace dspark {

constexpr int kVThreads = 256;
constexpr int kMaxCluster = 8;

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

// Bulk copy of `bytes` (multiple of 16) from global to this CTA's shared memory,
// completing on `bar`; every thread then waits (bounded) for phase `phase`.
__device__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                          uint32_t& phase, Status* st, int request, int* dead) {
  if (*(volatile int*)dead) {  // this CTA already gave up once: no more copies or waits
    phase ^= 1u;
    return;
  }
  const uint32_t b = smem_u32(bar);
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(b), "r"(bytes)
                 : "memory");
    for (uint32_t off = 0; off < bytes; off += 16384) {
      const uint32_t n = min(16384u, bytes - off);
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              smem_u32(static_cast<char*>(dst) + off)),
          "l"(static_cast<const char*>(src) + off), "r"(n), "r"(b)
          : "memory");
    }
  }
  if (!mbar_wait_bounded(b, phase)) {
    if (threadIdx.x == 0) report_wait(st, kWhereVerifyLoad, request);
    mbar_wait_bounded(b, phase);  // give an in-flight copy a last chance to land
    *(volatile int*)dead = 1;
  }
  __syncwarp();
  __syncthreads();  // every thread sees the same `dead` before the next copy
  phase ^= 1u;
}

// 16 bytes of shared memory as floats (8 bf16 or 4 fp32), in index order.
template <int DT>
struct Vec16;
template <>
struct Vec16<DSPARK_BF16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const uint16_t* p, float* v) {
    const uint4 q = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = __uint_as_float(w[j] << 16);
      v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
  }
};
template <>
struct Vec16<DSPARK_F32> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float* p, float* v) {
    const float4 q = *reinterpret_cast<const float4*>(p);
    v[0] = q.x;
    v[1] = q.y;
    v[2] = q.z;
    v[3] = q.w;
  }
};

template <int DT>
struct VerifyCta {
  using E = Elem<DT>;
  using T = typename E::T;

  int C, rank, tid, lane, warp;
  int lo, n, per, t0, t1;  // slice [lo, lo+n); this thread's elements [t0, t1) of it
  Exch* ex;                // [2] published slots (double buffered)
  Exch* got;               // [kMaxCluster] gathered copies (read-only after a gather)
  float* rw;               // [kMaxCluster] per-rank weights of the placement at hand
  float* pm;               // [kVThreads] per-thread running max (online rows)
  float* ps;               // [kVThreads] per-thread sums
  float* excl;             // [kVThreads] exclusive block scan of the weights
  float* red;              // [32] scratch
  int* sint;               // [4] scratch
  int parity;

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

  // f(i, value) over this thread's elements of `buf`, in index order, 16 B at a time
  template <class F>
  __device__ __forceinline__ void each(const T* buf, F f) const {
    constexpr int N = Vec16<DT>::N;
    for (int i = t0; i < t1; i += N) {
      float v[N];
      Vec16<DT>::load(buf + i, v);
#pragma unroll
      for (int j = 0; j < N; ++j) f(i + j, v[j]);
    }
  }
  template <class F>
  __device__ __forceinline__ void each2(const T* b1, const T* b2, F f) const {
    constexpr int N = Vec16<DT>::N;
    for (int i = t0; i < t1; i += N) {
      float v1[N], v2[N];
      Vec16<DT>::load(b1 + i, v1);
      Vec16<DT>::load(b2 + i, v2);
#pragma unroll
      for (int j = 0; j < N; ++j) f(i + j, v1[j], v2[j]);
    }
  }

  // Online (max, sum 2^(z - max)) of z = v * cs over this thread's elements,
  // kept in pm/ps for a later placement; returns the CTA's pair (thread 0's
  // result is the one published). NaN or +inf anywhere makes the sum NaN.
  __device__ float2 online_stats(const T* buf, float cs) {
    constexpr int N = Vec16<DT>::N;
    float m = -INFINITY, sum = 0.f;
    for (int i = t0; i < t1; i += N) {
      float v[N];
      Vec16<DT>::load(buf + i, v);
      float vm = v[0];
#pragma unroll
      for (int j = 1; j < N; ++j) vm = max_nan(vm, v[j]);
      const float zm = vm * cs;
      if (zm != zm) {  // NaN in this vector
        sum = NAN;
        continue;
      }
      if (zm > m) {
        sum = (m == -INFINITY) ? sum : sum * ex2(m - zm);
        m = zm;
      }
      if (m != -INFINITY) {  // entries at -inf weigh nothing; +inf makes the sum NaN
        const float neg = -m;
#pragma unroll
        for (int j = 0; j < N; ++j) sum += ex2(fmaf(v[j], cs, neg));
      }
    }
    pm[tid] = m;
    ps[tid] = sum;
    // warp combine, then the 8 warp results
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
      const float s2 = __shfl_xor_sync(0xffffffffu, sum, o);
      const float mm = fmaxf(m, m2);
      const float a = (m == -INFINITY) ? 0.f : sum * ex2(m - mm);
      const float b = (m2 == -INFINITY) ? 0.f : s2 * ex2(m2 - mm);
      sum = (sum != sum || s2 != s2) ? NAN : a + b;
      m = mm;
    }
    if (lane == 0) {
      red[warp] = m;
      red[8 + warp] = sum;
    }
    __syncthreads();
    float M = red[0], S = red[8];
    for (int w = 1; w < kVThreads / 32; ++w) {
      const float mm = fmaxf(M, red[w]);
      const float a = (M == -INFINITY) ? 0.f : S * ex2(M - mm);
      const float b = (red[w] == -INFINITY) ? 0.f : red[8 + w] * ex2(red[w] - mm);
      S = (S != S || red[8 + w] != red[8 + w]) ? NAN : a + b;
      M = mm;
    }
    __syncthreads();
    return make_float2(M, S);
  }

  // Block sum of per-thread values (also kept in ps for a later placement).
  __device__ float block_sum_keep(float v) {
    ps[tid] = v;
    pm[tid] = 0.f;  // weights are ps * 2^(pm - 0)
    const float w = warp_sum(v);
    if (lane == 0) red[warp] = w;
    __syncthreads();
    float t = 0.f;
    for (int i = 0; i < kVThreads / 32; ++i) t += red[i];
    __syncthreads();
    return t;
  }

  // Inverse-CDF placement of `thr` on weights wfun(i) (slice-local index i).
  // Per-rank totals are rw[r]; this thread's total weight is
  // ps[tid] * 2^(pm[tid] - Mref). Returns the global token index in every
  // thread of the owning CTA, -1 in the other CTAs, and -2 everywhere if no
  // rank holds positive mass. No cluster exchange happens here.
  template <class F>
  __device__ int place(float thr, float Mref, F wfun) {
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
    // this thread's weight and its exclusive prefix in index order
    const float wt = (pm[tid] == -INFINITY) ? 0.f : ps[tid] * ex2(pm[tid] - Mref);
    const float incl = warp_inclusive_scan(wt);
    if (lane == 31) red[warp] = incl;
    __syncthreads();
    float pre = 0.f;
    for (int w = 0; w < warp; ++w) pre += red[w];
    const float ex_t = pre + incl - wt;
    const float rem = fallback ? INFINITY : thr - Pown;
    if (tid == 0) sint[1] = 0x7fffffff;
    __syncthreads();
    if (wt > 0.f && rem < ex_t + wt) atomicMin(&sint[1], tid);
    __syncthreads();
    int ot = sint[1];
    bool tfall = fallback;
    if (ot == 0x7fffffff) {  // rounding: last thread with positive mass
      if (tid == 0) sint[2] = -1;
      __syncthreads();
      if (wt > 0.f) atomicMax(&sint[2], tid);
      __syncthreads();
      ot = sint[2];
      tfall = true;
    }
    if (tid == 0) sint[3] = -1;
    __syncthreads();
    if (tid == ot) {
      float r2 = tfall ? INFINITY : rem - ex_t;
      int found = -1, lastp = -1;
      for (int i = t0; i < t1; ++i) {
        const float w = wfun(i);
        if (w > 0.f) lastp = i;
        if (r2 < w) {
          found = i;
          break;
        }
        r2 -= w;
      }
      if (found < 0) found = lastp;
      sint[3] = found;
    }
    __syncthreads();
    const int f = sint[3];
    __syncthreads();
    return f < 0 ? lo : lo + f;
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

template <int DT>
__global__ void __launch_bounds__(kVThreads) verify_kernel(VerifyArgs a) {
  using E = Elem<DT>;
  using T = typename E::T;
  extern __shared__ __align__(128) unsigned char dsm[];
  __shared__ Exch ex[2];
  __shared__ Exch got[kMaxCluster];
  __shared__ float rw[kMaxCluster];
  __shared__ float pm[kVThreads], ps[kVThreads], excl[kVThreads], red[32];
  __shared__ int sint[4];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int dead;

  VerifyCta<DT> c;
  c.C = cluster_size();
  c.rank = cluster_rank();
  c.tid = threadIdx.x;
  c.lane = c.tid & 31;
  c.warp = c.tid >> 5;
  c.ex = ex;
  c.got = got;
  c.rw = rw;
  c.pm = pm;
  c.ps = ps;
  c.excl = excl;
  c.red = red;
  c.sint = sint;
  c.parity = 0;
  const int b = blockIdx.x / c.C;
  c.lo = c.rank * a.slice;
  c.n = max(0, min(a.slice, a.V - c.lo));
  {
    // each thread: a contiguous run of an odd number of 16-byte chunks, so that
    // the 16-byte shared-memory loads of a quarter warp fall in distinct banks
    constexpr int v16 = Vec16<DT>::N;
    int per = (c.n + kVThreads - 1) / kVThreads;
    per = (per + v16 - 1) / v16 * v16;
    if (((per / v16) & 1) == 0) per += v16;
    c.per = per;
  }
  c.t0 = min(c.tid * c.per, c.n);
  c.t1 = min(c.t0 + c.per, c.n);
  T* tb = reinterpret_cast<T*>(dsm);
  T* db = reinterpret_cast<T*>(dsm + a.slice_bytes_padded);
  Status* st = a.status;
  const int tid = c.tid;

  if (tid == 0) {
    dead = 0;
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  uint32_t phase = 0;

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
  const uint32_t nbytes = (uint32_t)c.n * E::kBytes;

  int acc = 0;
  bool rejected = false;
  bool badrow = false;
  float M = 0.f, Z = 0.f;  // current target row's max (z units) and sum
  int y = -1;

  for (int j = 0; j <= L; ++j) {
    bulk_load(tb, target + (long long)j * V + c.lo, nbytes, &bar, phase, st, b, &dead);
    const int xk = (j < L) ? a.x[(long long)b * K + j] : -1;
    if (j < L && (xk < 0 || xk >= V) && tid == 0 && c.rank == 0) report(st, DSPARK_STATUS_BAD_TOKEN, b);
    if (greedy) {
      float mv = -INFINITY, chk = -INFINITY;
      int mi = 0x7fffffff;
      c.each(tb, [&](int i, float v) {
        chk = max_nan(chk, v);
        if (v > mv) {
          mv = v;
          mi = c.lo + i;
        }
      });
      warp_argmax(mv, mi);
#pragma unroll
      for (int o = 16; o; o >>= 1) chk = max_nan(chk, __shfl_xor_sync(0xffffffffu, chk, o));
      if (c.lane == 0) {
        red[c.warp] = mv;
        red[8 + c.warp] = chk;
        reinterpret_cast<int*>(red)[16 + c.warp] = mi;
      }
      __syncthreads();
      float m = red[0], ck = red[8];
      int mm = reinterpret_cast<int*>(red)[16];
      for (int w = 1; w < kVThreads / 32; ++w) {
        argmax_merge(m, mm, red[w], reinterpret_cast<int*>(red)[16 + w]);
        ck = max_nan(ck, red[8 + w]);
      }
      __syncthreads();
      const bool bad = (ck != ck) || ck == INFINITY;
      c.gather(Exch{m, 0.f, 0.f, mm | (bad ? (int)0x80000000 : 0)});
      float gm = -INFINITY;
      int gi = 0x7fffffff;
      bool gbad = false;
      for (int r = 0; r < c.C; ++r) {
        argmax_merge(gm, gi, got[r].f0, got[r].i0 & 0x7fffffff);
        gbad |= got[r].i0 < 0;
      }
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

    // one online pass: (max, sum) of z = t * cs, and t[x] of the draft tested
    const float2 mz = c.online_stats(tb, cs);
    float tx = -INFINITY;
    if (xk >= c.lo && xk < c.lo + c.n) tx = E::to_float(tb[xk - c.lo]) * cs;
    c.gather(Exch{mz.x, mz.y, tx, 0});
    float gtx = -INFINITY;
    for (int r = 0; r < c.C; ++r) gtx = fmaxf(gtx, got[r].f2);
    const float2 MZ = combine_ranks(got, c.C);
    M = MZ.x;
    Z = MZ.y;
    // rank totals rescaled to the row maximum, for a placement on this row
    // (a separate array: every thread is still reading `got` above)
    if (tid < c.C) rw[tid] = (got[tid].f0 == -INFINITY) ? 0.f : got[tid].f1 * ex2(got[tid].f0 - M);
    __syncthreads();
    if (!(Z > 0.f) || Z == INFINITY || M == -INFINITY || M == INFINITY) {
      badrow = true;
      rejected = (j < L);
      y = 0;
      break;
    }
    if (j == L) {  // every verified draft accepted: bonus token from p of row L
      const float u = uniform24(a.seed, a.round_id, (uint32_t)b, (uint32_t)(acc + 1), kBonus);
      y = c.place(u * Z, M, [&](int i) { return ex2(fmaf(E::to_float(tb[i]), cs, -M)); });
      break;
    }
    const float p = ex2(gtx - M) / Z;
    const float u = uniform24(a.seed, a.round_id, (uint32_t)b, (uint32_t)(j + 1), kAccept);
    if (!(u < p / a.q_tok[(long long)b * K + j])) {
      rejected = true;
      break;
    }
    ++acc;
  }

  if (rejected && !greedy && !badrow) {
    // residual norm(max(0, p - q)) over target row acc (still in shared memory)
    // and draft row acc (q = softmax(d / temp), normaliser recomputed here)
    bulk_load(db, drow0 + (long long)acc * V + c.lo, nbytes, &bar, phase, st, b, &dead);
    const float2 mq = c.online_stats(db, cs);
    c.gather(Exch{mq.x, mq.y, 0.f, 0});
    const float2 MZq = combine_ranks(got, c.C);
    const float Mq = MZq.x, iZ = 1.f / Z, iZq = 1.f / MZq.y;
    auto resid_v = [&](float tv, float dv) {
      const float pp = ex2(fmaf(tv, cs, -M)) * iZ;
      const float qq = ex2(fmaf(dv, cs, -Mq)) * iZq;
      return fmaxf(0.f, pp - qq);
    };
    auto resid = [&](int i) { return resid_v(E::to_float(tb[i]), E::to_float(db[i])); };
    float sr = 0.f;
    c.each2(tb, db, [&](int, float tv, float dv) { sr += resid_v(tv, dv); });
    const float totr = c.block_sum_keep(sr);
    c.gather(Exch{0.f, totr, 0.f, 0});
    float R = 0.f;
    for (int r = 0; r < c.C; ++r) R += got[r].f1;
    if (tid < c.C) rw[tid] = got[tid].f1;
    __syncthreads();
    const float u = uniform24(a.seed, a.round_id, (uint32_t)b, (uint32_t)(acc + 1), kResidual);
    if (R > 0.f) {
      y = c.place(u * R, 0.f, resid);
    } else {
      // exact-zero residual (floating point only): draw from p instead
      const float2 mz = c.online_stats(tb, cs);
      c.gather(Exch{mz.x, mz.y, 0.f, 0});
      if (tid < c.C) rw[tid] = (got[tid].f0 == -INFINITY) ? 0.f : got[tid].f1 * ex2(got[tid].f0 - M);
      __syncthreads();
      y = c.place(u * Z, M, [&](int i) { return ex2(fmaf(E::to_float(tb[i]), cs, -M)); });
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
  // Aim for a few CTAs per SM and row slices of at most ~40 KB, with at most
  // kMaxCluster CTAs per request.
  const long long row_bytes = (long long)V * (dtype == DSPARK_F32 ? 4 : 2);
  int C = 1;
  while (C < kMaxCluster && (row_bytes / C > 40 * 1024 || (long long)B * C < 2LL * num_sms)) C <<= 1;
  return C;
}

size_t verify_smem_bytes(int V, int dtype, int C, int* slice, size_t* slice_padded) {
  const int es = dtype == DSPARK_F32 ? 4 : 2;
  int s = (V + C - 1) / C;
  s = (s + 7) & ~7;
  const size_t sb = ((size_t)s * es + 127) & ~(size_t)127;
  if (slice) *slice = s;
  if (slice_padded) *slice_padded = sb;
  return 2 * sb;
}

cudaError_t verify_launch(VerifyArgs a, int C, cudaStream_t s) {
  size_t padded = 0;
  const size_t sm = verify_smem_bytes(a.V, a.dtype, C, &a.slice, &padded);
  a.slice_bytes_padded = padded;
  auto kern = (a.dtype == DSPARK_F32) ? verify_kernel<DSPARK_F32> : verify_kernel<DSPARK_BF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.B * C));
  cfg.blockDim = dim3(kVThreads);
  cfg.dynamicSmemBytes = sm;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a);
  return e;
}

}  // namespace dspark
