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
__device__ __forceinline__ void cluster_sync() {
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
                          uint32_t& phase, Status* st, int request) {
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
  uint32_t done = 0;
  long long it = 0;
  while (!done) {
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(done)
        : "r"(b), "r"(phase)
        : "memory");
    if (!done && ++it > kSpinLimit) {
      if (threadIdx.x == 0) report(st, DSPARK_STATUS_TIMEOUT, request);
      break;
    }
  }
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
  Exch* got;               // [kMaxCluster] gathered copies
  float* part;             // [kVThreads] per-thread partial sums
  float* excl;             // [kVThreads] their exclusive block scan
  float* red;              // [32] scratch
  int* sint;               // [4] scratch
  int parity;

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
  // f(i, t_value, d_value) over this thread's elements of two buffers
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

  // block max of v (all threads get it)
  __device__ float block_max(float v) {
    v = warp_max(v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float m = red[0];
    for (int w = 1; w < kVThreads / 32; ++w) m = fmaxf(m, red[w]);
    __syncthreads();
    return m;
  }
  __device__ int block_any(int v) {
    v = __any_sync(0xffffffffu, v);
    if (lane == 0) sint[0] = 0;
    __syncthreads();
    if (v && lane == 0) atomicOr(&sint[0], 1);
    __syncthreads();
    const int r = sint[0];
    __syncthreads();
    return r;
  }
  // stores part[tid] = s and excl[tid] = exclusive scan; returns the block total
  __device__ float block_scan_store(float s) {
    const float incl = warp_inclusive_scan(s);
    if (lane == 31) red[warp] = incl;
    __syncthreads();
    float pre = 0.f, tot = 0.f;
    for (int w = 0; w < kVThreads / 32; ++w) {
      if (w < warp) pre += red[w];
      tot += red[w];
    }
    part[tid] = s;
    excl[tid] = pre + incl - s;
    __syncthreads();
    return tot;
  }

  // Inverse-CDF placement of `thr` on weights wfun(i) (slice-local index i)
  // whose per-rank totals are got[r].f1 (rank prefix computed here). Returns
  // the global token index in every thread of the owning CTA, -1 in the other
  // CTAs, and -2 everywhere if no rank holds positive mass. Control flow is
  // uniform inside the CTA; no cluster exchange happens here.
  template <class F>
  __device__ int place(float thr, F wfun) {
    // owner rank: first r with thr < P_r + s_r (positive s_r); else last positive
    int owner = -1, lastpos = -1;
    float P = 0.f, Pown = 0.f;
    for (int r = 0; r < C; ++r) {
      const float s = got[r].f1;
      if (s > 0.f) {
        lastpos = r;
        if (owner < 0 && thr < P + s) {
          owner = r;
          Pown = P;
        }
      }
      P += s;
    }
    bool fallback = false;
    if (owner < 0) {
      owner = lastpos;
      fallback = true;
    }
    if (owner < 0) return -2;
    if (owner != rank) return -1;
    float rem = fallback ? INFINITY : thr - Pown;
    // owner thread: first t with rem < excl_t + part_t
    if (tid == 0) sint[1] = 0x7fffffff;
    __syncthreads();
    if (part[tid] > 0.f && rem < excl[tid] + part[tid]) atomicMin(&sint[1], tid);
    __syncthreads();
    int ot = sint[1];
    bool tfall = fallback;
    if (ot == 0x7fffffff) {  // rounding: last thread with positive mass
      if (tid == 0) sint[2] = -1;
      __syncthreads();
      if (part[tid] > 0.f) atomicMax(&sint[2], tid);
      __syncthreads();
      ot = sint[2];
      tfall = true;
    }
    if (tid == 0) sint[3] = -1;
    __syncthreads();
    if (tid == ot) {
      float r2 = tfall ? INFINITY : rem - excl[tid];
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

template <int DT>
__global__ void __launch_bounds__(kVThreads) verify_kernel(VerifyArgs a) {
  using E = Elem<DT>;
  using T = typename E::T;
  extern __shared__ __align__(128) unsigned char dsm[];
  __shared__ Exch ex[2];
  __shared__ Exch got[kMaxCluster];
  __shared__ float part[kVThreads], excl[kVThreads], red[32];
  __shared__ int sint[4];
  __shared__ __align__(8) uint64_t bar;

  VerifyCta<DT> c;
  c.C = cluster_size();
  c.rank = cluster_rank();
  c.tid = threadIdx.x;
  c.lane = c.tid & 31;
  c.warp = c.tid >> 5;
  c.ex = ex;
  c.got = got;
  c.part = part;
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
  float tau = a.temp[b];
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
  float M = 0.f, Z = 0.f;     // current target row's max (scaled) and sum
  int y = -1;
  Exch rowtot[kMaxCluster];   // per-rank sums of the current target row

  for (int j = 0; j <= L; ++j) {
    bulk_load(tb, target + (long long)j * V + c.lo, nbytes, &bar, phase, st, b);
    const int xk = (j < L) ? a.x[(long long)b * K + j] : -1;
    if (j < L && (xk < 0 || xk >= V) && tid == 0 && c.rank == 0) report(st, DSPARK_STATUS_BAD_TOKEN, b);
    if (greedy) {
      float mv = -INFINITY;
      int mi = 0x7fffffff;
      int bad = 0;
      c.each(tb, [&](int i, float v) {
        bad |= bad_logit(v);
        argmax_merge(mv, mi, v, c.lo + i);
      });
      warp_argmax(mv, mi);
      if (c.lane == 0) {
        red[c.warp] = mv;
        reinterpret_cast<int*>(red)[16 + c.warp] = mi;
      }
      bad = c.block_any(bad);
      float m = red[0];
      int mm = reinterpret_cast<int*>(red)[16];
      for (int w = 1; w < kVThreads / 32; ++w) argmax_merge(m, mm, red[w], reinterpret_cast<int*>(red)[16 + w]);
      __syncthreads();
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

    // pass A: max (scaled), bad flag, and t[x] of the draft being tested
    float mv = -INFINITY;
    int bad = 0;
    c.each(tb, [&](int, float v) {
      bad |= bad_logit(v);
      mv = fmaxf(mv, v);
    });
    mv = c.block_max(mv) * cs;
    bad = c.block_any(bad);
    float tx = -INFINITY;
    if (xk >= c.lo && xk < c.lo + c.n) tx = E::to_float(tb[xk - c.lo]) * cs;
    c.gather(Exch{mv, 0.f, tx, bad});
    M = -INFINITY;
    float gtx = -INFINITY;
    bool gbad = false;
    for (int r = 0; r < c.C; ++r) {
      M = fmaxf(M, got[r].f0);
      gtx = fmaxf(gtx, got[r].f2);
      gbad |= got[r].i0 != 0;
    }
    // pass B: per-thread sums of exp2(z - M) in index order, block scan
    float s = 0.f;
    c.each(tb, [&](int, float v) { s += exp2f(v * cs - M); });
    const float tot = c.block_scan_store(s);
    c.gather(Exch{0.f, tot, 0.f, 0});
    Z = 0.f;
    for (int r = 0; r < c.C; ++r) {
      rowtot[r] = got[r];
      Z += got[r].f1;
    }
    if (gbad || !(Z > 0.f) || Z == INFINITY || M == -INFINITY) {
      badrow = true;
      rejected = (j < L);
      y = 0;
      break;
    }
    if (j == L) {  // every verified draft accepted: bonus token from p of row L
      const float u = uniform24(a.seed, a.round_id, (uint32_t)b, (uint32_t)(acc + 1), kBonus);
      y = c.place(u * Z, [&](int i) { return exp2f(E::to_float(tb[i]) * cs - M); });
      break;
    }
    const float p = exp2f(gtx - M) / Z;
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
    bulk_load(db, drow0 + (long long)acc * V + c.lo, nbytes, &bar, phase, st, b);
    float mq = -INFINITY;
    c.each(db, [&](int, float v) { mq = fmaxf(mq, v); });
    mq = c.block_max(mq) * cs;
    c.gather(Exch{mq, 0.f, 0.f, 0});
    float Mq = -INFINITY;
    for (int r = 0; r < c.C; ++r) Mq = fmaxf(Mq, got[r].f0);
    float sq = 0.f;
    c.each(db, [&](int, float v) { sq += exp2f(v * cs - Mq); });
    const float totq = c.block_scan_store(sq);
    c.gather(Exch{0.f, totq, 0.f, 0});
    float Zq = 0.f;
    for (int r = 0; r < c.C; ++r) Zq += got[r].f1;
    auto resid_v = [&](float tv, float dv) {
      const float p = exp2f(tv * cs - M) / Z;
      const float q = exp2f(dv * cs - Mq) / Zq;
      return fmaxf(0.f, p - q);
    };
    auto resid = [&](int i) { return resid_v(E::to_float(tb[i]), E::to_float(db[i])); };
    float sr = 0.f;
    c.each2(tb, db, [&](int, float tv, float dv) { sr += resid_v(tv, dv); });
    const float totr = c.block_scan_store(sr);
    c.gather(Exch{0.f, totr, 0.f, 0});
    float R = 0.f;
    for (int r = 0; r < c.C; ++r) R += got[r].f1;
    const float u = uniform24(a.seed, a.round_id, (uint32_t)b, (uint32_t)(acc + 1), kResidual);
    if (R > 0.f) {
      y = c.place(u * R, resid);
    } else {
      // exact-zero residual (floating point only): draw from p instead
      float s = 0.f;
      c.each(tb, [&](int, float v) { s += exp2f(v * cs - M); });
      c.block_scan_store(s);
      if (tid < c.C) got[tid] = rowtot[tid];
      __syncthreads();
      y = c.place(u * Z, [&](int i) { return exp2f(E::to_float(tb[i]) * cs - M); });
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
