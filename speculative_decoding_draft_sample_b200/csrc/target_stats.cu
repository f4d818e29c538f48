// Softmax statistics of the target rows that verification reads, in one
// streaming pass that needs nothing from the draft.
//
// "DSpark turns speculation into a scheduler" (intro, "Caveats") and "Fast
// Inference from Transformers via Speculative Decoding" (cited on
// "notes/dspark-deepseek", "Sources"): the test of draft token k needs
// p(x_k) = softmax(t_{k-1} / temp)(x_k), and the token after the accepted
// prefix is drawn from p of the bonus row or from norm(max(0, p - q)). Every
// one of those needs the normaliser of a target row j <= cut[b], and rows past
// the cut are never read. Those normalisers depend only on the target logits
// and the cut, so they are computed here for all rows 0..cut[b] at once, while
// the draft still runs on other SMs, instead of one dependent pass per
// verified position afterwards.
//
// Output: for every request b, row j <= cut[b] and 2 KB chunk c of the row
// (1024 bf16 or 512 fp32 entries), the online-softmax partial
// (max z, sum 2^(z - max z)) of z = t * log2(e) / temp[b], or for a greedy
// request (temp 0) (max t, lowest argmax) with the maximum NaN when the chunk
// holds NaN or +inf.
//
// Design (B200): persistent CTAs, three per SM; one producer warp claims work
// items (request b, 16 KB vocabulary segment s) from a global counter and
// streams segment s of rows 0..cut[b] through a ring of four 16 KB
// shared-memory slots with bulk asynchronous copies (cp.async.bulk, one
// "full" mbarrier per slot completing with the bytes); eight consumer warps
// take one 2 KB chunk of every slot each (128-bit shared loads, one partial
// per warp) and hand the slot back by an arrival on its "empty" mbarrier. An
// item carries cut[b] + 1 rows, so the tail is at most one item. Every wait is
// bounded; a CTA that gives up reports DSPARK_STATUS_TIMEOUT.
#include "common.cuh"
#include "verify.cuh"

namespace dspark {

namespace {

constexpr int kSegBytes = 16384;                        // one ring slot
constexpr int kChunksPerSeg = kSegBytes / kStatChunkBytes;
constexpr int kSlots = 4;
constexpr int kConsumers = kChunksPerSeg;              // one chunk per consumer warp
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kCtasPerSm = 3;

__device__ __forceinline__ uint32_t saddr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

template <int DT>
struct Lanes;
// 16 bytes as floats in index order
template <>
struct Lanes<DSPARK_BF16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const unsigned char* p, float* v) {
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
struct Lanes<DSPARK_F32> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const unsigned char* p, float* v) {
    const float4 q = *reinterpret_cast<const float4*>(p);
    v[0] = q.x;
    v[1] = q.y;
    v[2] = q.z;
    v[3] = q.w;
  }
};

__device__ __forceinline__ float warp_max_nan_all(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = max_nan(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace

// The order in which verification takes the requests: cut descending, index
// ascending (the longest chains of rows first), by one warp: a histogram of
// the clamped cuts, the start of every cut value's range, then every request's
// place, 32 requests at a time (peers with the same cut keep index order).
__device__ void write_order(const StatsArgs& a, int lane, int* cnt) {
  const int K = a.K;
  for (int v = lane; v <= K; v += 32) cnt[v] = 0;
  __syncwarp();
  for (int i = lane; i < a.B; i += 32) atomicAdd(&cnt[min(max(a.cut[i], 0), K)], 1);
  __syncwarp();
  if (lane == 0) {  // cnt[v] becomes the first place of cut value v
    int base = 0;
    for (int v = K; v >= 0; --v) {
      const int c = cnt[v];
      cnt[v] = base;
      base += c;
    }
  }
  __syncwarp();
  const unsigned below = (1u << lane) - 1u;
  for (int i0 = 0; i0 < a.B; i0 += 32) {
    const int i = i0 + lane;
    const int L = (i < a.B) ? min(max(a.cut[i], 0), K) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, L);
    const int rank = __popc(peers & below);
    if (L >= 0) a.order[cnt[L] + rank] = i;
    __syncwarp();
    if (L >= 0 && rank == 0) cnt[L] += __popc(peers);
    __syncwarp();
  }
}

template <int DT>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) target_stats_kernel(StatsArgs a) {
  extern __shared__ __align__(128) unsigned char ring_raw[];
  unsigned char (*ring)[kSegBytes] = reinterpret_cast<unsigned char (*)[kSegBytes]>(ring_raw);
  __shared__ __align__(8) uint64_t full[kSlots];
  __shared__ __align__(8) uint64_t empty[kSlots];
  __shared__ int4 meta[kSlots];  // (request, row, segment, bytes); request < 0 ends the stream
  __shared__ int dead;
  __shared__ int ord_cnt[65];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int es = Elem<DT>::kBytes;
  const long long row_bytes = (long long)a.V * es;
  const int S = (int)((row_bytes + kSegBytes - 1) / kSegBytes);  // segments per row
  const long long items = (long long)a.B * S;

  if (tid == 0) {
    dead = 0;
    for (int i = 0; i < kSlots; ++i) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(&full[i])) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(&empty[i])), "r"(kConsumers)
                   : "memory");
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == kConsumers) {
    // ---------------- producer ----------------
    if (blockIdx.x == 0 && a.cut && a.order) write_order(a, lane, ord_cnt);
    __syncwarp();
    if (lane == 0) {
      const char* target = static_cast<const char*>(a.target);
      uint32_t u = 0;             // units (row segments) issued
      int last[kSlots];           // last unit issued per slot
      for (int i = 0; i < kSlots; ++i) last[i] = -1;
      long long item = atomicAdd(a.next, 1ull);
      bool stop = false;
      while (!stop) {
        int b = -1, s = 0, L = 0;
        if (item < items) {
          b = (int)(item / S);
          s = (int)(item - (long long)b * S);
          L = a.cut ? a.cut[b] : a.K;
          L = L < 0 ? 0 : (L > a.K ? a.K : L);  // a bad cut is reported by verification
        }
        // claim the next item now, so its latency hides behind these copies
        const long long next = (item < items) ? (long long)atomicAdd(a.next, 1ull) : items;
        const int units = (b < 0) ? 1 : L + 1;
        for (int j = 0; j < units; ++j, ++u) {
          const int slot = u % kSlots;
          const uint32_t use = u / kSlots;
          if (use > 0 && (*(volatile int*)&dead ||
                          !mbar_wait_bounded(saddr(&empty[slot]), (use - 1) & 1u))) {
            if (!*(volatile int*)&dead) report_wait(a.status, kWhereStatsEmpty, b < 0 ? 0 : b);
            *(volatile int*)&dead = 1;
            stop = true;
            break;
          }
          if (b < 0) {  // end of the stream: a slot whose phase completes with no bytes
            meta[slot] = make_int4(-1, 0, 0, 0);
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(&full[slot])) : "memory");
            stop = true;
            break;
          }
          const long long off = (long long)s * kSegBytes;
          const int bytes = (int)min((long long)kSegBytes, row_bytes - off);
          meta[slot] = make_int4(b, j, s, bytes);
          const char* src = target + ((long long)b * (a.K + 1) + j) * row_bytes + off;
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(&full[slot])),
                       "r"(bytes)
                       : "memory");
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                  saddr(ring[slot])),
              "l"(src), "r"(bytes), "r"(saddr(&full[slot]))
              : "memory");
          last[slot] = (int)u;
        }
        item = next;
      }
      if (*(volatile int*)&dead)  // let issued copies land before the CTA exits
        for (int i = 0; i < kSlots; ++i)
          if (last[i] >= 0) mbar_wait_bounded(saddr(&full[i]), ((uint32_t)last[i] / kSlots) & 1u);
    }
  } else {
    // ---------------- consumers: warp w takes chunk w of every slot ----------------
    using L = Lanes<DT>;
    constexpr int N = L::N;
    const int nchunk = a.nchunk;
    for (uint32_t u = 0;; ++u) {
      const int slot = u % kSlots;
      if (!mbar_wait_bounded(saddr(&full[slot]), (u / kSlots) & 1u)) {
        if (lane == 0) report_wait(a.status, kWhereStatsFull, 0);
        *(volatile int*)&dead = 1;
        break;
      }
      __syncwarp();
      const int4 m = meta[slot];
      if (m.x < 0) break;
      const int b = m.x, j = m.y, s = m.z, bytes = m.w;
      const int cbyte = warp * kStatChunkBytes;  // this warp's chunk inside the segment
      if (cbyte < bytes) {
        const float tau = a.temp[b];
        const bool greedy = !(tau > 0.f);
        // element index of this lane's first entry of vector q: chunk base +
        // 512 bytes per vector round, 16 bytes per lane
        const long long e0 = ((long long)s * kSegBytes + cbyte) / es;
        float v[4][N];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int boff = cbyte + q * 512 + lane * 16;
          if (boff < bytes) {
            L::load(ring[slot] + boff, v[q]);
          } else {
#pragma unroll
            for (int i = 0; i < N; ++i) v[q][i] = -INFINITY;
          }
        }
        float2 part;
        if (greedy) {
          float mv = -INFINITY, chk = -INFINITY;
          int mi = 0x7fffffff;
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int i = 0; i < N; ++i) {
              const int e = (int)(e0 + (q * 512 + lane * 16) / es + i);
              chk = max_nan(chk, v[q][i]);
              argmax_merge(mv, mi, v[q][i], e);
            }
          warp_argmax(mv, mi);
          chk = warp_max_nan_all(chk);
          const bool bad = chk != chk || chk == INFINITY;
          part = make_float2(bad ? NAN : mv, __int_as_float(mi));
        } else {
          const float cs = kLog2e / tau;
          float mv = -INFINITY;
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int i = 0; i < N; ++i) mv = max_nan(mv, v[q][i]);
          mv = warp_max_nan_all(mv);
          const float mz = mv * cs;
          if (mz != mz) {
            part = make_float2(NAN, NAN);
          } else if (mz == -INFINITY) {
            part = make_float2(-INFINITY, 0.f);  // every entry masked
          } else {
            // +inf makes the sum NaN, which marks the row bad downstream
            const float neg = -mz;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int i = 0; i < N; ++i) acc[i & 3] += ex2(fmaf(v[q][i], cs, neg));
            part = make_float2(mz, warp_sum((acc[0] + acc[1]) + (acc[2] + acc[3])));
          }
        }
        if (lane == 0)
          a.partials[((long long)b * (a.K + 1) + j) * nchunk + s * kChunksPerSeg + warp] = part;
      }
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(&empty[slot])) : "memory");
    }
  }
}

int stats_chunks(int V, int dtype) {
  const long long bytes = (long long)V * (dtype == DSPARK_F32 ? 4 : 2);
  return (int)((bytes + kStatChunkBytes - 1) / kStatChunkBytes);
}

cudaError_t target_stats_launch(const StatsArgs& a, int num_sms, cudaStream_t s) {
  // the work counter starts at zero in every launch
  cudaError_t e = cudaMemsetAsync(a.next, 0, sizeof(unsigned long long), s);
  if (e != cudaSuccess) return e;
  auto kern = (a.dtype == DSPARK_F32) ? target_stats_kernel<DSPARK_F32> : target_stats_kernel<DSPARK_BF16>;
  constexpr int smem = kSlots * kSegBytes;  // the ring (the barriers are static)
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<num_sms * kCtasPerSm, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace dspark
