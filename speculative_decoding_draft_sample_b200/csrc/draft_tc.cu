// Tensor-core (tcgen05) draft-logit kernel for bf16 logits, sm_100a.
//
// Per draft position k this computes, for every request b and vocabulary entry v,
//   d[b, k-1, v] = bf16(base[b, k-1, v] + scale_b * sum_j U[x_{b,k-1}, j] W[j, v])
// ("DSpark turns speculation into a scheduler", "DSpark's semi-autoregressive
// compromise": a low-rank transition bias from the previous sampled token added
// to the parallel drafter's base logits), and each (request, 256-entry chunk)'s
// online-softmax partial (max, sum exp2) of d * log2(e) / temperature, or
// (max, argmax) for greedy requests.
//
// GEMM shape: M = requests (128 per tile), N = vocabulary (256 per tile, as
// two MMA halves of 128), K = Markov rank (<= 256). A = the gathered U rows
// (K-major, built in shared memory once per position), B = W (vocabulary-
// major; stages arrive by TMA with 128-byte swizzle), D = fp32 in tensor
// memory (two 256-column buffers).
//
// Persistent CTAs, one per SM, warp-specialised:
//   warp 0     TMA producer of W tiles (ring of six 16 KB stages of 64 ranks x
//              128 vocabulary entries: a vocabulary half of a tile per four stages)
//   warp 1     TMEM allocator and the single-thread tcgen05.mma issuer (it
//              waits at a named barrier for A, which the epilogue warps gather
//              while the producers already stream W and base)
//   warp 2     TMA producer of base tiles (ring of four 16 KB [128 x 64] blocks)
//              and the TMA store of d from the same slots: a slot is refilled
//              once its store has read it, so the epilogue never waits on a
//              store
//   warps 4-11 epilogue, two halves of four warps (one per TMEM lane
//              quadrant): half h takes column blocks h and h+2 of every tile.
//              tcgen05.ld of the accumulator (lane = request row), + base,
//              round to bf16 (packed), write d back into the staged block and
//              hand it to the producer's store, running (max, sum exp2) per
//              row; the halves merge their row statistics through shared
//              memory at the end of a tile.
// Every wait on an mbarrier is bounded; a CTA that gives up reports
// DSPARK_STATUS_TIMEOUT and winds down instead of hanging.
#include <cuda.h>

#include "draft.cuh"
#include "draft_tc.cuh"
#include "sample_warp.cuh"

namespace dspark {

namespace tc {

constexpr int kThreads = 384;      // 4 role warps + 8 epilogue warps
constexpr int kTileM = 128;
constexpr int kTileN = 256;
constexpr int kWRows = 64;          // Markov ranks per W stage
constexpr int kWCols = 128;         // vocabulary columns per W stage (one MMA half)
constexpr int kWStages = 6;         // W ring depth (stages of 64 ranks x 128 vocab)
constexpr int kWStageBytes = kWRows * kWCols * 2;
constexpr int kWBoxBytes = kWRows * 64 * 2;  // one [64 ranks x 64 vocab] TMA box
constexpr int kBaseSlots = 4;       // base/d ring of [128 x 64] blocks: one tile
constexpr int kBlockBytes = 128 * 64 * 2;
constexpr int kABytes = 128 * 256 * 2;  // gathered U rows, 4 k-blocks of [128 x 64]

// shared-memory layout (offsets from a 1024-byte aligned base)
constexpr int kOffA = 0;
constexpr int kOffW = kOffA + kABytes;
constexpr int kOffBase = kOffW + kWStages * kWStageBytes;
constexpr int kOffBar = kOffBase + kBaseSlots * kBlockBytes;
constexpr int kNumBars = 2 * kWStages + 2 * kBaseSlots + 7;
constexpr int kOffX = kOffBar + kNumBars * 8 + 16;              // [2][128] float2 row stats
constexpr int kSmemBytes = kOffX + 2 * 128 * 8;
static_assert(kSmemBytes <= 232448, "exceeds the 227 KB of shared memory per block");

// instruction descriptor, kind::f16: D fp32, A bf16 K-major, B bf16 MN-major,
// M = 128, N = 128 (a tile's accumulator is two such halves, committed apart,
// so that the epilogue starts on the first half while W of the second arrives)
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                            ((uint32_t)(kWCols >> 3) << 17) | ((uint32_t)(kTileM >> 4) << 24);

__device__ __forceinline__ uint32_t su32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// shared-memory matrix descriptor, 128-byte swizzle, sm100 version bits
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;  // version
  d |= (uint64_t)2 << 61;  // SWIZZLE_128B
  return d;
}

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t par) {
  return mbar_wait_bounded(su32(b), par);
}
// True once the phase of parity `par` has completed (no waiting).
__device__ __forceinline__ bool mbar_test(uint64_t* b, uint32_t par) {
  uint32_t ok;
  asm volatile("{ .reg .pred p; mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
               : "=r"(ok)
               : "r"(su32(b)), "r"(par)
               : "memory");
  return ok != 0;
}

// L2 eviction policies: W is re-read by every draft position (keep it), base
// streams through once per position (let it go first).
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(su32(dst)),
      "l"(map), "r"(su32(bar)), "r"(x), "r"(y), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(su32(dst)),
      "l"(map), "r"(su32(bar)), "r"(x), "r"(y), "r"(z), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y,
                                             int z, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3, %4}], [%1], %5;" ::"l"(
          map),
      "r"(su32(src)), "r"(x), "r"(y), "r"(z), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Named barrier of the eight epilogue warps that also ORs a flag across them,
// so that giving up after a timed-out wait is one decision for all 256 threads.
__device__ __forceinline__ bool epi_bar_any(bool flag) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 3, 256, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)flag)
      : "memory");
  return r != 0;
}

// Two fp32 values rounded to nearest-even bf16, packed (lo in the low half).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// Named barrier 4: the eight epilogue warps arrive once A is in shared memory,
// the MMA warp waits for them.
__device__ __forceinline__ void a_ready_arrive() {
  asm volatile("bar.arrive 4, 288;" ::: "memory");
}
__device__ __forceinline__ void a_ready_sync() {
  asm volatile("bar.sync 4, 288;" ::: "memory");
}
__device__ __forceinline__ void half_bar(int h) {  // the four warps of one epilogue half
  asm volatile("bar.sync %0, 128;" ::"r"(1 + h) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

struct Params {
  const void* U;           // [V, r] bf16
  const int32_t* prev;     // token feeding the bias: last_tok (k = 1) or x[:, k-2]
  int prev_stride;         // element stride between requests in `prev`
  const float* bias_scale;
  const float* temp;
  int B, V, r, k;          // k: 1-based draft position
  int m_tiles, n_tiles;    // tile counts
  int m_first;             // first M-tile of this launch
  int m_per_launch;        // M-tiles covered by this launch
  int ctas_per_m;          // CTAs sharing one M-tile
  float2* partials;        // [B, n_tiles]
  int nchunk;
  Status* status;
  int k_last;              // positions p.k .. k_last in this launch
  int fused;               // 1: sample every position in the kernel (grid barriers)
  unsigned int* gbar;      // grid-barrier counter, zero at launch (fused only)
  DraftArgs da;            // the draft call (sampling, next position's tokens)
};



__global__ void __launch_bounds__(kThreads, 1)
    draft_logits_tc(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_base,
                    const __grid_constant__ CUtensorMap map_d, Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 128-byte-swizzled TMA tiles and MMA operands need 1024-byte alignment
  if (su32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) report(p.status, DSPARK_STATUS_INTERNAL, 0);
    return;
  }
  unsigned char* smem = smem_raw;
  unsigned char* sA = smem + kOffA;
  unsigned char* sW = smem + kOffW;
  unsigned char* sBase = smem + kOffBase;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* w_full = bars;
  uint64_t* w_empty = bars + kWStages;
  uint64_t* b_full = bars + 2 * kWStages;
  uint64_t* t_full = b_full + kBaseSlots;    // [2 buffers][2 halves]
  uint64_t* t_empty = t_full + 4;            // [2]
  uint64_t* d_full = t_empty + 2;            // [kBaseSlots] the block's d is written
  uint64_t* d_done = d_full + kBaseSlots;    // the position's d stores are complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float2* xstat = reinterpret_cast<float2*>(smem + kOffX);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mt_local = blockIdx.x % p.m_per_launch;
  const int mt = p.m_first + mt_local;
  const int m0 = mt * kTileM;
  const int nt0 = blockIdx.x / p.m_per_launch;
  const int nstride = p.ctas_per_m;
  const int n_my = (nt0 < p.n_tiles) ? (p.n_tiles - nt0 + nstride - 1) / nstride : 0;
  const int kbh = (p.r + kWRows - 1) / kWRows;  // W stages per MMA half
  const int kblocks = 2 * kbh;                   // W stages per tile
  const int npos = p.k_last - p.k + 1;  // draft positions in this launch
  const int ksteps = p.r / 16;           // MMAs per tile

  if (tid == 0) {
    for (int i = 0; i < kWStages; ++i) {
      mbar_init(&w_full[i], 1);
      mbar_init(&w_empty[i], 1);
    }
    for (int i = 0; i < kBaseSlots; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&d_full[i], 1);
    }
    mbar_init(d_done, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&t_full[i], 1);
    for (int i = 0; i < 2; ++i) mbar_init(&t_empty[i], 256);
    // w_full, w_empty, b_full, t_full (4), t_empty (2), d_full, d_done
    static_assert(2 * kWStages + 2 * kBaseSlots + 7 == kNumBars, "barrier count");
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // 512 TMEM columns: two 256-column fp32 accumulators
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     su32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }

  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- W producer ----------------
    const uint64_t pol_w = policy_evict_last();
    int it = 0;
    int last[kWStages];
    for (int q = 0; q < kWStages; ++q) last[q] = -1;
    for (int t = 0; t < n_my * npos; ++t) {  // W is the same at every position
      const int n0 = (nt0 + (t % n_my) * nstride) * kTileN;
      bool stop = false;
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int s = it % kWStages;
        if (*(volatile int*)abort_flag || !mbar_wait(&w_empty[s], ((it / kWStages) & 1) ^ 1)) {
          if (!*(volatile int*)abort_flag) report_wait(p.status, kWhereTcWEmpty, m0);
          *(volatile int*)abort_flag = 1;
          stop = true;
          break;
        }
        mbar_expect_tx(&w_full[s], kWStageBytes);
        unsigned char* dst = sW + s * kWStageBytes;
        // stage kb: ranks (kb % kbh) * 64 .. + 63 of vocabulary half kb / kbh
#pragma unroll
        for (int vb = 0; vb < 2; ++vb)
          tma_load_2d(dst + vb * kWBoxBytes, &map_w, n0 + (kb / kbh) * kWCols + vb * 64,
                      (kb % kbh) * kWRows, &w_full[s], pol_w);
        last[s] = it;
      }
      if (stop) break;
    }
    if (*(volatile int*)abort_flag)  // let issued loads land before the CTA winds down
      for (int q = 0; q < kWStages; ++q)
        if (last[q] >= 0) mbar_wait(&w_full[q], (last[q] / kWStages) & 1);
  } else if (warp == 2 && lane == 0) {
    // ---------------- base producer and d stores ----------------
    // block j of tile t (counted over all positions) is block g = 4t + j of
    // the ring (slot g % kBaseSlots). The epilogue writes a block's d back
    // into its slot and arrives on d_full; this thread stores it (in block
    // order) and refills the slot once the store has read it.
    const uint64_t pol_base = policy_evict_first();
    // d keeps the normal L2 priority: the sampler re-reads a chunk of every row
    const uint64_t pol_d = policy_evict_normal();
    const int total = 4 * n_my * npos;
    int last[kBaseSlots];
    for (int q = 0; q < kBaseSlots; ++q) last[q] = -1;
    int next_store = 0;
    // 1: block gsb's store issued; 0: its d is not written yet (no wait); -1: gave up
    auto store_block = [&](int gsb, bool wait) -> int {
      const int s2 = gsb % kBaseSlots;
      const uint32_t par = (gsb / kBaseSlots) & 1;
      if (wait) {
        if (!mbar_wait(&d_full[s2], par)) return -1;
      } else if (!mbar_test(&d_full[s2], par)) {
        return 0;
      }
      const int t = gsb >> 2;
      const int n0 = (nt0 + (t % n_my) * nstride) * kTileN;
      const int kpos = p.k + t / n_my;
      tma_store_3d(&map_d, sBase + s2 * kBlockBytes, n0 + (gsb & 3) * 64, kpos - 1, m0, pol_d);
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      if (p.fused && (gsb + 1) % (4 * n_my) == 0) {
        // the position's last block: its d must be in global memory before
        // the grid barrier, where the sampler starts reading it
        asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
        asm volatile("fence.proxy.async.global;" ::: "memory");
        mbar_arrive(d_done);
      }
      return 1;
    };
    bool gave_up = false;
    for (int g = 0; g < total && !gave_up; ++g) {
      const int s = g % kBaseSlots;
      if (*(volatile int*)abort_flag) break;
      if (g >= kBaseSlots) {
        // the slot's previous block (g - kBaseSlots) must be stored and read
        while (next_store <= g - kBaseSlots) {
          if (store_block(next_store, true) < 0) {
            gave_up = true;
            break;
          }
          ++next_store;
        }
        if (gave_up) break;
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      }
      const int t = g >> 2;
      const int n0 = (nt0 + (t % n_my) * nstride) * kTileN;
      const int kpos = p.k + t / n_my;
      mbar_expect_tx(&b_full[s], kBlockBytes);
      tma_load_3d(sBase + s * kBlockBytes, &map_base, n0 + (g & 3) * 64, kpos - 1, m0, &b_full[s], pol_base);
      last[s] = g;
      // blocks whose d is already written go out now
      while (next_store < g && store_block(next_store, false) == 1) ++next_store;
    }
    while (!gave_up && next_store < total && !*(volatile int*)abort_flag) {
      if (store_block(next_store, true) < 0) gave_up = true;
      else ++next_store;
    }
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    if (gave_up) {
      if (!*(volatile int*)abort_flag) report_wait(p.status, kWhereTcDStore, m0);
      *(volatile int*)abort_flag = 1;
    }
    if (*(volatile int*)abort_flag)  // let issued loads land before the CTA winds down
      for (int q = 0; q < kBaseSlots; ++q)
        if (last[q] >= 0) mbar_wait(&b_full[q], (last[q] / kBaseSlots) & 1);
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // A is gathered by the epilogue warps meanwhile (the producers are already
    // streaming W and base); the whole warp waits for it at the named barrier
    int it = 0;
    int last_it = -1;  // last W stage whose MMAs were committed
    const uint32_t a_base = su32(sA);
    for (int kp = 0; kp < npos; ++kp) {
    a_ready_sync();  // A of this position is in shared memory
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (__shfl_sync(0xffffffffu, *(volatile int*)abort_flag, 0)) break;
    if (lane == 0) {
    for (int i = 0; i < n_my; ++i) {
      const int ti = kp * n_my + i;  // tile counted over all positions
      const int buf = ti & 1;
      if (*(volatile int*)abort_flag || !mbar_wait(&t_empty[buf], ((ti >> 1) & 1) ^ 1)) {
        if (!*(volatile int*)abort_flag) report_wait(p.status, kWhereTcAccEmpty, m0);
        *(volatile int*)abort_flag = 1;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      bool ok = true;
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int hh = kb / kbh, rb = kb % kbh;  // vocabulary half, rank block
        const uint32_t d_tmem = tmem + buf * kTileN + hh * kWCols;
        const int s = it % kWStages;
        if (!mbar_wait(&w_full[s], (it / kWStages) & 1)) {
          report_wait(p.status, kWhereTcWFull, m0);
          ok = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t w_base = su32(sW + s * kWStageBytes);
#pragma unroll
        for (int kk = 0; kk < kWRows / 16; ++kk) {
          const int step = rb * (kWRows / 16) + kk;  // 16 ranks per MMA
          if (step < ksteps) {
            // A: 64-rank sub-tile rb, 32-byte step kk inside its 128-byte swizzle row
            const uint64_t ad = sdesc(a_base + rb * 16384 + kk * 32, 16, 1024);
            // B: 16 k-rows (2 groups of 8) per step; the two 64-vocab boxes kWBoxBytes apart
            const uint64_t bd = sdesc(w_base + kk * 2048, kWBoxBytes, 1024);
            const uint32_t acc = (step > 0) ? 1u : 0u;
            asm volatile(
                "{\n .reg .pred pa;\n setp.ne.b32 pa, %4, 0;\n"
                " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, pa;\n}" ::"r"(d_tmem),
                "l"(ad), "l"(bd), "r"(kIdesc), "r"(acc)
                : "memory");
          }
        }
        asm volatile(
            "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                su32(&w_empty[s]))
            : "memory");
        last_it = it;
        if (rb == kbh - 1)  // this half of the accumulator is complete
          asm volatile(
              "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                  su32(&t_full[2 * buf + hh]))
              : "memory");
      }
      if (!ok) {
        *(volatile int*)abort_flag = 1;
        break;
      }
    }
    }
    __syncwarp();
    }
    // MMAs complete in order: once the last commit has landed, tensor memory is quiet
    if (lane == 0 && *(volatile int*)abort_flag && last_it >= 0)
      mbar_wait(&w_empty[last_it % kWStages], (last_it / kWStages) & 1);
  } else if (warp >= 4) {
    // ---------------- A gather, then the epilogue ----------------
    // A = U[prev_b, :] for the 128 rows of this M-tile, 128-byte swizzled,
    // K-major: k-block kb (64 ranks) at kb * 16 KB, row m at m * 128 B, 16-byte
    // chunk c at (c ^ (m & 7)) * 16 B. Rows past B and ranks past r are zero.
    // Epilogue warp e gathers rows 16e .. 16e + 15: lanes 0-15 read the rows'
    // tokens, then every lane loads one 16-byte chunk of each of the 16 rows
    // (all loads in flight at once; a row is one 512-byte coalesced read).
    // Position kq's rows come from U by token, or (recurrent head, kq >= 2)
    // from the states the draw left in H; the first states h_1 = U[x_0] are
    // written out by the M-tile's first CTA.
    auto gather_a = [&](const int32_t* prev, int prev_stride, int kq) {
      const int ew = warp - 4;
      int tokv = 0;
      if (lane < 16) {
        const int b = m0 + ew * 16 + lane;
        if (b < p.B) tokv = prev[(long long)b * prev_stride];
        if (tokv < 0 || tokv >= p.V) tokv = 0;  // reported by the sampler
      }
      uint4 v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int tok = __shfl_sync(0xffffffffu, tokv, i);
        const int bq = m0 + ew * 16 + i;
        v[i] = make_uint4(0, 0, 0, 0);
        if (bq < p.B && lane * 8 < p.r)
          v[i] = *reinterpret_cast<const uint4*>(a_row<uint16_t>(p.da, bq, kq, tok) + lane * 8);
      }
      if (p.da.R && kq == 1 && nt0 == 0) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int bq = m0 + ew * 16 + i;
          if (bq < p.B && lane * 8 < p.r)
            *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.da.H) + (long long)bq * p.da.K * p.r + lane * 8) = v[i];
        }
      }
      const int kb = lane >> 3, c = lane & 7;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int m = ew * 16 + i;
        *reinterpret_cast<uint4*>(sA + kb * 16384 + m * 128 + ((c ^ (m & 7)) << 4)) = v[i];
      }
      fence_async_smem();
    };
    // The recurrent head's next states h_{kq+1} of the rows this CTA drew at
    // position kq (rows blockIdx.x + j * gridDim.x, j = 0, 1, ..., four at a
    // time), by its 256 epilogue threads (thread t: output t): R goes
    // through the A buffer, which holds nothing between the position's last
    // MMA and the next gather, in halves of 128 rows; up to four drawn rows'
    // states h_kq at a time sit in the row-statistics buffer. The sums run in
    // ascending j with one fused multiply-add per term, as in rnn_step, so the
    // states are those of the per-position path bit for bit.
    auto rnn_cta = [&](int kq) {
      const int et = tid - 128;  // epilogue thread 0..255
      const int r = p.r;
      const int K = p.da.K;
      const uint16_t* Rm = static_cast<const uint16_t*>(p.da.R);
      const uint16_t* Um = static_cast<const uint16_t*>(p.da.U);
      uint16_t* Hm = static_cast<uint16_t*>(p.da.H);
      uint16_t* sR = reinterpret_cast<uint16_t*>(sA);      // [128][r]
      uint16_t* sh = reinterpret_cast<uint16_t*>(xstat);   // [4][256]
      // the trip count depends only on the grid and B: every epilogue thread
      // takes the same named barriers
      for (int w0 = 0; blockIdx.x + (long long)w0 * gridDim.x < p.B; w0 += 4) {
        int rows[4];
        int nr = 0;
        for (int g = 0; g < 4; ++g) {
          const long long rr = blockIdx.x + (long long)(w0 + g) * gridDim.x;
          rows[g] = rr < p.B ? (int)rr : -1;
          if (rr < p.B) ++nr;
        }
        if (nr == 0) break;
        epi_bar_any(false);  // the statistics buffer and the A buffer are free
        for (int i = et; i < 4 * r; i += 256) {
          const int g = i / r, j = i - g * r;
          sh[g * 256 + j] = rows[g] >= 0 ? Hm[((long long)rows[g] * K + (kq - 1)) * r + j] : (uint16_t)0;
        }
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int j0 = 0; j0 < r; j0 += 128) {
          const int jn = min(128, r - j0);
          epi_bar_any(false);
          for (int v = et; v < jn * r / 8; v += 256)  // 16-byte pieces of R rows j0 .. j0 + jn - 1
            reinterpret_cast<uint4*>(sR)[v] = reinterpret_cast<const uint4*>(Rm + (long long)j0 * r)[v];
          epi_bar_any(false);
          if (et < r) {
            for (int j = 0; j < jn; ++j) {
              const float rv = bf16_bits_to_float(sR[j * r + et]);
#pragma unroll
              for (int g = 0; g < 4; ++g) acc[g] = fmaf(bf16_bits_to_float(sh[g * 256 + j0 + j]), rv, acc[g]);
            }
          }
        }
        if (et < r) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            if (rows[g] < 0) continue;
            int tok = p.da.x[(long long)rows[g] * K + (kq - 1)];
            if (tok < 0 || tok >= p.V) tok = 0;  // reported by the draw
            const float u = bf16_bits_to_float(Um[(long long)tok * r + et]);
            Hm[((long long)rows[g] * K + kq) * r + et] =
                __bfloat16_as_ushort(__float2bfloat16_rn(u + tanhf(acc[g])));
          }
        }
      }
      epi_bar_any(false);  // A is free for the gather
    };
    gather_a(p.prev, p.prev_stride, p.k);
    a_ready_arrive();
    // ---------------- epilogue ----------------
    const int q = warp & 3;             // TMEM lane quadrant
    const int h = (warp - 4) >> 2;      // half: column blocks h and h + 2
    const int row = q * 32 + lane;      // request row inside the tile
    const int b = m0 + row;
    const bool valid = b < p.B;
    const float tau = valid ? p.temp[b] : 1.f;
    const bool greedy = !(tau > 0.f);
    const float cs = greedy ? 1.f : kLog2e / tau;
    const float sc = (valid && p.bias_scale) ? p.bias_scale[b] : 1.f;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const bool elected = (warp == 4 + 4 * h) && lane == 0;
    bool miss = false;
    bool aborted = false;
    const bool leader = warp == 4 && lane == 0;
    unsigned int nbar = 0;  // grid barriers passed
    for (int kp = 0; kp < npos && !aborted; ++kp) {
    const int kpos = p.k + kp;  // 1-based draft position
    for (int i = 0; i < n_my; ++i) {
      const int ti = kp * n_my + i;  // tile counted over all positions
      const int nt = nt0 + i * nstride;
      const int n0 = nt * kTileN;
      const int buf = ti & 1;
      // sampled rows: running max of z = d * cs and sum of 2^(z - max)
      // greedy rows: running (max d, argmax), NaN-propagating check value
      float run_m = -INFINITY, run_s = 0.f, chk = -INFINITY;
      int arg = 0x7fffffff;
#pragma unroll 1
      for (int jj = 0; jj < 2; ++jj) {
        const int j = h + 2 * jj;       // column block of the tile
        const int g = 4 * ti + j;       // block of the ring
        const int slot = g % kBaseSlots;
        if (!mbar_wait(&b_full[slot], (g / kBaseSlots) & 1)) {
          miss = true;
          report_wait(p.status, kWhereTcBaseFull, m0);
        }
        // column block j lies in MMA half jj: wait for that half's commit
        if (!mbar_wait(&t_full[2 * buf + jj], (ti >> 1) & 1)) {
          miss = true;
          report_wait(p.status, kWhereTcAccFull, m0);
        }
        __syncwarp();  // tcgen05.ld is warp-aligned: every lane, together
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        float acc[64];
        const uint32_t col = tmem + lane_base + buf * kTileN + j * 64;
        tmem_ld32(col, acc);
        tmem_ld32(col + 32, acc + 32);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        unsigned char* blk = sBase + slot * kBlockBytes + row * 128;
        uint32_t dp[32];                // the block's 64 stored logits, packed
        // d = round(base + sc * acc); the running maximum is taken on the
        // unrounded sums: rounding to nearest is monotonic, so the rounded
        // maximum is the maximum of the stored values (NaN propagates)
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4* ptr = reinterpret_cast<uint4*>(blk + ((c ^ (row & 7)) << 4));
          const uint4 v = *ptr;
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float y0 = fmaf(sc, acc[c * 8 + 2 * e], __uint_as_float(w[e] << 16));
            const float y1 = fmaf(sc, acc[c * 8 + 2 * e + 1], __uint_as_float(w[e] & 0xffff0000u));
            dp[c * 4 + e] = pack_bf16x2(y0, y1);
            mx[e] = max_nan(mx[e], max_nan(y0, y1));
          }
          *ptr = make_uint4(dp[c * 4], dp[c * 4 + 1], dp[c * 4 + 2], dp[c * 4 + 3]);
        }
        const int vcols = min(64, p.V - (n0 + j * 64));
        if (valid && vcols > 0) {
          if (greedy) {
#pragma unroll
            for (int e = 0; e < 64; ++e) {
              const float dv = __uint_as_float((e & 1) ? (dp[e >> 1] & 0xffff0000u) : (dp[e >> 1] << 16));
              if (vcols == 64 || e < vcols) {
                chk = max_nan(chk, dv);
                if (dv > run_m) {
                  run_m = dv;
                  arg = n0 + j * 64 + e;
                }
              }
            }
          } else {
            float bm;
            if (vcols == 64) {
              const float m4 = max_nan(max_nan(mx[0], mx[1]), max_nan(mx[2], mx[3]));
              bm = __uint_as_float(pack_bf16x2(m4, 0.f) << 16);  // = max of the stored values
            } else {  // ragged last block: only the columns inside the vocabulary
              bm = -INFINITY;
#pragma unroll
              for (int e = 0; e < 64; ++e)
                if (e < vcols)
                  bm = max_nan(bm, __uint_as_float((e & 1) ? (dp[e >> 1] & 0xffff0000u) : (dp[e >> 1] << 16)));
            }
            if (bm != bm) {
              run_s = NAN;  // a NaN logit: the chunk partial reports it
            } else {
              const float nm = fmaxf(run_m, bm * cs);
              if (nm != -INFINITY) {  // -inf entries weigh nothing; +inf makes the sum NaN
                const float neg = -nm;
                float sacc[4] = {0.f, 0.f, 0.f, 0.f};
                if (vcols == 64) {
#pragma unroll
                  for (int q2 = 0; q2 < 32; ++q2) {
                    sacc[q2 & 3] += ex2(fmaf(__uint_as_float(dp[q2] << 16), cs, neg)) +
                                    ex2(fmaf(__uint_as_float(dp[q2] & 0xffff0000u), cs, neg));
                  }
                } else {
#pragma unroll
                  for (int e = 0; e < 64; ++e)
                    if (e < vcols)
                      sacc[e & 3] += ex2(fmaf(__uint_as_float((e & 1) ? (dp[e >> 1] & 0xffff0000u)
                                                                      : (dp[e >> 1] << 16)),
                                              cs, neg));
                }
                const float acc_s = (sacc[0] + sacc[1]) + (sacc[2] + sacc[3]);
                run_s = (run_m == -INFINITY ? 0.f : run_s * ex2(run_m - nm)) + acc_s;
              }
              run_m = nm;
            }
          }
        }
        fence_async_smem();
        __syncwarp();
        half_bar(h);  // the half's four warps have written the block
        if (elected) mbar_arrive(&d_full[slot]);
        __syncwarp();
      }
      // this thread is done reading accumulator buffer `buf`
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      mbar_arrive(&t_empty[buf]);
      // merge the two halves' statistics of this row
      float2* xs = xstat + (ti & 1) * 128;
      if (h == 1) {
        // greedy rows fold the NaN / +inf check into the max
        const bool bad_g = greedy && (chk != chk || chk == INFINITY);
        xs[row] = greedy ? make_float2(bad_g ? NAN : run_m, __int_as_float(arg))
                         : make_float2(run_m, run_s);
      }
      __syncwarp();
      if (epi_bar_any(miss)) {  // a wait gave up somewhere: every epilogue thread stops here
        *(volatile int*)abort_flag = 1;
        aborted = true;
        break;
      }
      if (h == 0 && valid) {
        const float2 o = xs[row];
        float2 part;
        if (greedy) {
          float m = run_m;
          int a = arg;
          argmax_merge(m, a, o.x, __float_as_int(o.y));
          const bool bad = chk != chk || chk == INFINITY || o.x != o.x;
          part.x = bad ? NAN : m;
          part.y = __int_as_float(a);
        } else {
          const float m = fmaxf(run_m, o.x);
          const float s0 = run_m == -INFINITY ? 0.f : run_s * ex2(run_m - m);
          const float s1 = o.x == -INFINITY ? 0.f : o.y * ex2(o.x - m);
          part.x = m;
          part.y = s0 + s1;  // NaN propagates; a chunk all at -inf is (-inf, 0)
        }
        p.partials[(long long)b * p.nchunk + nt] = part;
      }
    }
    if (!aborted && p.fused) {
      // this position's d is complete in global memory (the sampler reads it)
      // (d_done completes once per position, so this wait is never two phases
      // behind; a CTA without tiles stores nothing and skips it)
      bool fail = leader && n_my > 0 && !mbar_wait(d_done, kp & 1);
      if (fail) report_wait(p.status, kWhereTcDStore, m0);
      __syncwarp();
      aborted = epi_bar_any(fail);
      // every CTA's partials and d of this position -> sample -> every token
      if (!aborted) {
        fail = leader && !grid_arrive_wait(p.gbar, (++nbar) * gridDim.x);
        if (fail) report_wait(p.status, kWhereTcGrid, m0);
        aborted = epi_bar_any(fail);
      }
      if (!aborted) {
        for (int rr = blockIdx.x + (warp - 4) * gridDim.x; rr < p.B; rr += 8 * gridDim.x)
          sample_row_warp<DSPARK_BF16>(p.da, rr, kpos);
        if (p.da.R && kpos < p.da.K) rnn_cta(kpos);
        if (kp + 1 < npos) {
          epi_bar_any(false);
          fail = leader && !grid_arrive_wait(p.gbar, (++nbar) * gridDim.x);
          if (fail) report_wait(p.status, kWhereTcGrid, m0);
          aborted = epi_bar_any(fail);
        }
      }
      if (aborted) *(volatile int*)abort_flag = 1;
    }
    if (kp + 1 < npos) {
      // A of the next position from this position's tokens; on a failure the
      // MMA warp still gets its arrival (it then sees the abort flag)
      if (!aborted) gather_a(p.da.x + kpos - 1, p.da.K, kpos + 1);
      a_ready_arrive();
    }
    }
  }

  __syncwarp();  // role lanes rejoin their warps before the block barrier
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ---------------------------------------------------------------------------
// host side: tensor maps through the driver entry point, launch geometry
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

static bool make_map(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims,
                     const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

bool draft_tc_supported(const DraftArgs& a) {
  return a.dtype == DSPARK_BF16 && a.r % 16 == 0 && a.r <= 256 && tc::encode_fn() != nullptr;
}

// Tensor maps and the fields of Params that every launch shares.
static cudaError_t tc_setup(const DraftArgs& a, CUtensorMap* mw, CUtensorMap* mb, CUtensorMap* md,
                            tc::Params* pp) {
  using namespace tc;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)a.V, (cuuint64_t)a.r};
    const cuuint64_t strides[1] = {(cuuint64_t)a.V * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kWRows};
    if (!make_map(mw, a.W, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {(cuuint64_t)a.V, (cuuint64_t)a.K, (cuuint64_t)a.B};
    const cuuint64_t strides[2] = {(cuuint64_t)a.V * 2, (cuuint64_t)a.V * a.K * 2};
    const cuuint32_t box[3] = {64, 1, 128};
    if (!make_map(mb, a.base, 3, dims, strides, box)) return cudaErrorInvalidValue;
    if (!make_map(md, a.d, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(draft_logits_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e != cudaSuccess) return e;
  Params& p = *pp;
  p.U = a.U;
  p.bias_scale = a.bias_scale;
  p.temp = a.temp;
  p.B = a.B;
  p.V = a.V;
  p.r = a.r;
  p.m_tiles = (a.B + kTileM - 1) / kTileM;
  p.n_tiles = (a.V + kTileN - 1) / kTileN;
  p.partials = a.partials;
  p.nchunk = a.nchunk;
  p.status = a.status;
  p.fused = 0;
  p.gbar = nullptr;
  p.da = a;
  return cudaSuccess;
}

cudaError_t draft_logits_tc_launch(const DraftArgs& a, int k, int num_sms, cudaStream_t s) {
  using namespace tc;
  CUtensorMap mw, mb, md;
  Params p;
  cudaError_t e = tc_setup(a, &mw, &mb, &md, &p);
  if (e != cudaSuccess) return e;
  p.prev = (k == 1) ? a.last_tok : a.x + (k - 2);
  p.prev_stride = (k == 1) ? 1 : a.K;
  p.k = k;
  p.k_last = k;
  // launches of at most num_sms CTAs; each CTA keeps one M-tile (its A operand)
  for (int mf = 0; mf < p.m_tiles;) {
    const int m_here = min(p.m_tiles - mf, num_sms);
    const int per_m = max(1, num_sms / m_here);
    p.m_first = mf;
    p.m_per_launch = m_here;
    p.ctas_per_m = per_m;
    draft_logits_tc<<<m_here * per_m, kThreads, kSmemBytes, s>>>(mw, mb, md, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    mf += m_here;
  }
  return cudaSuccess;
}

bool draft_round_tc_supported(const DraftArgs& a, int num_sms) {
  return draft_tc_supported(a) && (a.B + tc::kTileM - 1) / tc::kTileM <= num_sms - kDraftFreeSms;
}

cudaError_t draft_round_tc_launch(const DraftArgs& a, int num_sms, int free_sms, cudaStream_t s) {
  using namespace tc;
  CUtensorMap mw, mb, md;
  Params p;
  cudaError_t e = tc_setup(a, &mw, &mb, &md, &p);
  if (e != cudaSuccess) return e;
  if (p.m_tiles > num_sms) return cudaErrorInvalidValue;
  p.prev = a.last_tok;
  p.prev_stride = 1;
  p.k = 1;
  p.k_last = a.K;
  p.fused = 1;
  // the grid-barrier counter lives in the unused tail of the status block
  p.gbar = reinterpret_cast<unsigned int*>(reinterpret_cast<char*>(a.status) + kGridBarrierOffset);
  e = cudaMemsetAsync(p.gbar, 0, sizeof(unsigned int), s);
  if (e != cudaSuccess) return e;
  // free_sms SMs stay free for work on other streams (the prefix schedule and
  // the target rows' statistics need none of the draft's outputs and run there
  // at the same time); every M-tile keeps at least one CTA
  const int free_eff = min(max(free_sms, 0), num_sms - p.m_tiles);
  const int per_m = max(1, (num_sms - free_eff) / p.m_tiles);
  p.m_first = 0;
  p.m_per_launch = p.m_tiles;
  p.ctas_per_m = per_m;
  // cooperative: every CTA is resident at once (one per SM), or the launch fails
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.m_tiles * per_m));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, draft_logits_tc, mw, mb, md, p);
}

}  // namespace dspark
