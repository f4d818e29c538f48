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
// GEMM shape: M = requests (128 per tile), N = vocabulary (256 per tile),
// K = Markov rank (<= 256). A = the gathered U rows (K-major, built in shared
// memory once per CTA), B = W (vocabulary-major; tiles arrive by TMA with
// 128-byte swizzle), D = fp32 in tensor memory (two 256-column buffers).
//
// Persistent CTAs, one per SM, warp-specialised:
//   warp 0     TMA producer of W tiles (4-stage-per-tile ring of 32 KB stages)
//   warp 1     TMEM allocator and the single-thread tcgen05.mma issuer
//   warp 2     TMA producer of base tiles (ring of 16 KB [128 x 64] blocks)
//   warps 4-7  epilogue: tcgen05.ld of the accumulator (lane = request row),
//              + base, round to bf16, write d back into the staged block, TMA
//              store of d, running (max, sum) per row.
// Every wait on an mbarrier is bounded; a CTA that gives up reports
// DSPARK_STATUS_TIMEOUT and winds down instead of hanging.
#include <cuda.h>

#include "draft.cuh"
#include "draft_tc.cuh"

namespace dspark {

namespace tc {

constexpr int kThreads = 256;
constexpr int kTileM = 128;
constexpr int kTileN = 256;
constexpr int kWStages = 3;         // W ring depth (stages of 64 k-rows x 256 vocab)
constexpr int kWStageBytes = 64 * 256 * 2;
constexpr int kBaseSlots = 4;       // base/d ring depth ([128 x 64] blocks)
constexpr int kBlockBytes = 128 * 64 * 2;
constexpr int kABytes = 128 * 256 * 2;  // gathered U rows, 4 k-blocks of [128 x 64]

// shared-memory layout (offsets from a 1024-byte aligned base)
constexpr int kOffA = 0;
constexpr int kOffW = kOffA + kABytes;
constexpr int kOffBase = kOffW + kWStages * kWStageBytes;
constexpr int kOffBar = kOffBase + kBaseSlots * kBlockBytes;
constexpr int kNumBars = 2 * kWStages + 2 * kBaseSlots + 4;
constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;  // + tmem slot + alignment slack

// instruction descriptor, kind::f16: D fp32, A bf16 K-major, B bf16 MN-major,
// M = 128, N = 256
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                            ((uint32_t)(kTileN >> 3) << 17) | ((uint32_t)(kTileM >> 4) << 24);

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
// Bounded wait for the phase of parity `par`; false when it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t par) {
  const uint32_t a = su32(b);
  for (long long it = 0; it < kSpinLimit; ++it) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(a), "r"(par)
        : "memory");
    if (ok) return true;
  }
  return false;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          su32(dst)),
      "l"(map), "r"(su32(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          su32(dst)),
      "l"(map), "r"(su32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y,
                                             int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   map),
               "r"(su32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Named barrier of the four epilogue warps that also ORs a flag across them,
// so that giving up after a timed-out wait is one decision for all 128 threads.
__device__ __forceinline__ bool epi_bar_any(bool flag) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, 128, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)flag)
      : "memory");
  return r != 0;
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
};

__global__ void __launch_bounds__(kThreads, 1)
    draft_logits_tc(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_base,
                    const __grid_constant__ CUtensorMap map_d, Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* sA = smem + kOffA;
  unsigned char* sW = smem + kOffW;
  unsigned char* sBase = smem + kOffBase;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* w_full = bars;
  uint64_t* w_empty = bars + kWStages;
  uint64_t* b_full = bars + 2 * kWStages;
  uint64_t* b_empty = b_full + kBaseSlots;
  uint64_t* t_full = b_empty + kBaseSlots;   // [2]
  uint64_t* t_empty = t_full + 2;            // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mt_local = blockIdx.x % p.m_per_launch;
  const int mt = p.m_first + mt_local;
  const int m0 = mt * kTileM;
  const int nt0 = blockIdx.x / p.m_per_launch;
  const int nstride = p.ctas_per_m;
  const int n_my = (nt0 < p.n_tiles) ? (p.n_tiles - nt0 + nstride - 1) / nstride : 0;
  const int kblocks = (p.r + 63) / 64;   // W stages per tile
  const int ksteps = p.r / 16;           // MMAs per tile

  if (tid == 0) {
    for (int i = 0; i < kWStages; ++i) {
      mbar_init(&w_full[i], 1);
      mbar_init(&w_empty[i], 1);
    }
    for (int i = 0; i < kBaseSlots; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&t_full[i], 1);
      mbar_init(&t_empty[i], 128);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // 512 TMEM columns: two 256-column fp32 accumulators
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     su32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }

  // A = U[prev_b, :] for the 128 rows of this M-tile, 128-byte swizzled, K-major:
  // k-block kb (64 ranks) at kb * 16 KB, row m at m * 128 B, 16-byte chunk c at
  // (c ^ (m & 7)) * 16 B. Rows past B and ranks past r are zero.
  {
    const uint16_t* U = static_cast<const uint16_t*>(p.U);
    const int chunks_per_row = 32;  // 256 ranks / 8
    for (int e = tid; e < kTileM * chunks_per_row; e += kThreads) {
      const int m = e / chunks_per_row, cc = e % chunks_per_row;
      const int b = m0 + m;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (b < p.B && cc * 8 < p.r) {
        int tok = p.prev[(long long)b * p.prev_stride];
        if (tok < 0 || tok >= p.V) tok = 0;  // reported by the sampler
        v = *reinterpret_cast<const uint4*>(U + (long long)tok * p.r + cc * 8);
      }
      const int kb = cc >> 3, c = cc & 7;
      *reinterpret_cast<uint4*>(sA + kb * 16384 + m * 128 + ((c ^ (m & 7)) << 4)) = v;
    }
    fence_async_smem();
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- W producer ----------------
    int it = 0;
    int last[kWStages];
    for (int q = 0; q < kWStages; ++q) last[q] = -1;
    for (int i = 0; i < n_my; ++i) {
      const int n0 = (nt0 + i * nstride) * kTileN;
      bool stop = false;
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int s = it % kWStages;
        if (*(volatile int*)abort_flag || !mbar_wait(&w_empty[s], ((it / kWStages) & 1) ^ 1)) {
          *(volatile int*)abort_flag = 1;
          stop = true;
          break;
        }
        mbar_expect_tx(&w_full[s], kWStageBytes);
        unsigned char* dst = sW + s * kWStageBytes;
#pragma unroll
        for (int vb = 0; vb < 4; ++vb) tma_load_2d(dst + vb * 8192, &map_w, n0 + vb * 64, kb * 64, &w_full[s]);
        last[s] = it;
      }
      if (stop) break;
    }
    if (*(volatile int*)abort_flag)  // let issued loads land before the CTA winds down
      for (int q = 0; q < kWStages; ++q)
        if (last[q] >= 0) mbar_wait(&w_full[q], (last[q] / kWStages) & 1);
  } else if (warp == 2 && lane == 0) {
    // ---------------- base producer ----------------
    int g = 0;
    int last[kBaseSlots];
    for (int q = 0; q < kBaseSlots; ++q) last[q] = -1;
    for (int i = 0; i < n_my; ++i) {
      const int n0 = (nt0 + i * nstride) * kTileN;
      bool stop = false;
      for (int j = 0; j < 4; ++j, ++g) {
        const int s = g % kBaseSlots;
        if (*(volatile int*)abort_flag || !mbar_wait(&b_empty[s], ((g / kBaseSlots) & 1) ^ 1)) {
          *(volatile int*)abort_flag = 1;
          stop = true;
          break;
        }
        mbar_expect_tx(&b_full[s], kBlockBytes);
        tma_load_3d(sBase + s * kBlockBytes, &map_base, n0 + j * 64, p.k - 1, m0, &b_full[s]);
        last[s] = g;
      }
      if (stop) break;
    }
    if (*(volatile int*)abort_flag)
      for (int q = 0; q < kBaseSlots; ++q)
        if (last[q] >= 0) mbar_wait(&b_full[q], (last[q] / kBaseSlots) & 1);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    int it = 0;
    int last_it = -1;  // last W stage whose MMAs were committed
    const uint32_t a_base = su32(sA);
    for (int i = 0; i < n_my; ++i) {
      const int buf = i & 1;
      if (*(volatile int*)abort_flag || !mbar_wait(&t_empty[buf], ((i >> 1) & 1) ^ 1)) {
        *(volatile int*)abort_flag = 1;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t d_tmem = tmem + buf * kTileN;
      bool ok = true;
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int s = it % kWStages;
        if (!mbar_wait(&w_full[s], (it / kWStages) & 1)) {
          ok = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t w_base = su32(sW + s * kWStageBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int step = kb * 4 + kk;
          if (step < ksteps) {
            // A: k-block kb, 32-byte step kk inside the 128-byte swizzle row
            const uint64_t ad = sdesc(a_base + kb * 16384 + kk * 32, 16, 1024);
            // B: 16 k-rows (2 groups of 8) per step; 64-vocab blocks 8 KB apart
            const uint64_t bd = sdesc(w_base + kk * 2048, 8192, 1024);
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
      }
      if (!ok) {
        *(volatile int*)abort_flag = 1;
        break;
      }
      asm volatile(
          "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
              su32(&t_full[buf]))
          : "memory");
    }
    // MMAs complete in order: once the last commit has landed, tensor memory is quiet
    if (*(volatile int*)abort_flag && last_it >= 0)
      mbar_wait(&w_empty[last_it % kWStages], (last_it / kWStages) & 1);
  } else if (warp >= 4) {
    // ---------------- epilogue ----------------
    const int q = warp & 3;             // TMEM lane quadrant
    const int row = q * 32 + lane;      // request row inside the tile
    const int b = m0 + row;
    const bool valid = b < p.B;
    const float tau = valid ? p.temp[b] : 1.f;
    const bool greedy = !(tau > 0.f);
    const float cs = greedy ? 1.f : kLog2e / tau;
    const float sc = (valid && p.bias_scale) ? p.bias_scale[b] : 1.f;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    int g = 0;
    bool fail = false;
    for (int i = 0; i < n_my && !fail; ++i) {
      const int nt = nt0 + i * nstride;
      const int n0 = nt * kTileN;
      const int buf = i & 1;
      bool miss = !mbar_wait(&t_full[buf], (i >> 1) & 1);
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      float run_m = -INFINITY, run_s = 0.f;
      int arg = 0x7fffffff;
      bool bad = false;
      for (int j = 0; j < 4; ++j, ++g) {
        const int s = g % kBaseSlots;
        miss |= !mbar_wait(&b_full[s], (g / kBaseSlots) & 1);
        float acc[64];
        const uint32_t col = tmem + lane_base + buf * kTileN + j * 64;
        tmem_ld32(col, acc);
        tmem_ld32(col + 32, acc + 32);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        unsigned char* blk = sBase + s * kBlockBytes + row * 128;
        float z[64];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4* ptr = reinterpret_cast<uint4*>(blk + ((c ^ (row & 7)) << 4));
          uint4 v = *ptr;
          uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float b0 = __uint_as_float(w[h] << 16);
            const float b1 = __uint_as_float(w[h] & 0xffff0000u);
            const uint16_t d0 = __bfloat16_as_ushort(__float2bfloat16_rn(fmaf(sc, acc[c * 8 + 2 * h], b0)));
            const uint16_t d1 = __bfloat16_as_ushort(__float2bfloat16_rn(fmaf(sc, acc[c * 8 + 2 * h + 1], b1)));
            w[h] = (uint32_t)d0 | ((uint32_t)d1 << 16);
            z[c * 8 + 2 * h] = __uint_as_float((uint32_t)d0 << 16);
            z[c * 8 + 2 * h + 1] = __uint_as_float((uint32_t)d1 << 16);
          }
          *ptr = make_uint4(w[0], w[1], w[2], w[3]);
        }
        // statistics over the valid columns of this block
        const int vcols = min(64, p.V - (n0 + j * 64));
        if (valid) {
          if (greedy) {
#pragma unroll
            for (int e = 0; e < 64; ++e) {
              if (e < vcols) {
                bad |= bad_logit(z[e]);
                argmax_merge(run_m, arg, z[e], n0 + j * 64 + e);
              }
            }
          } else {
            float bm = -INFINITY;
#pragma unroll
            for (int e = 0; e < 64; ++e) {
              if (e < vcols) {
                bad |= bad_logit(z[e]);
                z[e] *= cs;
                bm = fmaxf(bm, z[e]);
              }
            }
            const float nm = fmaxf(run_m, bm);
            float acc_s = 0.f;
#pragma unroll
            for (int e = 0; e < 64; ++e)
              if (e < vcols) acc_s += exp2f(z[e] - nm);
            run_s = (run_m == -INFINITY ? 0.f : run_s * exp2f(run_m - nm)) + acc_s;
            run_m = nm;
          }
        }
        fence_async_smem();
        if (epi_bar_any(miss)) {  // a wait gave up somewhere: every epilogue thread stops here
          fail = true;
          *(volatile int*)abort_flag = 1;
          break;
        }
        if (warp == 4 && lane == 0) {
          tma_store_3d(&map_d, sBase + s * kBlockBytes, n0 + j * 64, p.k - 1, m0);
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          // the previous block's smem has been read by its store: free that slot
          asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
          if (g > 0) mbar_arrive(&b_empty[(g - 1) % kBaseSlots]);
        }
      }
      if (fail) break;
      // this thread is done reading accumulator buffer `buf`
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      mbar_arrive(&t_empty[buf]);
      if (valid) {
        float2 part;
        if (greedy) {
          part.x = bad ? NAN : run_m;
          part.y = __int_as_float(arg);
        } else {
          part.x = run_m;
          part.y = bad ? NAN : run_s;
        }
        p.partials[(long long)b * p.nchunk + nt] = part;
      }
    }
    if (warp == 4 && lane == 0) {
      asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
      if (g > 0 && !fail) mbar_arrive(&b_empty[(g - 1) % kBaseSlots]);
    }
  }

  __syncthreads();
  if (tid == 0 && *(volatile int*)abort_flag) report(p.status, DSPARK_STATUS_TIMEOUT, m0);
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

cudaError_t draft_logits_tc_launch(const DraftArgs& a, int k, int num_sms, cudaStream_t s) {
  using namespace tc;
  CUtensorMap mw, mb, md;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)a.V, (cuuint64_t)a.r};
    const cuuint64_t strides[1] = {(cuuint64_t)a.V * 2};
    const cuuint32_t box[2] = {64, 64};
    if (!make_map(&mw, a.W, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {(cuuint64_t)a.V, (cuuint64_t)a.K, (cuuint64_t)a.B};
    const cuuint64_t strides[2] = {(cuuint64_t)a.V * 2, (cuuint64_t)a.V * a.K * 2};
    const cuuint32_t box[3] = {64, 1, 128};
    if (!make_map(&mb, a.base, 3, dims, strides, box)) return cudaErrorInvalidValue;
    if (!make_map(&md, a.d, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(draft_logits_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e != cudaSuccess) return e;
  Params p;
  p.U = a.U;
  p.prev = (k == 1) ? a.last_tok : a.x + (k - 2);
  p.prev_stride = (k == 1) ? 1 : a.K;
  p.bias_scale = a.bias_scale;
  p.temp = a.temp;
  p.B = a.B;
  p.V = a.V;
  p.r = a.r;
  p.k = k;
  p.m_tiles = (a.B + kTileM - 1) / kTileM;
  p.n_tiles = (a.V + kTileN - 1) / kTileN;
  p.partials = a.partials;
  p.nchunk = a.nchunk;
  p.status = a.status;
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

}  // namespace dspark
