// Shared device helpers of the speculative-round kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/dspark.h"

namespace dspark {

// Status block at the start of every workspace.
struct Status {
  unsigned int code;       // OR of DSPARK_STATUS_* bits
  int first_bad_enc;       // INT_MAX - lowest offending request; 0 when none
  unsigned int where;      // first wait site that gave up (kWhere*), 0 when none
  unsigned int pad[61];
};

// Wait sites recorded in Status::where when a bounded wait gives up.
enum WaitSite : unsigned int {
  kWhereVerifyLoad = 1,
  kWhereTcWFull = 10,
  kWhereTcWEmpty = 11,
  kWhereTcBaseFull = 12,
  kWhereTcBaseEmpty = 13,
  kWhereTcAccFull = 14,
  kWhereTcAccEmpty = 15,
  kWhereTcGrid = 16,
  kWhereTcDStore = 17,
  kWhereStatsEmpty = 20,
  kWhereStatsFull = 21,
};

__device__ __forceinline__ void report_wait(Status* st, unsigned int site, int request) {
  atomicCAS(&st->where, 0u, site);
  atomicOr(&st->code, (unsigned int)DSPARK_STATUS_TIMEOUT);
  atomicMax(&st->first_bad_enc, 0x7fffffff - request);
}
static_assert(sizeof(Status) == 256, "status block is 256 bytes");
constexpr size_t kStatusBytes = 256;
// Byte offset, inside the status block's padding, of the grid-barrier counter
// of the one-launch draft round (zeroed by the launcher before each launch).
constexpr size_t kGridBarrierOffset = 64;

__device__ __forceinline__ void report(Status* st, unsigned int bits, int request) {
  atomicOr(&st->code, bits);
  atomicMax(&st->first_bad_enc, 0x7fffffff - request);
}

// log2(e): every sampling kernel works with z = logit * log2(e) / temperature,
// so that exp2 gives the unnormalised softmax weight.
constexpr float kLog2e = 1.44269504088896340736f;

// Bound on every device-side wait (mbarrier polls), in nanoseconds of the
// global timer: a legitimate wait lasts microseconds, so a wait that passes
// this limit reports DSPARK_STATUS_TIMEOUT instead of hanging the GPU.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait for completion of the phase of parity `par` of the mbarrier at
// shared address `bar`; false when it gave up. Each thread polls on its own;
// callers reconverge the warp (__syncwarp) before any warp-aligned instruction.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t par) {
  unsigned long long start = 0;
  for (unsigned it = 0;; ++it) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(bar), "r"(par)
        : "memory");
    if (ok) return true;
    if (it == 0) start = global_ns();
    else if ((it & 255u) == 0 && global_ns() - start > kWaitLimitNs) return false;
  }
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
// as 1, 2, 3", SC'11): ten rounds of two 32x32->64 multiplies whose halves are
// mixed with the other counter words and the key; the key is bumped by the
// Weyl constants between rounds.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t philox_word0(uint32_t c0, uint32_t c1, uint32_t c2,
                                                 uint32_t c3, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    if (i) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t hi0 = __umulhi(0xD2511F53u, c0), lo0 = 0xD2511F53u * c0;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2), lo1 = 0xCD9E8D57u * c2;
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return c0;
}

// Grid-wide barrier of a cooperative launch, by one thread per CTA after a
// CTA barrier: a release arrival on a counter that is zero at launch, then a
// bounded acquire spin until every CTA of barrier number n (1-based; target
// n * gridDim.x) has arrived. False when the wait gave up.
__device__ __forceinline__ bool grid_arrive_wait(unsigned int* ctr, unsigned int target) {
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
  const unsigned long long t0 = global_ns();
  for (unsigned int it = 1;; ++it) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= target) break;
    if ((it & 255u) == 0 && global_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

enum Purpose : uint32_t { kDraft = 0, kAccept = 1, kResidual = 2, kBonus = 3 };

// The round's 24-bit uniform for (request, position, purpose); exact in fp32.
__device__ __forceinline__ float uniform24(uint64_t seed, uint64_t round_id, uint32_t request,
                                           uint32_t position, uint32_t purpose) {
  const uint32_t w = philox_word0(request, (purpose << 24) | position, (uint32_t)round_id,
                                  (uint32_t)(round_id >> 32), (uint32_t)seed,
                                  (uint32_t)(seed >> 32));
  return (float)(w >> 8) * (1.0f / 16777216.0f);
}

// ---------------------------------------------------------------------------
// element access
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

template <int DT>
struct Elem;

template <>
struct Elem<DSPARK_F32> {
  using T = float;
  static constexpr int kBytes = 4;
  __device__ __forceinline__ static float load(const T* p, long long i) { return p[i]; }
  __device__ __forceinline__ static T store_round(float v) { return v; }
  __device__ __forceinline__ static float to_float(T v) { return v; }
};

template <>
struct Elem<DSPARK_BF16> {
  using T = uint16_t;
  static constexpr int kBytes = 2;
  __device__ __forceinline__ static float load(const T* p, long long i) {
    return bf16_bits_to_float(p[i]);
  }
  __device__ __forceinline__ static T store_round(float v) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
  __device__ __forceinline__ static float to_float(T v) { return bf16_bits_to_float(v); }
};

// 16 bytes of logits (8 bf16 or 4 fp32) as floats in index order, from shared
// or global memory.
template <int DT>
struct Vec16;
template <>
struct Vec16<DSPARK_BF16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const void* p, float* v) {
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
  __device__ __forceinline__ static void load(const void* p, float* v) {
    const float4 q = *reinterpret_cast<const float4*>(p);
    v[0] = q.x;
    v[1] = q.y;
    v[2] = q.z;
    v[3] = q.w;
  }
};

// 2^x on the special-function unit (ex2.approx; subnormal results flush to
// zero, far below anything a sampling decision can see).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// max that propagates NaN (any NaN operand gives NaN)
__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// A row is unusable for sampling when it holds NaN or +inf, or is all -inf.
__device__ __forceinline__ bool bad_logit(float v) { return v != v || v == __int_as_float(0x7f800000); }

// ---------------------------------------------------------------------------
// reductions
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
// (value, index) max with the lowest index on ties.
__device__ __forceinline__ void argmax_merge(float& v, int& i, float v2, int i2) {
  if (v2 > v || (v2 == v && i2 < i)) {
    v = v2;
    i = i2;
  }
}
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
    const int i2 = __shfl_xor_sync(0xffffffffu, i, o);
    argmax_merge(v, i, v2, i2);
  }
}
// Inclusive prefix sum over a warp (lane order).
__device__ __forceinline__ float warp_inclusive_scan(float v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

}  // namespace dspark
