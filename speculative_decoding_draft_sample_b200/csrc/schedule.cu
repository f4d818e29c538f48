// Calibrated confidence, survival products and the prefix cut.
//
// "DSpark turns speculation into a scheduler", "Confidence is a serving
// primitive": c_k is the probability that draft k survives given that every
// earlier draft survived; P(prefix 1:k survives) = prod_{i<=k} c_i; Sequential
// Temperature Scaling gives every position its own temperature; the
// hardware-aware scheduler picks per-request verify lengths from the survival
// curve and a profiled cost curve, trimming under load. "The speculative loop":
// the latency equation (draft + verify time per accepted token) is the
// objective. "DSpark LLM inference speedup", "The Real Innovation": the
// scheduler stops early, so that the cut of a request never looks past the
// draft being decided.
//
// Cost rule: one CTA of 1024 threads, B*K <= 8192 items, sorted in shared
// memory by a bitonic network on (descending S, k, b), then two fp64 prefix
// scans (expected emitted tokens and verification cost) evaluate every
// admission test at once; the first failing test is the stopping point.
// Threshold and no-cut modes: one thread per request.
#include "common.cuh"
#include "schedule.cuh"

namespace dspark {

constexpr int kSchedThreads = 1024;

// Exclusive scan of one double per thread across the block (thread order).
__device__ double block_exclusive_scan(double v, double* warp_tot, double& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  double pre = 0.0, tot = 0.0;
  for (int w = 0; w < kSchedThreads / 32; ++w) {
    if (w < warp) pre += warp_tot[w];
    tot += warp_tot[w];
  }
  total = tot;
  __syncthreads();
  return pre + incl - v;
}

// c = sigmoid(z / T_k), S = running product, for request b; writes survival
// and returns false on a NaN confidence or a non-positive temperature.
__device__ bool survival_row(const SchedArgs& a, int b, double* S_out) {
  double S = 1.0;
  bool ok = true;
  for (int k = 0; k < a.K; ++k) {
    const double T = (double)a.pos_temp[k];
    const double z = (double)a.conf_logit[b * a.K + k];
    if (!(T > 0.0)) ok = false;
    const double c = 1.0 / (1.0 + exp(-z / T));
    S *= c;
    if (S != S) ok = false;
    const double Sv = (S != S) ? 0.0 : S;
    a.survival[b * a.K + k] = (float)Sv;
    if (S_out) S_out[k] = Sv;
  }
  return ok;
}

// Static threshold and no-cut modes: one thread per request, any batch size.
__global__ void __launch_bounds__(256) survival_cut_kernel(SchedArgs a) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= a.B) return;
  double S[64];
  if (!survival_row(a, b, S)) report(a.status, DSPARK_STATUS_BAD_ROW, b);
  int L = a.K;
  if (a.mode == DSPARK_CUT_THRESHOLD) {
    L = 0;
    for (int k = 0; k < a.K; ++k)
      if (S[k] >= (double)a.threshold) ++L;
  }
  a.cut[b] = L;
}

__global__ void __launch_bounds__(kSchedThreads) prefix_schedule_kernel(SchedArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int n = a.B * a.K;
  int npad = 1;
  while (npad < n) npad <<= 1;
  uint64_t* khi = reinterpret_cast<uint64_t*>(smem);       // ~bits(S): ascending = descending S
  uint32_t* klo = reinterpret_cast<uint32_t*>(khi + npad);  // (k << 13) | b
  int* cut_s = reinterpret_cast<int*>(klo + npad);          // [B]
  __shared__ double warp_tot[kSchedThreads / 32];
  __shared__ int s_stop;
  const int tid = threadIdx.x;

  // survival products, one request per thread iteration
  for (int b = tid; b < a.B; b += kSchedThreads) {
    double S[64];
    if (!survival_row(a, b, S)) report(a.status, DSPARK_STATUS_BAD_ROW, b);
    for (int k = 0; k < a.K; ++k) {
      khi[b * a.K + k] = ~(uint64_t)__double_as_longlong(S[k]);
      klo[b * a.K + k] = ((uint32_t)k << 13) | (uint32_t)b;
    }
    cut_s[b] = 0;
  }
  for (int i = n + tid; i < npad; i += kSchedThreads) {
    khi[i] = ~0ull;
    klo[i] = 0xffffffffu;
  }
  __syncthreads();

  // bitonic sort of (khi, klo) ascending
  for (int size = 2; size <= npad; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < npad / 2; i += kSchedThreads) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint64_t h0 = khi[lo], h1 = khi[hi];
        const uint32_t l0 = klo[lo], l1 = klo[hi];
        const bool gt = (h0 > h1) || (h0 == h1 && l0 > l1);
        if (gt == up) {
          khi[lo] = h1;
          khi[hi] = h0;
          klo[lo] = l1;
          klo[hi] = l0;
        }
      }
      __syncthreads();
    }
  }

  // scans: A_j = B + sum_{i<j} S_i, C_j = fixed + sum_{m < B + j} step_cost[m]
  const int per = npad / kSchedThreads > 0 ? npad / kSchedThreads : 1;
  const int j0 = tid * per;
  double sS = 0.0, sC = 0.0;
  for (int j = j0; j < j0 + per && j < npad; ++j) {
    if (j < n) {
      sS += __longlong_as_double((long long)~khi[j]);
      sC += (double)a.step_cost[a.B + j];
    }
  }
  // cost of the B always-verified slots
  double base_c = 0.0;
  for (int m = tid; m < a.B; m += kSchedThreads) base_c += (double)a.step_cost[m];
  double tS, tC, tB;
  const double exS = block_exclusive_scan(sS, warp_tot, tS);
  const double exC = block_exclusive_scan(sC, warp_tot, tC);
  // block sum of base_c in a fixed order: scan's total
  block_exclusive_scan(base_c, warp_tot, tB);
  if (tid == 0) s_stop = n;
  __syncthreads();
  double A = (double)a.B + exS;
  double Cc = (double)a.fixed_cost + tB + exC;
  for (int j = j0; j < j0 + per && j < n; ++j) {
    const double S = __longlong_as_double((long long)~khi[j]);
    const double c = (double)a.step_cost[a.B + j];
    if (!(S * Cc >= A * c)) atomicMin(&s_stop, j);
    A += S;
    Cc += c;
  }
  __syncthreads();
  const int stop = s_stop;
  for (int j = tid; j < stop; j += kSchedThreads) atomicAdd(&cut_s[klo[j] & 8191u], 1);
  __syncthreads();
  for (int b = tid; b < a.B; b += kSchedThreads) a.cut[b] = cut_s[b];
}

size_t prefix_schedule_smem(int B, int K) {
  int npad = 1;
  while (npad < B * K) npad <<= 1;
  return (size_t)npad * (sizeof(uint64_t) + sizeof(uint32_t)) + (size_t)B * sizeof(int);
}

cudaError_t prefix_schedule_launch(const SchedArgs& a, cudaStream_t s) {
  if (a.mode != DSPARK_CUT_COST) {
    survival_cut_kernel<<<(a.B + 255) / 256, 256, 0, s>>>(a);
    return cudaGetLastError();
  }
  const size_t sm = prefix_schedule_smem(a.B, a.K);
  cudaError_t e = cudaFuncSetAttribute(prefix_schedule_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  prefix_schedule_kernel<<<1, kSchedThreads, sm, s>>>(a);
  return cudaGetLastError();
}

}  // namespace dspark
