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
// memory by a bitonic network on packed (descending S, k, b) keys (stages
// inside a warp's segment synchronise the warp only), then one fused fp64
// prefix scan (expected emitted tokens and verification cost) evaluates every
// admission test at once; the first failing test is the stopping point.
// Threshold and no-cut modes: one thread per request.
#include "common.cuh"
#include "schedule.cuh"

namespace dspark {

constexpr int kSchedThreads = 1024;

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

// Sort key of a draft: ascending key = descending survival S, then smaller k,
// then smaller b. S in [0, 1] keeps its sign bit clear; its top 44 bits
// (exponent and 33 mantissa bits, 2^-33 relative) are inverted above the 6-bit
// position and 13-bit request fields. Drafts whose S agree to 2^-33 are ordered
// by (k, b); such near-ties only matter across the stopping point.
__device__ __forceinline__ uint64_t sort_key(double S, int k, int b) {
  const uint64_t hi = ((uint64_t)__double_as_longlong(S) >> 19) & ((1ull << 44) - 1);
  return ((~hi & ((1ull << 44) - 1)) << 19) | ((uint64_t)k << 13) | (uint64_t)b;
}

__global__ void __launch_bounds__(kSchedThreads) prefix_schedule_kernel(SchedArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int n = a.B * a.K;
  int npad = 64;
  while (npad < n) npad <<= 1;
  uint64_t* key = reinterpret_cast<uint64_t*>(smem);        // [npad]
  double* Sd = reinterpret_cast<double*>(key + npad);        // [n]: c, then S, by b * K + k
  int* cut_s = reinterpret_cast<int*>(Sd + n);               // [B]
  __shared__ double warp_tot[2][kSchedThreads / 32];
  __shared__ int s_stop;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // calibrated confidences, one draft per thread
  for (int i = tid; i < n; i += kSchedThreads) {
    const int k = i % a.K;
    const double T = (double)a.pos_temp[k];
    const double z = (double)a.conf_logit[i];
    Sd[i] = (T > 0.0) ? 1.0 / (1.0 + exp(-z / T)) : NAN;
  }
  for (int b = tid; b < a.B; b += kSchedThreads) cut_s[b] = 0;
  __syncthreads();
  // survival products, one request per thread; then the sort keys
  for (int b = tid; b < a.B; b += kSchedThreads) {
    double S = 1.0;
    bool bad = false;
    for (int k = 0; k < a.K; ++k) {
      S *= Sd[b * a.K + k];
      if (S != S) bad = true;
      const double Sv = (S != S) ? 0.0 : S;
      Sd[b * a.K + k] = Sv;
      a.survival[b * a.K + k] = (float)Sv;
      key[b * a.K + k] = sort_key(Sv, k, b);
    }
    if (bad) report(a.status, DSPARK_STATUS_BAD_ROW, b);
  }
  for (int i = n + tid; i < npad; i += kSchedThreads) key[i] = ~0ull;
  __syncthreads();

  // bitonic sort, ascending. Thread t owns compare-exchange pairs [t q, t q + q);
  // a warp's pairs touch one segment of 64 q keys, so between two stages whose
  // strides both fit in that segment a warp barrier is enough.
  const int pairs = npad / 2;
  const int q = pairs / kSchedThreads > 0 ? pairs / kSchedThreads : 1;
  const int warp_span = 32 * q;  // pairs per warp
  for (int size = 2; size <= npad; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid * q; i < tid * q + q && i < pairs; ++i) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint64_t k0 = key[lo], k1 = key[hi];
        if ((k0 > k1) == up) {
          key[lo] = k1;
          key[hi] = k0;
        }
      }
      // the next stage reads what other warps wrote unless it stays inside
      // each warp's segment as well
      const int next_stride = stride > 1 ? stride >> 1 : size;
      if (stride <= warp_span && next_stride <= warp_span)
        __syncwarp();
      else
        __syncthreads();
    }
  }
  __syncthreads();

  // one fused scan: A_j = B + sum_{i<j} S_i, C_j = fixed + base cost + sum_{i<j} step_cost[B + i]
  const int per = npad / kSchedThreads > 0 ? npad / kSchedThreads : 1;
  const int j0 = tid * per;
  double sS = 0.0, sC = 0.0;
  for (int j = j0; j < j0 + per && j < n; ++j) {
    const uint64_t kk = key[j];
    sS += Sd[(int)(kk & 8191u) * a.K + (int)((kk >> 13) & 63u)];
    sC += (double)a.step_cost[a.B + j];
  }
  double base_c = 0.0;  // the B always-verified slots
  for (int m = tid; m < a.B; m += kSchedThreads) base_c += (double)a.step_cost[m];
  double iS = sS, iC = sC, iB = base_c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double nS = __shfl_up_sync(0xffffffffu, iS, o);
    const double nC = __shfl_up_sync(0xffffffffu, iC, o);
    if (lane >= o) {
      iS += nS;
      iC += nC;
    }
    iB += __shfl_xor_sync(0xffffffffu, iB, o);
  }
  if (lane == 31) {
    warp_tot[0][warp] = iS;
    warp_tot[1][warp] = iC;
  }
  __shared__ double base_tot[kSchedThreads / 32];
  if (lane == 0) base_tot[warp] = iB;
  if (tid == 0) s_stop = n;
  __syncthreads();
  double preS = 0.0, preC = 0.0, tB = 0.0;
  for (int w = 0; w < kSchedThreads / 32; ++w) {
    if (w < warp) {
      preS += warp_tot[0][w];
      preC += warp_tot[1][w];
    }
    tB += base_tot[w];
  }
  double A = (double)a.B + preS + iS - sS;
  double Cc = (double)a.fixed_cost + tB + preC + iC - sC;
  for (int j = j0; j < j0 + per && j < n; ++j) {
    const uint64_t kk = key[j];
    const double S = Sd[(int)(kk & 8191u) * a.K + (int)((kk >> 13) & 63u)];
    const double c = (double)a.step_cost[a.B + j];
    if (!(S * Cc >= A * c)) {
      atomicMin(&s_stop, j);
      break;
    }
    A += S;
    Cc += c;
  }
  __syncthreads();
  const int stop = s_stop;
  for (int j = tid; j < stop; j += kSchedThreads) atomicAdd(&cut_s[key[j] & 8191u], 1);
  __syncthreads();
  for (int b = tid; b < a.B; b += kSchedThreads) a.cut[b] = cut_s[b];
}

size_t prefix_schedule_smem(int B, int K) {
  int npad = 64;
  while (npad < B * K) npad <<= 1;
  return (size_t)npad * sizeof(uint64_t) + (size_t)B * K * sizeof(double) + (size_t)B * sizeof(int);
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
