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
// Cost rule: one CTA of 1024 threads (it runs on the SMs the draft kernel
// leaves free), B*K <= 24576 items. Every request's drafts already come in
// order (S never increases along a request), so the global order is a merge of
// B sorted runs of K packed (descending S, k, b) keys: log2(B) merge levels in
// shared memory, each thread placing its share of output positions by a
// merge-path split and a sequential merge. One fused fp64 prefix scan
// (expected emitted tokens and verification cost) then evaluates every
// admission test at once; the first failing test is the stopping point.
// Threshold and no-cut modes: one thread per request.
#include "common.cuh"
#include "schedule.cuh"

namespace dspark {

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
// then smaller b. S in [0, 1] keeps its sign bit clear; its next 43 bits
// (exponent and 32 mantissa bits, 2^-32 relative) are inverted above the 6-bit
// position and 15-bit request fields. Drafts whose S agree to 2^-32 are ordered
// by (k, b); such near-ties only matter across the stopping point.
constexpr int kKeyBBits = 15;
constexpr int kKeyKBits = 6;
constexpr int kKeyLow = kKeyBBits + kKeyKBits;
__device__ __forceinline__ uint64_t sort_key(double S, int k, int b) {
  const uint64_t hi = ((uint64_t)__double_as_longlong(S) >> (63 - (64 - kKeyLow))) & ((1ull << (64 - kKeyLow)) - 1);
  return ((~hi & ((1ull << (64 - kKeyLow)) - 1)) << kKeyLow) | ((uint64_t)k << kKeyBBits) | (uint64_t)b;
}
// S of a key, truncated to the 43 bits it keeps (within 2^-32 of the exact
// product: the admission tests compare at far coarser margins).
__device__ __forceinline__ double key_survival(uint64_t key) {
  const uint64_t hi = ~(key >> kKeyLow) & ((1ull << (64 - kKeyLow)) - 1);
  return __longlong_as_double((long long)(hi << (63 - (64 - kKeyLow))));
}
__device__ __forceinline__ int key_request(uint64_t key) { return (int)(key & ((1u << kKeyBBits) - 1)); }

// Items per thread in the merge levels and the scan (kMaxScheduleItems / threads).
constexpr int kPer = kMaxScheduleItems / kSchedThreads;
static_assert(kMaxScheduleItems % kSchedThreads == 0, "items per thread");
static_assert(kMaxScheduleItems < (1 << kKeyBBits), "request field of the sort key");

// Merge path: how many of the d smallest keys of the sorted runs A (length la)
// and B (length lb) come from A (keys are distinct).
__device__ __forceinline__ int merge_split(const uint64_t* A, int la, const uint64_t* Bk, int lb, int d) {
  int lo = max(0, d - lb), hi = min(d, la);
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (A[mid] < Bk[d - 1 - mid]) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(kSchedThreads) prefix_schedule_kernel(SchedArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int n = a.B * a.K;
  uint64_t* key = reinterpret_cast<uint64_t*>(smem);        // [n]
  int* cut_s = reinterpret_cast<int*>(key + n);              // [B]
  __shared__ double warp_tot[2][kSchedThreads / 32];
  __shared__ double base_tot[kSchedThreads / 32];
  __shared__ int s_stop;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + kSchedThreads - 1) / kSchedThreads;   // items per thread (<= kPer)
  const int o0 = min(n, tid * per), o1 = min(n, o0 + per);

  // survival products, one request per thread, and the sort keys: every
  // request's keys form a sorted run of K (S never increases along a request)
  for (int b = tid; b < a.B; b += kSchedThreads) {
    double S = 1.0;
    bool bad = false;
    for (int k = 0; k < a.K; ++k) {
      const double T = (double)a.pos_temp[k];
      const double z = (double)a.conf_logit[b * a.K + k];
      const double c = (T > 0.0) ? 1.0 / (1.0 + exp(-z / T)) : NAN;
      S *= c;
      if (S != S) bad = true;
      const double Sv = (S != S) ? 0.0 : S;
      a.survival[b * a.K + k] = (float)Sv;
      key[b * a.K + k] = sort_key(Sv, k, b);
    }
    if (bad) report(a.status, DSPARK_STATUS_BAD_ROW, b);
    cut_s[b] = 0;
  }
  __syncthreads();

  // merge sort of the runs, log2(B) levels: thread t writes sorted positions
  // [o0, o1) of every level, found by a merge-path split and a sequential
  // merge into registers; all threads read before any writes back in place
  for (int R = a.K; R < n; R <<= 1) {
    uint64_t out[kPer];
    int o = o0;
    int pair_end = o0, i = 0, j = 0, la = 0, lb = 0;
    const uint64_t* A = key;
    const uint64_t* Bk = key;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      if (o < o1) {
        if (o == pair_end) {  // start (or continue in) the pair holding position o
          const int p0 = (o / (2 * R)) * (2 * R);
          la = min(R, n - p0);
          lb = max(0, min(R, n - p0 - R));
          A = key + p0;
          Bk = key + p0 + la;
          pair_end = min(p0 + la + lb, o1);
          const int d = o - p0;
          i = merge_split(A, la, Bk, lb, d);
          j = d - i;
        }
        const bool takeA = i < la && (j >= lb || A[i] < Bk[j]);
        out[e] = takeA ? A[i] : Bk[j];
        i += takeA ? 1 : 0;
        j += takeA ? 0 : 1;
        ++o;
      }
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < kPer; ++e)
      if (o0 + e < o1) key[o0 + e] = out[e];
    __syncthreads();
  }

  // one fused scan: A_j = B + sum_{i<j} S_i, C_j = fixed + base cost + sum_{i<j} step_cost[B + i]
  double sS = 0.0, sC = 0.0;
  for (int q = o0; q < o1; ++q) {
    sS += key_survival(key[q]);
    sC += (double)a.step_cost[a.B + q];
  }
  double base_c = 0.0;  // the B always-verified slots
  for (int m = tid; m < a.B; m += kSchedThreads) base_c += (double)a.step_cost[m];
  double iS = sS, iC = sC, iB = base_c;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const double nS = __shfl_up_sync(0xffffffffu, iS, off);
    const double nC = __shfl_up_sync(0xffffffffu, iC, off);
    if (lane >= off) {
      iS += nS;
      iC += nC;
    }
    iB += __shfl_xor_sync(0xffffffffu, iB, off);
  }
  if (lane == 31) {
    warp_tot[0][warp] = iS;
    warp_tot[1][warp] = iC;
  }
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
  for (int q = o0; q < o1; ++q) {
    const double S = key_survival(key[q]);
    const double c = (double)a.step_cost[a.B + q];
    if (!(S * Cc >= A * c)) {
      atomicMin(&s_stop, q);
      break;
    }
    A += S;
    Cc += c;
  }
  __syncthreads();
  const int stop = s_stop;
  for (int q = tid; q < stop; q += kSchedThreads) atomicAdd(&cut_s[key_request(key[q])], 1);
  __syncthreads();
  for (int b = tid; b < a.B; b += kSchedThreads) a.cut[b] = cut_s[b];
}

size_t prefix_schedule_smem(int B, int K) {
  return (size_t)B * K * sizeof(uint64_t) + (size_t)B * sizeof(int);
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
