// Sequential Temperature Scaling of the per-position confidences and their
// expected calibration error.
//
// "DSpark turns speculation into a scheduler", "Confidence is a serving
// primitive": one temperature per draft position, fitted left to right,
// because the scheduler multiplies the calibrated confidences into survival
// probabilities. "DSpark LLM inference speedup", "The Real Innovation": the
// calibration error drops from a few percent to about one.
//
// Position k: S = prod_{i<k} sigmoid(z_i / T_i) * sigmoid(z_k / T) against the
// label "drafts 1..k+1 all survived"; T_k is the temperature of a fixed
// log-spaced grid (kGrid values on [kTLo, kTHi]) with the least negative
// log-likelihood (lowest index on ties). Work per position: every CTA takes a
// contiguous range of samples and thread t accumulates, in fp64 and in sample
// order, the loss of grid temperature t over it (the samples of a tile sit in
// shared memory, with their survival products so far); one CTA then adds the
// CTAs' partials in a fixed order and takes the argmin. ECE: 15 equal-width
// bins of S per position, counts and sums per CTA in shared memory, then one
// CTA per position that adds the CTAs in a fixed order.
#include "calib.cuh"

namespace dspark {

namespace {

constexpr int kCT = 256;  // threads per CTA (= grid temperatures)
static_assert(kCT == kCalGrid, "one thread per grid temperature");
constexpr int kTile = 256;  // samples staged in shared memory at a time
constexpr double kTLo = 0.05, kTHi = 20.0, kEps = 1e-12;

__device__ __forceinline__ double grid_t(int i) {
  return exp(log(kTLo) + i * (log(kTHi) - log(kTLo)) / (kCalGrid - 1));
}
__device__ __forceinline__ double sigm(double x) { return 1.0 / (1.0 + exp(-x)); }

// samples [n0, n1) of CTA blk
__device__ __forceinline__ void block_range(int N, int& n0, int& n1) {
  const long long per = ((long long)N + kCalBlocks - 1) / kCalBlocks;
  n0 = (int)min((long long)N, per * blockIdx.x);
  n1 = (int)min((long long)N, per * (blockIdx.x + 1));
}

// Loss of every grid temperature at position k over this CTA's samples.
__global__ void __launch_bounds__(kCT) sts_nll_partials(CalibArgs a, int k) {
  __shared__ double s_prev[kTile];
  __shared__ double s_z[kTile];
  __shared__ unsigned char s_y[kTile];
  const int t = threadIdx.x;
  const double inv_t = 1.0 / grid_t(t);
  int n0, n1;
  block_range(a.N, n0, n1);
  double acc = 0.0;
  for (int base = n0; base < n1; base += kTile) {
    const int m = min(kTile, n1 - base);
    if (t < m) {
      const long long n = base + t;
      double prev = 1.0;
      for (int i = 0; i < k; ++i) prev *= sigm((double)a.z[n * a.K + i] / (double)a.T[i]);
      s_prev[t] = prev;
      s_z[t] = (double)a.z[n * a.K + k];
      s_y[t] = a.y[n * a.K + k];
    }
    __syncthreads();
    for (int j = 0; j < m; ++j) {
      double p = s_prev[j] * sigm(s_z[j] * inv_t);
      p = fmin(fmax(p, kEps), 1.0 - kEps);
      acc -= s_y[j] ? log(p) : log1p(-p);
    }
    __syncthreads();
  }
  a.partial[(long long)blockIdx.x * kCalGrid + t] = acc;
}

// Totals over the CTAs (eight interleaved running sums per grid temperature,
// added in a fixed order), the argmin (lowest index on ties), T_k.
__global__ void __launch_bounds__(kCT) sts_argmin(CalibArgs a, int k) {
  __shared__ double s_loss[kCalGrid];
  const int t = threadIdx.x;
  constexpr int kLanes = 8;
  static_assert(kCalBlocks % kLanes == 0, "whole groups of CTAs");
  double part[kLanes] = {};
  for (int b = 0; b < kCalBlocks; b += kLanes) {
#pragma unroll
    for (int j = 0; j < kLanes; ++j) part[j] += a.partial[(long long)(b + j) * kCalGrid + t];
  }
  double tot = 0.0;
#pragma unroll
  for (int j = 0; j < kLanes; ++j) tot += part[j];
  s_loss[t] = tot;
  __syncthreads();
  if (t == 0) {
    int best = 0;
    for (int i = 1; i < kCalGrid; ++i)
      if (s_loss[i] < s_loss[best]) best = i;
    a.T[k] = (float)grid_t(best);
    if (a.index) a.index[k] = best;
  }
}

// Per-CTA bin counts and sums of S and of the label, all positions.
__global__ void __launch_bounds__(kCT) ece_partials(CalibArgs a, int fitted) {
  extern __shared__ double s_bins[];  // [K][kCalBins][3]
  const int nb = a.K * kCalBins * 3;
  for (int i = threadIdx.x; i < nb; i += kCT) s_bins[i] = 0.0;
  __syncthreads();
  int n0, n1;
  block_range(a.N, n0, n1);
  for (int n = n0 + threadIdx.x; n < n1; n += kCT) {
    double S = 1.0;
    for (int k = 0; k < a.K; ++k) {
      const double T = fitted ? (double)a.T[k] : 1.0;
      S *= sigm((double)a.z[(long long)n * a.K + k] / T);
      const int bin = min((int)(S * kCalBins), kCalBins - 1);
      double* c = s_bins + (k * kCalBins + bin) * 3;
      atomicAdd(c, 1.0);
      atomicAdd(c + 1, S);
      atomicAdd(c + 2, (double)a.y[(long long)n * a.K + k]);
    }
  }
  __syncthreads();
  double* out = a.bins + (long long)blockIdx.x * nb;
  for (int i = threadIdx.x; i < nb; i += kCT) out[i] = s_bins[i];
}

// ECE of position blockIdx.x from the CTAs' bins. Per bin, thread t adds the
// CTAs t, t + kCT, ... in order, then a fixed tree adds the threads' sums.
__global__ void __launch_bounds__(kCT) ece_finalize(CalibArgs a, float* ece) {
  __shared__ double s_sum[3][kCT];
  const int k = blockIdx.x, t = threadIdx.x;
  const int nb = a.K * kCalBins * 3;
  double e = 0.0;
  for (int bin = 0; bin < kCalBins; ++bin) {
    double v[3] = {0.0, 0.0, 0.0};
    for (int b = t; b < kCalBlocks; b += kCT) {
      const double* c = a.bins + (long long)b * nb + (k * kCalBins + bin) * 3;
#pragma unroll
      for (int f = 0; f < 3; ++f) v[f] += c[f];
    }
#pragma unroll
    for (int f = 0; f < 3; ++f) s_sum[f][t] = v[f];
    __syncthreads();
    for (int w = kCT / 2; w > 0; w >>= 1) {
      if (t < w)
#pragma unroll
        for (int f = 0; f < 3; ++f) s_sum[f][t] += s_sum[f][t + w];
      __syncthreads();
    }
    const double cnt = s_sum[0][0], sp = s_sum[1][0], sy = s_sum[2][0];
    if (cnt > 0.0) e += cnt / a.N * fabs(sp / cnt - sy / cnt);
    __syncthreads();  // s_sum is refilled for the next bin
  }
  if (t == 0) ece[k] = (float)e;
}

}  // namespace

size_t calib_workspace_bytes(int N, int K) {
  (void)N;
  const size_t partial = (size_t)kCalBlocks * kCalGrid * sizeof(double);
  const size_t bins = (size_t)kCalBlocks * K * kCalBins * 3 * sizeof(double);
  return kStatusBytes + partial + bins;
}

cudaError_t calib_launch(CalibArgs a, void* ws, float* ece_before, float* ece_after, cudaStream_t s) {
  char* p = static_cast<char*>(ws) + kStatusBytes;
  a.partial = reinterpret_cast<double*>(p);
  a.bins = reinterpret_cast<double*>(p + (size_t)kCalBlocks * kCalGrid * sizeof(double));
  const size_t ece_smem = (size_t)a.K * kCalBins * 3 * sizeof(double);
  if (ece_smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(ece_partials, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)ece_smem);
    if (e != cudaSuccess) return e;
  }
  if (ece_before) {
    ece_partials<<<kCalBlocks, kCT, ece_smem, s>>>(a, 0);
    ece_finalize<<<a.K, kCT, 0, s>>>(a, ece_before);
  }
  for (int k = 0; k < a.K; ++k) {
    sts_nll_partials<<<kCalBlocks, kCT, 0, s>>>(a, k);
    sts_argmin<<<1, kCT, 0, s>>>(a, k);
  }
  if (ece_after) {
    ece_partials<<<kCalBlocks, kCT, ece_smem, s>>>(a, 1);
    ece_finalize<<<a.K, kCT, 0, s>>>(a, ece_after);
  }
  return cudaGetLastError();
}

}  // namespace dspark
