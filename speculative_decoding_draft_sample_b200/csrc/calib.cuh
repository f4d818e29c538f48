// Internal interface of the Sequential Temperature Scaling kernels.
#pragma once

#include "common.cuh"

namespace dspark {

constexpr int kCalGrid = 256;    // grid temperatures, log-spaced on [0.05, 20]
constexpr int kCalBins = 15;     // equal-width ECE bins of S on [0, 1]
// CTAs of the sample-parallel passes: one resident wave on B200 (6 CTAs of
// 256 threads on each of 148 SMs), so that the fp64 exp / log chains of
// enough warps overlap
constexpr int kCalBlocks = 888;

struct CalibArgs {
  const float* z;          // [N, K] confidence logits
  const uint8_t* y;        // [N, K] survival labels (0 / 1)
  int N, K;
  float* T;                // [K] fitted temperatures (written left to right)
  int32_t* index;          // [K] grid index of each, or null
  double* partial;         // [kCalBlocks, kCalGrid] losses (workspace)
  double* bins;            // [kCalBlocks, K, kCalBins, 3] (workspace)
};

size_t calib_workspace_bytes(int N, int K);
cudaError_t calib_launch(CalibArgs a, void* ws, float* ece_before, float* ece_after, cudaStream_t s);

}  // namespace dspark
