// Internal interface of the prefix-schedule kernel.
#pragma once

#include "common.cuh"

namespace dspark {

// Largest B*K the cost rule handles (one CTA, 8-byte keys sorted in shared memory).
constexpr int kMaxScheduleItems = 16384;
constexpr int kSchedThreads = 1024;

struct SchedArgs {
  const float* conf_logit;  // [B, K]
  const float* pos_temp;    // [K]
  const float* step_cost;   // [B * (K + 1)]
  float fixed_cost;
  int B, K, mode;
  float threshold;
  int32_t* cut;             // [B]
  float* survival;          // [B, K]
  Status* status;
};

size_t prefix_schedule_smem(int B, int K);
cudaError_t prefix_schedule_launch(const SchedArgs& a, cudaStream_t s);

}  // namespace dspark
