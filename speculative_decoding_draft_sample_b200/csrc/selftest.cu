// Self-test of the bounded device waits that every kernel of the library uses.
//
// One thread waits first on an mbarrier phase that expects an arrival nobody
// makes, then at a grid barrier it reaches alone (a second CTA that never
// comes). Both waits are the library's own helpers with the kernels' own limit
// (kWaitLimitNs, 2 s): each must give up, record DSPARK_STATUS_TIMEOUT with
// the self-test's site, and let the kernel return, so that the context stays
// usable.
#include "common.cuh"

namespace dspark {

namespace {

constexpr unsigned int kWhereSelfTest = 30;  // wait site recorded by the self-test

__global__ void selftest_waits_kernel(Status* st, unsigned int* ctr, int32_t* result) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = (uint32_t)__cvta_generic_to_shared(&bar);
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(b) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  const bool mbar_done = mbar_wait_bounded(b, 0u);  // phase 0 never completes
  if (!mbar_done) report_wait(st, kWhereSelfTest, 0);
  const bool grid_done = grid_arrive_wait(ctr, 2u);  // one CTA of the two arrives
  if (!grid_done) report_wait(st, kWhereSelfTest, 1);
  result[0] = mbar_done ? 0 : 1;
  result[1] = grid_done ? 0 : 1;
}

}  // namespace

cudaError_t selftest_waits_launch(Status* st, int32_t* result, cudaStream_t s) {
  unsigned int* ctr =
      reinterpret_cast<unsigned int*>(reinterpret_cast<char*>(st) + kGridBarrierOffset);
  cudaError_t e = cudaMemsetAsync(ctr, 0, sizeof(unsigned int), s);
  if (e != cudaSuccess) return e;
  selftest_waits_kernel<<<1, 32, 0, s>>>(st, ctr, result);
  return cudaGetLastError();
}

}  // namespace dspark
