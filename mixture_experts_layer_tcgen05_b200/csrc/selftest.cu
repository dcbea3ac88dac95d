// Self-test of the bounded device waits that every pipelined kernel uses.
//
// One thread initialises an mbarrier that nothing ever arrives at and waits
// on it through the same bounded wait as the GEMM pipelines, with a caller
// chosen budget. The wait must give up, record MOE_ERR_TIMEOUT at
// kSiteSelfTest in the status word and return, leaving the context usable;
// when the status word already holds a failure the wait must give up at its
// first check instead of spending its budget (the cascade the pipelines rely
// on when one of their waits has failed).
#include "ptx.cuh"

namespace moe {

__global__ void wait_selftest_kernel(int32_t* status, long long budget) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = ptx::smem_addr(&bar);
  if (threadIdx.x == 0) {
    ptx::mbar_init(b, 1);
    ptx::fence_barrier_init();
    ptx::mbar_wait(b, 0, status, kSiteSelfTest, budget);
  }
}

cudaError_t launch_wait_selftest(int32_t* status, long long budget, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(status, budget);
  note_launch();
  return cudaGetLastError();
}

}  // namespace moe
