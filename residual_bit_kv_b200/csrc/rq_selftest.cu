// rq_selftest.cu -- a kernel that exercises the device-side failure path: a
// bounded mbarrier wait that runs out records the timeout and returns.
#include "rq_internal.cuh"

namespace rq {
namespace {

__global__ void selftest_wait_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // Nothing arrives on `bar`: the wait on its first phase can only run out.
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0u, err, limit_ns);
}

}  // namespace

cudaError_t launch_selftest_wait(uint32_t* err, uint64_t limit_ns, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace rq
