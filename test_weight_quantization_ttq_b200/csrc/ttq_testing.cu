// Test hooks (include/ttq_testing.h): waits that cannot complete, made with
// the kernels' own bounded wait routines and a short limit, so that a test
// can see the timeout path end in TTQ_FLAG_TIMEOUT and a usable context.
#include "ttq_device.cuh"
#include "ttq_kernels.h"
#include "ttq_testing.h"

namespace ttq {
namespace {

__global__ void wait_timeout_kernel(uint64_t limit_ns, uint32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // one arrival expected; none ever comes
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int never = 0;
    if (!mbar_wait(&bar, 0, &never, limit_ns)) set_flag(status, TTQ_FLAG_TIMEOUT);
  }
}

}  // namespace
}  // namespace ttq

extern "C" ttq_status ttq_testing_wait_timeout(int kind, uint64_t limit_ns, int blocks, void* ws,
                                               size_t ws_bytes, void* stream) {
  if (kind != TTQ_TESTING_WAIT_MBARRIER ||
      limit_ns < 1000 || limit_ns > 1000000000ull || blocks < 1 || blocks > 148 || ws == nullptr ||
      ws_bytes < 4096 || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return TTQ_ERR_INVALID_ARG;
  const cudaError_t e = ttq::launch_kernel(ttq::wait_timeout_kernel, dim3(blocks), dim3(64), 0,
                                           static_cast<cudaStream_t>(stream), false, limit_ns,
                                           static_cast<uint32_t*>(ws));
  return e == cudaSuccess ? TTQ_OK : TTQ_ERR_CUDA;
}
