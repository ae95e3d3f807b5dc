// Self-test of the kernels' failure path: every wait of the library's kernels
// is bounded (oq_ptx.cuh), and a wait that runs out records
// OQ_DEVERR_TIMEOUT in the layer's error word and returns instead of
// blocking.  This kernel makes one such wait run out on purpose, with a short
// bound, so that the host side (oq_poll_error) can be checked end to end: an
// mbarrier that expects one arrival, which no thread ever makes.
#include <cuda_runtime.h>

#include <string>

#include "oq_internal.h"
#include "oq_ptx.cuh"

namespace oq {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(int* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  // phase 0 never completes: the wait gives up after limit_ns, sets the error
  // bit and returns false; the kernel then ends normally
  if (threadIdx.x == 0) mbar_wait(&bar, 0u, err, limit_ns);
  __syncwarp();
}

}  // namespace

oq_status wait_timeout_launch(int* err, uint64_t limit_ns, void* stream) {
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, limit_ns);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string("wait-timeout self-test launch: ") + cudaGetErrorString(e));
    return OQ_ERR_CUDA;
  }
  return OQ_OK;
}

}  // namespace oq
