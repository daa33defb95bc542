// Failure detection of the device-side bounded waits, exercised without a GPU
// fault: one thread waits, with the poll limit every kernel of this library
// uses, on an mbarrier phase that nothing ever completes. The wait gives up,
// raises the device error flag and the kernel returns normally, so the context
// stays usable and the host reads MSA_ERR_TIMEOUT from msa_get_device_error.
#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

__global__ void wait_timeout_kernel(int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, err);  // phase 0 never completes
  __syncthreads();
}

}  // namespace

cudaError_t launch_wait_timeout(int* err, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>(err);
  return cudaGetLastError();
}

}  // namespace msa
