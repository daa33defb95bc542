// Failure detection of the device-side bounded waits, exercised without a GPU
// fault: one thread waits, with the poll limit every kernel of this library
// uses, on an mbarrier phase that nothing ever completes. The wait gives up,
// raises the device error flag and the kernel returns normally, so the context
// stays usable and the host reads MSA_ERR_TIMEOUT from msa_get_device_error.
#include "common.cuh"
#include "internal.h"
#include "../../include/msa_selftest.h"

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

// ---------------------------------------------------------------------------
// Self-test of exp2_poly3x2, the polynomial 2^x that the tcgen05 prefill kernel
// runs on the FMA pipe for part of its exponentials: y[i] = exp2_poly3x2(x[i])
// and, beside it, CUDA's exp2f(x[i]), so a test can compare both against an
// fp64 reference over the polynomial's whole domain.
namespace msa {
namespace {

__global__ void exp2_poly_kernel(const float* x, float* y_poly, float* y_lib, int64_t n) {
  const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x1 = i + 1 < n ? x[i + 1] : 0.f;
  const float2 p = exp2_poly3x2(make_float2(x[i], x1));
  y_poly[i] = p.x;
  y_lib[i] = exp2f(x[i]);
  if (i + 1 < n) {
    y_poly[i + 1] = p.y;
    y_lib[i + 1] = exp2f(x1);
  }
}

}  // namespace
}  // namespace msa

extern "C" msa_status msa_selftest_exp2_poly(const float* x, float* y_poly, float* y_lib, int64_t n,
                                             void* stream) {
  if (!x || !y_poly || !y_lib || n < 1 || n > (int64_t(1) << 30)) return MSA_ERR_INVALID_ARG;
  const int threads = 256;
  const int64_t blocks = ((n + 1) / 2 + threads - 1) / threads;
  msa::exp2_poly_kernel<<<(unsigned)blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(x, y_poly, y_lib, n);
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Self-test of the document selection: either top-k kernel on caller scores.
extern "C" msa_status msa_selftest_topk(const float* scores, int32_t rows, int32_t n, int32_t k, int32_t* idx,
                                        float* top_scores, int32_t path, void* stream) {
  if (!scores || !idx || rows < 1 || n < 1 || k < 1 || k > n || k > 64 || path < 0 || path > 2)
    return MSA_ERR_INVALID_ARG;
  msa::TopkArgs a{};
  a.scores = scores;
  a.idx = idx;
  a.top_scores = top_scores;
  a.rows = rows;
  a.n = n;
  a.k = k;
  const cudaError_t e = msa::launch_topk_path(a, path, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorInvalidValue) return MSA_ERR_INVALID_ARG;
  return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}
