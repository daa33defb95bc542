// Gather of the selected K/V slabs from the pinned-host tier into the device
// staging pool, by the SMs themselves reading page-locked host memory through
// its device mapping ("MSA (Memory Sparse Attention)", robocikowo.com,
// Komponenty: full K/V in CPU RAM; Pułapki implementacyjne: pinned memory and
// asynchronous prefetch).
//
// A copy-engine transfer carries a fixed cost per call, so a step of many 1 MB
// slabs moves well below the PCIe rate that one large copy reaches. Here one
// launch moves every slab of a stretch: each job (a run of host-contiguous rows
// and its staging rows) is cut into pieces of kPieceBytes of K plus the same of
// V, CTAs take pieces in turn, and each thread keeps kUnroll 16-byte loads of K
// and of V in flight, so the link sees enough outstanding reads whatever the
// slab size.
#include "internal.h"

namespace msa {
namespace {

constexpr int kThreads = 256;
#ifndef MSA_GATHER_UNROLL
#define MSA_GATHER_UNROLL 4
#endif
#ifndef MSA_GATHER_CTAS_PER_SM
#define MSA_GATHER_CTAS_PER_SM 1
#endif
constexpr int kUnroll = MSA_GATHER_UNROLL;
constexpr int64_t kPieceBytes = 64 * 1024;
constexpr int64_t kPieceVec = kPieceBytes / 16;

__global__ void __launch_bounds__(kThreads) host_gather_kernel(const HostGatherJob* __restrict__ jobs, int njobs,
                                                               int64_t npieces, const uint4* hk, const uint4* hv,
                                                               uint4* __restrict__ dk, uint4* __restrict__ dv,
                                                               int vec_per_row) {
  for (int64_t p = blockIdx.x; p < npieces; p += gridDim.x) {
    // the job holding piece p: the last one whose first piece is <= p (jobs ascend)
    int lo = 0, hi = njobs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (jobs[mid].piece0 <= p) lo = mid;
      else hi = mid - 1;
    }
    const HostGatherJob j = jobs[lo];
    const int64_t v0 = (p - j.piece0) * kPieceVec;
    const int64_t total = j.rows * vec_per_row;
    const int64_t nv = total - v0 < kPieceVec ? total - v0 : kPieceVec;
    const uint4* sk = hk + j.src_row * vec_per_row + v0;
    const uint4* sv = hv + j.src_row * vec_per_row + v0;
    uint4* ok = dk + j.dst_row * vec_per_row + v0;
    uint4* ov = dv + j.dst_row * vec_per_row + v0;
    for (int64_t i = threadIdx.x; i < nv; i += (int64_t)kThreads * kUnroll) {
      uint4 a[kUnroll], b[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t x = i + (int64_t)u * kThreads;
        if (x < nv) {
          a[u] = sk[x];
          b[u] = sv[x];
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t x = i + (int64_t)u * kThreads;
        if (x < nv) {
          ok[x] = a[u];
          ov[x] = b[u];
        }
      }
    }
  }
}

}  // namespace

int64_t host_gather_piece_rows(int head_dim) { return kPieceBytes / ((int64_t)head_dim * 2); }

cudaError_t launch_host_gather(const HostGatherJob* jobs, int njobs, int64_t npieces, const void* hk, const void* hv,
                               void* dk, void* dv, int head_dim, int ctas, cudaStream_t s) {
  if (njobs <= 0 || npieces <= 0) return cudaSuccess;
  ctas *= MSA_GATHER_CTAS_PER_SM;
  const int grid = (int)(npieces < ctas ? npieces : ctas);
  host_gather_kernel<<<grid, kThreads, 0, s>>>(jobs, njobs, npieces, static_cast<const uint4*>(hk),
                                               static_cast<const uint4*>(hv), static_cast<uint4*>(dk),
                                               static_cast<uint4*>(dv), head_dim * 2 / 16);
  return cudaGetLastError();
}

}  // namespace msa
