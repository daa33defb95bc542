// msa_route_noalloc: the routing step (q_r, chunk scores, per-document max,
// top-k) with its scratch in a fixed device array instead of memory the
// library allocates. For callers that may not allocate device memory while
// they run: a process whose device memory is owned by a pool or budget it must
// not grow, or a host that drives the GPU from a context where a cudaMalloc
// (which can synchronise the device) is not acceptable.
//
// The scratch is one file-scope __device__ array of kRouteScratchBytes; every
// GPU that loads libmsa holds it until the process exits. The routing itself is
// msa_route's (msa_route_with_scratch): the same argument checks, router choice,
// kernels and error flag, with this array in place of the bank's workspace.
#include <mutex>

#include "../../include/msa.h"
#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kRouteScratchBytes = size_t(4) << 20;  // 4 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_route_scratch on the current device. The host-side name
// of the array is only a stand-in: the address comes from cudaGetSymbolAddress,
// asked once per device with that device current.
msa_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return MSA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MSA_OK;
}

}  // namespace

extern "C" msa_status msa_route_noalloc(msa_bank* bank, const msa_query* q, int32_t top_k, float* doc_scores,
                                        int32_t* topk_idx, float* topk_scores, void* stream) {
  if (!bank || !q || !topk_idx) return MSA_ERR_INVALID_ARG;
  void* base = nullptr;
  const msa_status st = scratch_address(&base);
  if (st != MSA_OK) return st;
  return msa_route_with_scratch(bank, q, top_k, doc_scores, topk_idx, topk_scores, base, kRouteScratchBytes,
                                static_cast<cudaStream_t>(stream));
}
