// msa_route_noalloc: the routing step (q_r, chunk scores, per-document max,
// top-k) with its scratch in a fixed device array instead of memory the
// library allocates. For callers that may not allocate device memory while
// they run: code inside a CUDA-graph capture, a process whose device memory is
// owned by a pool or budget it must not grow, or a host that drives the GPU
// from a context where a cudaMalloc (which can synchronise the device) is not
// acceptable.
//
// The scratch is one file-scope __device__ array of kRouteScratchBytes; every
// GPU that loads libmsa holds it until the process exits.
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

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" msa_status msa_route_noalloc(msa_bank* bank, const msa_query* q, int32_t top_k, float* doc_scores,
                                        int32_t* topk_idx, float* topk_scores, void* stream) {
  if (!bank || !q || !topk_idx || !q->qr) return MSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q->qr) & 15u) != 0) return MSA_ERR_INVALID_ARG;
  msa::BankRouteView v;
  msa_bank_route_view(bank, &v);
  if (q->batch < 1 || q->n_q_heads < 1 || q->q_tokens < 1 || q->local_len < 1 || q->route_block < 1)
    return MSA_ERR_INVALID_ARG;
  if (q->n_q_heads % v.n_kv_heads || q->q_tokens > q->local_len || q->q_tokens % q->route_block)
    return MSA_ERR_INVALID_ARG;
  if (top_k < 1 || top_k > v.n_docs) return MSA_ERR_INVALID_ARG;
  if (top_k > 64) return MSA_ERR_UNSUPPORTED;
  const int nblk = q->q_tokens / q->route_block;
  const size_t rows = (size_t)q->batch * nblk;
  if (rows * v.n_kv_heads > 65535) return MSA_ERR_UNSUPPORTED;
  // scratch: q_r [rows][Hkv][d_r], 1/|q_r| [rows][Hkv], and the document scores
  // [rows][Hkv][n_docs] unless the caller asked for them.
  const size_t b_qr = up256(rows * v.n_kv_heads * v.route_dim * sizeof(float));
  const size_t b_inv = up256(rows * v.n_kv_heads * sizeof(float));
  const size_t b_sc = doc_scores ? 0 : up256(rows * v.n_kv_heads * (size_t)v.n_docs * sizeof(float));
  if (b_qr + b_inv + b_sc > kRouteScratchBytes) return MSA_ERR_UNSUPPORTED;
  void* base = nullptr;
  msa_status st = scratch_address(&base);
  if (st != MSA_OK) return st;
  uint8_t* p = static_cast<uint8_t*>(base);
  float* q_r = reinterpret_cast<float*>(p);
  float* q_inv = reinterpret_cast<float*>(p + b_qr);
  float* scores = doc_scores ? doc_scores : reinterpret_cast<float*>(p + b_qr + b_inv);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  msa::QrArgs qa{static_cast<const uint16_t*>(q->qr), q_r, q_inv, q->batch, v.n_kv_heads, q->q_tokens,
                 q->route_block, v.route_dim};
  if (msa::launch_qr_prep(qa, s) != cudaSuccess) return MSA_ERR_CUDA;
  msa::RouteArgs ra{};
  ra.chunk_off = v.chunk_off;
  ra.q_r = q_r;
  ra.q_r_inv = q_inv;
  ra.doc_scores = scores;
  ra.nch = v.nch;
  ra.rows = (int32_t)rows;
  ra.n_kv_heads = v.n_kv_heads;
  ra.n_docs = v.n_docs;
  ra.route_dim = v.route_dim;
  ra.kr_bf16 = v.kr_bf16;
  // the same router msa_route takes for this shape
  const cudaError_t e = msa::route_tc_supported(v.route_dim, (int)rows) ? msa::launch_route_tc(ra, v.maps, v.sms, s)
                                                                          : msa::launch_route(ra, v.maps, s);
  if (e != cudaSuccess) return MSA_ERR_CUDA;
  msa::TopkArgs ta{scores, topk_idx, topk_scores, (int32_t)(rows * v.n_kv_heads), v.n_docs, top_k};
  if (msa::launch_topk(ta, s) != cudaSuccess) return MSA_ERR_CUDA;
  return MSA_OK;
}
