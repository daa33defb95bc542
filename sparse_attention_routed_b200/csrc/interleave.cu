// Memory Interleave: routing in several hops, each expanding the context
//   -- "MSA (Memory Sparse Attention)" (robocikowo.com), Komponenty (Memory
//      Interleave: document identifiers and context expansion alternate, so
//      retrieval proceeds in several steps over scattered memory);
//   -- "MSA架构：突破大模型记忆瓶颈的稀疏注意力技术", §3.2 (retrieval in rounds).
// With no generating model, the next hop's routing query is the stated update
// q' = q/|q| + (1/k) sum_j kbar_j/|kbar_j| over the hop's k documents, kbar_j the
// mean of document j's routing keys = its chunks' K_r weighted by their lengths
// (the 1/L_j cancels in the normalisation).
//
// interleave_context_kernel: per (routing row, KV head), copies the documents
// already in the context into the first n_ctx columns of the expanded context and
// sets their scores to -inf, so the hop's top-k takes new documents only (the
// top-k kernel then writes the hop's documents into the next k columns).
// interleave_update_kernel: one CTA per (routing row, KV head), a thread per
// dimension: the hop's documents' weighted chunk sums, normalised with a CTA
// reduction, averaged and added to the normalised query.
#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int kUpdThreads = 128;

__global__ void interleave_context_kernel(const int32_t* __restrict__ ctx, int n_ctx, int64_t rows_h, int n_docs,
                                          int doc_lo, int n_docs_index, float* __restrict__ scores,
                                          int32_t* __restrict__ ctx_out, int ld_out, int* err) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows_h * n_ctx) return;
  const int64_t r = i / n_ctx;
  const int c = (int)(i % n_ctx);
  const int j = ctx[r * n_ctx + c];
  ctx_out[r * ld_out + c] = j;
  const int jl = j - doc_lo;
  if (jl >= 0 && jl < n_docs) scores[r * n_docs + jl] = -INFINITY;
  else if (j < 0 || j >= n_docs_index) atomicCAS(err, 0, kErrInvalidArg);
}

template <int DR>
__global__ void __launch_bounds__(kUpdThreads) interleave_update_kernel(InterleaveUpdateArgs a) {
  __shared__ float red[kUpdThreads / 32];
  __shared__ float bcast;
  const int row = blockIdx.x, h = blockIdx.y;  // row = b * nblk + blk
  const int tid = threadIdx.x;
  const int b = row / a.nblk, blk = row % a.nblk;
  const bool mine = tid < DR;
  auto block_sum = [&](float v) -> float {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if ((tid & 31) == 0) red[tid >> 5] = v;
    __syncthreads();
    if (tid == 0) {
      float t = 0.f;
      for (int w = 0; w < kUpdThreads / 32; ++w) t += red[w];
      bcast = t;
    }
    __syncthreads();
    const float t = bcast;
    __syncthreads();
    return t;
  };
  const int64_t qo = ((int64_t)row * a.n_kv_heads + h) * DR;
  float out = mine ? a.q_r[qo + tid] * a.q_r_inv[(int64_t)row * a.n_kv_heads + h] : 0.f;
  const int32_t* sel = a.sel + ((int64_t)row * a.n_kv_heads + h) * a.sel_ld + a.sel_col;
  for (int i = 0; i < a.k; ++i) {
    const int j = sel[i] - a.doc_lo;
    float acc = 0.f;
    if (j >= 0 && j < a.n_docs && mine) {
      for (int c = a.chunk_off[j]; c < a.chunk_off[j + 1]; ++c)
        acc = fmaf((float)a.chunk_len[c], a.k_r[((int64_t)h * a.nch + c) * DR + tid], acc);
    }
    const float nrm = sqrtf(block_sum(acc * acc));
    out += acc / fmaxf(nrm, 1e-30f) / (float)a.k;
  }
  if (mine) a.q_r_out[(((int64_t)b * a.n_kv_heads + h) * a.nblk + blk) * DR + tid] = out;
}

}  // namespace

cudaError_t launch_interleave_context(const int32_t* ctx, int n_ctx, int64_t rows_h, int n_docs, int doc_lo,
                                      int n_docs_index, float* scores, int32_t* ctx_out, int ld_out, int* err,
                                      cudaStream_t s) {
  if (n_ctx <= 0) return cudaSuccess;
  const int64_t n = rows_h * n_ctx;
  interleave_context_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(ctx, n_ctx, rows_h, n_docs, doc_lo,
                                                                       n_docs_index, scores, ctx_out, ld_out, err);
  return cudaGetLastError();
}

cudaError_t launch_interleave_update(const InterleaveUpdateArgs& a, int route_dim, cudaStream_t s) {
  dim3 grid(a.rows, a.n_kv_heads);
  if (route_dim == 128)
    interleave_update_kernel<128><<<grid, kUpdThreads, 0, s>>>(a);
  else
    interleave_update_kernel<64><<<grid, kUpdThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace msa
