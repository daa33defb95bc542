// Memory Parallel merges: the bank's documents live in contiguous shards (one per
// device); each shard routes over its own documents and attends over the selected
// documents it holds, and these two kernels combine what the shards produced
//   -- "MSA架构：突破大模型记忆瓶颈的稀疏注意力技术", §2.1 item 3 (distributed memory
//      retrieval across GPUs through an AllGather);
//   -- "MSA (Memory Sparse Attention)" (robocikowo.com), Równoległość (router
//      scoring spread over devices; top-k and the K/V fetch follow in sequence).
//
// merge_topk_kernel: per row, n_parts candidate lists of k (score, global index),
// each ordered (score desc, index asc), indices disjoint between lists. Candidate
// c's place in the union is its place in its own list plus, for every other list,
// the length of that list's prefix that precedes c (a binary search: the lists are
// sorted by the same order). Places are distinct, so the first k are written once
// each. One CTA per row; a thread per candidate.
//
// merge_partials_kernel: per row, n_parts softmax outputs over disjoint key sets
// and their log-sum-exps: L = log sum_s exp(lse_s), out = sum_s exp(lse_s - L) out_s
// (parts with lse = -inf weigh nothing). One warp per row, lanes over dimensions.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int kMergeThreads = 256;
constexpr int kMaxParts = 64;
constexpr int kMaxK = 64;

// (score, index) a precedes b: larger score first, equal scores by lower index
__device__ __forceinline__ bool precedes(float sa, int ia, float sb, int ib) {
  return sa > sb || (sa == sb && ia < ib);
}

__global__ void __launch_bounds__(kMergeThreads)
    merge_topk_kernel(int n_parts, int rows, int k, const float* __restrict__ cs, const int32_t* __restrict__ ci,
                      int32_t* __restrict__ idx, float* __restrict__ scores) {
  __shared__ float s_sc[kMaxParts * kMaxK];
  __shared__ int s_ix[kMaxParts * kMaxK];
  const int row = blockIdx.x;
  const int n = n_parts * k;
  for (int c = threadIdx.x; c < n; c += blockDim.x) {
    const int part = c / k, pos = c % k;
    const int64_t g = ((int64_t)part * rows + row) * k + pos;
    s_sc[c] = cs[g];
    s_ix[c] = ci[g];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < n; c += blockDim.x) {
    const int part = c / k;
    const float sc = s_sc[c];
    const int ix = s_ix[c];
    int place = c % k;
    for (int o = 0; o < n_parts && place < k; ++o) {
      if (o == part) continue;
      // length of list o's prefix that precedes (sc, ix)
      int lo = 0, hi = k;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (precedes(s_sc[o * k + mid], s_ix[o * k + mid], sc, ix)) lo = mid + 1;
        else hi = mid;
      }
      place += lo;
    }
    if (place < k) {
      idx[(int64_t)row * k + place] = ix;
      if (scores) scores[(int64_t)row * k + place] = sc;
    }
  }
}

__global__ void __launch_bounds__(kMergeThreads)
    merge_partials_kernel(int n_parts, int64_t rows, int d, const float* __restrict__ po,
                          const float* __restrict__ pl, float* __restrict__ out, float* __restrict__ lse) {
  const int64_t row = (int64_t)blockIdx.x * (kMergeThreads / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float m = -INFINITY;
  for (int s = 0; s < n_parts; ++s) m = fmaxf(m, pl[(int64_t)s * rows + row]);
  float total = 0.f;
  if (m != -INFINITY)
    for (int s = 0; s < n_parts; ++s) {
      const float x = pl[(int64_t)s * rows + row];
      if (x != -INFINITY) total += expf(x - m);
    }
  const float L = m != -INFINITY ? m + logf(total) : -INFINITY;
  for (int dim = lane; dim < d; dim += 32) {
    float o = 0.f;
    if (L != -INFINITY)
      for (int s = 0; s < n_parts; ++s) {
        const float x = pl[(int64_t)s * rows + row];
        if (x != -INFINITY) o = fmaf(expf(x - L), po[((int64_t)s * rows + row) * d + dim], o);
      }
    out[row * d + dim] = o;
  }
  if (lse && lane == 0) lse[row] = L;
}

}  // namespace

cudaError_t launch_merge_topk(int n_parts, int rows, int k, const float* cand_scores, const int32_t* cand_idx,
                              int32_t* idx, float* scores, cudaStream_t s) {
  if (n_parts < 1 || n_parts > kMaxParts || k < 1 || k > kMaxK || rows < 1 || rows > 65535)
    return cudaErrorInvalidValue;
  merge_topk_kernel<<<rows, kMergeThreads, 0, s>>>(n_parts, rows, k, cand_scores, cand_idx, idx, scores);
  return cudaGetLastError();
}

cudaError_t launch_merge_partials(int n_parts, int64_t rows, int head_dim, const float* part_out,
                                  const float* part_lse, float* out, float* lse, cudaStream_t s) {
  if (n_parts < 1 || rows < 1 || head_dim < 1) return cudaErrorInvalidValue;
  const int64_t blocks = (rows + kMergeThreads / 32 - 1) / (kMergeThreads / 32);
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  merge_partials_kernel<<<(unsigned)blocks, kMergeThreads, 0, s>>>(n_parts, rows, head_dim, part_out, part_lse,
                                                                   out, lse);
  return cudaGetLastError();
}

}  // namespace msa
