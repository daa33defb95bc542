// Routing: q_r block means, cosine scores against every chunk of K_r with the
// per-document max, and the top-k document selection.
//   Router: "MSA架构：突破大模型记忆瓶颈的稀疏注意力技术", §2.1 item 1 (cosine
//   top-k router); "MSA (Memory Sparse Attention)" (robocikowo.com), Komponenty
//   (Router / Routing Projector) and Złożoność obliczeniowa (scoring the whole
//   bank is the bottleneck, so the router is an HBM stream over K_r).
//   Top-k: robocikowo.com, Hiperparametry (Top-k documents).
#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

// ---------------------------------------------------------------- q_r
// One block per (row = b*nblk + blk, head); threads over d_r.
__global__ void qr_prep_kernel(QrArgs a) {
  const int nblk = a.q_tokens / a.route_block;
  const int row = blockIdx.x;
  const int h = blockIdx.y;
  const int b = row / nblk, blk = row % nblk;
  __shared__ float red[32];
  float ss = 0.f;
  for (int i = threadIdx.x; i < a.route_dim; i += blockDim.x) {
    const uint16_t* src =
        a.qr + (((int64_t)b * a.n_kv_heads + h) * a.q_tokens + (int64_t)blk * a.route_block) * a.route_dim + i;
    float s = 0.f;
    for (int t = 0; t < a.route_block; ++t) s += __uint_as_float((uint32_t)src[(int64_t)t * a.route_dim] << 16);
    s /= (float)a.route_block;
    a.q_r[((int64_t)row * a.n_kv_heads + h) * a.route_dim + i] = s;
    ss += s * s;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < (int)(blockDim.x + 31) / 32; ++w) t += red[w];
    a.q_r_inv[(int64_t)row * a.n_kv_heads + h] = 1.0f / fmaxf(sqrtf(t), 1e-30f);
  }
}

// ---------------------------------------------------------------- router
// Warp per document: the warp streams the document's K_r rows (one 16-byte
// vector per lane per chunk for d_r = 128) and keeps a running max per query
// row. NR rows are scored per pass; the per-row dot products are finished by
// a reduce-scatter butterfly so that after log2(32) steps lane l holds the
// total of row l >> (5 - log2 NR).
template <int DR, int NR>
__global__ void __launch_bounds__(256) route_kernel(RouteArgs a, int row0) {
  constexpr int VEC = DR / 32;  // floats per lane per chunk (4 or 2)
  constexpr int LOG_NR = (NR == 1) ? 0 : (NR == 2) ? 1 : (NR == 4) ? 2 : (NR == 8) ? 3 : (NR == 16) ? 4 : 5;
  __shared__ __align__(16) float qs[NR * DR];
  __shared__ float qinv[NR];
  const int h = blockIdx.y;
  const int nrows = min(NR, a.rows - row0);
  for (int i = threadIdx.x; i < NR * DR; i += blockDim.x) {
    const int r = i / DR;
    qs[i] = (r < nrows) ? a.q_r[((int64_t)(row0 + r) * a.n_kv_heads + h) * DR + (i % DR)] : 0.f;
  }
  for (int r = threadIdx.x; r < NR; r += blockDim.x)
    qinv[r] = (r < nrows) ? a.q_r_inv[(int64_t)(row0 + r) * a.n_kv_heads + h] : 0.f;
  __syncthreads();

  const int lane = threadIdx.x & 31;
  // This lane's slice of every query row.
  float q[NR][VEC];
#pragma unroll
  for (int r = 0; r < NR; ++r)
#pragma unroll
    for (int v = 0; v < VEC; ++v) q[r][v] = qs[r * DR + lane * VEC + v];
  const int my_row = lane >> (5 - LOG_NR);
  const float my_qinv = qinv[my_row];

  const float* kr = a.k_r + (int64_t)h * a.nch * DR;
  const float* kinv = a.k_r_inv + (int64_t)h * a.nch;
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  for (int doc = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); doc < a.n_docs; doc += warps_total) {
    const int c0 = a.chunk_off[doc], c1 = a.chunk_off[doc + 1];
    float best = -INFINITY;
    for (int c = c0; c < c1; c += 4) {
      float kv[4][VEC];
      float ki[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int cc = min(c + u, c1 - 1);
        if constexpr (VEC == 4) {
          float4 t = __ldcs(reinterpret_cast<const float4*>(kr + (int64_t)cc * DR) + lane);
          kv[u][0] = t.x; kv[u][1] = t.y; kv[u][2] = t.z; kv[u][3] = t.w;
        } else {
          float2 t = __ldcs(reinterpret_cast<const float2*>(kr + (int64_t)cc * DR) + lane);
          kv[u][0] = t.x; kv[u][1] = t.y;
        }
        ki[u] = __ldg(kinv + cc);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float p[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          float s = 0.f;
#pragma unroll
          for (int v = 0; v < VEC; ++v) s = fmaf(q[r][v], kv[u][v], s);
          p[r] = s;
        }
        // reduce-scatter: halve the live rows per step on lane bits 4..(5-LOG_NR)
#pragma unroll
        for (int step = 0; step < LOG_NR; ++step) {
          const int off = 16 >> step;
          const int half = NR >> (step + 1);
          const bool upper = (lane & off) != 0;
#pragma unroll
          for (int i = 0; i < half; ++i) {
            const float send = upper ? p[i] : p[i + half];
            const float keep = upper ? p[i + half] : p[i];
            p[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
          }
        }
        float tot = p[0];
#pragma unroll
        for (int off = (16 >> LOG_NR); off > 0; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
        const float sc = tot * ki[u] * my_qinv;
        if (c + u < c1) best = fmaxf(best, sc);
      }
    }
    // lanes holding the same row agree; the first of each group writes
    if ((lane & ((32 >> LOG_NR) - 1)) == 0 && my_row < nrows)
      a.doc_scores[((int64_t)(row0 + my_row) * a.n_kv_heads + h) * a.n_docs + doc] = best;
  }
}

template <int DR>
cudaError_t launch_route_dr(const RouteArgs& a, cudaStream_t s) {
  const int warps_per_block = 8;
  int blocks_x = (a.n_docs + warps_per_block - 1) / warps_per_block;
  for (int row0 = 0; row0 < a.rows; row0 += 32) {
    const int nr = a.rows - row0;
    dim3 grid(blocks_x, a.n_kv_heads);
    if (nr <= 1) route_kernel<DR, 1><<<grid, 256, 0, s>>>(a, row0);
    else if (nr <= 2) route_kernel<DR, 2><<<grid, 256, 0, s>>>(a, row0);
    else if (nr <= 4) route_kernel<DR, 4><<<grid, 256, 0, s>>>(a, row0);
    else if (nr <= 8) route_kernel<DR, 8><<<grid, 256, 0, s>>>(a, row0);
    else if (nr <= 16) route_kernel<DR, 16><<<grid, 256, 0, s>>>(a, row0);
    else route_kernel<DR, 32><<<grid, 256, 0, s>>>(a, row0);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- top-k
// One block per row. Radix select (4 passes of 8 bits, MSB first) finds the
// exact order key T of the k-th largest score; every score above T is taken,
// and the lowest-index scores equal to T fill the remaining slots (an ordered
// block-wide scan). The <= k winners are ranked by (score desc, index asc).
constexpr int TOPK_THREADS = 512;
constexpr int TOPK_MAX = 64;

__global__ void __launch_bounds__(TOPK_THREADS) topk_kernel(TopkArgs a) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t sel_key[TOPK_MAX];
  __shared__ int32_t sel_idx[TOPK_MAX];
  __shared__ uint32_t s_prefix, s_remaining, s_count;
  __shared__ uint32_t warp_cnt[TOPK_THREADS / 32];
  const int row = blockIdx.x;
  const float* sc = a.scores + (int64_t)row * a.n;
  const int tid = threadIdx.x;

  uint32_t prefix = 0, mask = 0, remaining = (uint32_t)a.k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += TOPK_THREADS) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < a.n; i += TOPK_THREADS) {
      const uint32_t key = float_order_key(sc[i]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      uint32_t cum = 0;
      int dg = 0;
      for (int d = 255; d >= 0; --d) {
        if (cum + hist[d] >= remaining) { dg = d; break; }
        cum += hist[d];
      }
      s_prefix = prefix | ((uint32_t)dg << shift);
      s_remaining = remaining - cum;
    }
    __syncthreads();
    prefix = s_prefix;
    remaining = s_remaining;
    mask |= 255u << shift;
  }
  // prefix == T; `remaining` of the elements equal to T are needed.
  const uint32_t T = prefix;
  const uint32_t need_eq = remaining;
  const uint32_t n_gt = (uint32_t)a.k - need_eq;
  if (tid == 0) s_count = 0;
  __syncthreads();
  for (int i = tid; i < a.n; i += TOPK_THREADS) {
    const uint32_t key = float_order_key(sc[i]);
    if (key > T) {
      const uint32_t p = atomicAdd(&s_count, 1u);
      if (p < TOPK_MAX) { sel_key[p] = key; sel_idx[p] = i; }
    }
  }
  // ties at T, lowest index first
  uint32_t taken = 0;
  for (int base = 0; base < a.n && taken < need_eq; base += TOPK_THREADS) {
    const int i = base + tid;
    const bool eq = (i < a.n) && float_order_key(sc[i]) == T;
    const uint32_t bal = __ballot_sync(0xffffffffu, eq);
    const int w = tid >> 5, l = tid & 31;
    __syncthreads();
    if (l == 0) warp_cnt[w] = __popc(bal);
    __syncthreads();
    uint32_t before = 0, total = 0;
    for (int j = 0; j < TOPK_THREADS / 32; ++j) {
      if (j < w) before += warp_cnt[j];
      total += warp_cnt[j];
    }
    const uint32_t rank = taken + before + __popc(bal & ((1u << l) - 1u));
    if (eq && rank < need_eq) {
      sel_key[n_gt + rank] = T;
      sel_idx[n_gt + rank] = i;
    }
    taken += total;
  }
  __syncthreads();
  if (tid < a.k) {
    const uint32_t kk = sel_key[tid];
    const int ii = sel_idx[tid];
    int rank = 0;
    for (int j = 0; j < a.k; ++j) {
      const uint32_t kj = sel_key[j];
      rank += (kj > kk) || (kj == kk && sel_idx[j] < ii);
    }
    a.idx[(int64_t)row * a.k + rank] = ii;
    if (a.top_scores) a.top_scores[(int64_t)row * a.k + rank] = sc[ii];
  }
}

}  // namespace

cudaError_t launch_qr_prep(const QrArgs& a, cudaStream_t s) {
  const int nblk = a.q_tokens / a.route_block;
  dim3 grid(a.batch * nblk, a.n_kv_heads);
  qr_prep_kernel<<<grid, 128, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s) {
  if (a.route_dim == 128) return launch_route_dr<128>(a, s);
  return launch_route_dr<64>(a, s);
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
  topk_kernel<<<a.rows, TOPK_THREADS, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace msa
