// sparse_attend for fp32 banks: the routed attention of the bf16 kernels -- one
// softmax over the selected documents' keys (Parallel RoPE already stored, every
// token visible) and the causal local context (Global RoPE at k_off + u) --
// with every operand, product and sum in fp32.
//   "MSA (Memory Sparse Attention)" (robocikowo.com), Komponenty (Memory Sparse
//   Attention Layer), Pułapki implementacyjne (Global RoPE with a k-offset),
//   Paradygmat wykonania (only the k selected documents take part).
//
// CUDA cores, not tensor cores: the point of this path is fp32 arithmetic end to
// end (no bf16 rounding of the rotated query, the keys or P). A CTA holds
// kRows query rows of one problem (4 warps x 4 rows) in shared memory and streams
// the problem's key list in tiles of 32 keys (K padded to D + 1 words per row, so
// lane j reading key j is conflict-free). Per row and tile, lane j scores key j,
// the warp takes the max and the sum, and each lane updates D / 32 output dims
// with the tile's probabilities broadcast by shuffles (online softmax, exp2
// domain).
#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int kWarps = 4;
constexpr int kRowsPerWarp = 4;
constexpr int kRows = kWarps * kRowsPerWarp;
constexpr int kTile = 32;
constexpr int kMaxTopK = 64;

template <int D>
__global__ void __launch_bounds__(kWarps * 32) attend_f32_kernel(const AttendF32Args a) {
  constexpr int DL = D / 32;  // output dims per lane
  __shared__ float ks[kTile][D + 1];
  __shared__ __align__(16) float vs[kTile][D];
  __shared__ float qs[kRows][D];
  __shared__ int len_s[kMaxTopK];
  __shared__ long long base_s[kMaxTopK];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int p = blockIdx.y;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int nblk = a.q_tokens / a.route_block;
  const int h = p % a.n_kv_heads;
  const int blk = (p / a.n_kv_heads) % nblk;
  const int b = p / (a.n_kv_heads * nblk);
  const int rows = G * a.route_block;
  const int r0 = blockIdx.x * kRows;
  const int i_first = a.local_len - a.q_tokens + blk * a.route_block;  // local index of row 0
  const int i_last = i_first + (min(rows, r0 + kRows) - 1) / G;         // of this CTA's last row
  const int k = a.top_k;

  if (tid < k) {
    const int j = a.sel[(int64_t)p * k + tid];  // a global index on a shard bank
    const int jl = j - a.doc_lo;
    int len = 0;
    long long base = 0;
    if (jl >= 0 && jl < a.n_docs) {
      len = a.doc_len[jl];
      base = (long long)h * a.kv_rows + a.doc_row[jl];
    } else if (j < 0 || j >= a.n_docs_index) {
      atomicCAS(a.err, 0, kErrInvalidArg);
    }
    len_s[tid] = len;
    base_s[tid] = base;
  }
  // the CTA's query rows with Global RoPE at k_off + i
  for (int idx = tid; idx < kRows * (D / 2); idx += blockDim.x) {
    const int rr = idx / (D / 2), dd = idx % (D / 2);
    const int r = r0 + rr;
    float x = 0.f, y = 0.f;
    if (r < rows) {
      const int t = blk * a.route_block + r / G;
      const int hq = h * G + r % G;
      const int i = a.local_len - a.q_tokens + t;
      const float* qrow = a.q + (((int64_t)b * a.n_q_heads + hq) * a.q_tokens + t) * D;
      const float2 cs = a.gtab[(int64_t)i * (D / 2) + dd];
      const float qx = qrow[dd], qy = qrow[dd + D / 2];
      x = qx * cs.x - qy * cs.y;
      y = qy * cs.x + qx * cs.y;
    }
    qs[rr][dd] = x;
    qs[rr][dd + D / 2] = y;
  }

  float m[kRowsPerWarp], l[kRowsPerWarp], o[kRowsPerWarp][DL];
  int lim[kRowsPerWarp];
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int e = 0; e < DL; ++e) o[rr][e] = 0.f;
    lim[rr] = i_first + (r0 + warp * kRowsPerWarp + rr) / G;
  }

  // one tile of nk keys in ks / vs; local tiles mask keys after each row's position
  auto consume = [&](int nk, bool local, int key0) {
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int qrow = warp * kRowsPerWarp + rr;
      if (r0 + qrow >= rows) continue;  // warp-uniform
      const bool vis = lane < nk && (!local || key0 + lane <= lim[rr]);
      float s = -INFINITY;
      if (vis) {
        float acc = 0.f;
#pragma unroll 16
        for (int d = 0; d < D; ++d) acc = fmaf(qs[qrow][d], ks[lane][d], acc);
        s = acc * a.scale_log2;
      }
      float mx = s;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m[rr], mx);
      if (m_new == -INFINITY) continue;  // nothing visible yet (warp-uniform)
      const float alpha = exp2f(m[rr] - m_new);
      const float pj = vis ? exp2f(s - m_new) : 0.f;
      float sum = pj;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      l[rr] = l[rr] * alpha + sum;
#pragma unroll
      for (int e = 0; e < DL; ++e) o[rr][e] *= alpha;
      for (int j = 0; j < nk; ++j) {
        const float pb = __shfl_sync(0xffffffffu, pj, j);
#pragma unroll
        for (int e = 0; e < DL; ++e) o[rr][e] = fmaf(pb, vs[j][lane + 32 * e], o[rr][e]);
      }
      m[rr] = m_new;
    }
  };

  __syncthreads();
  // the selected documents' keys (all visible)
  for (int di = 0; di < k; ++di) {
    const int len = len_s[di];
    const long long base = base_s[di];
    for (int t0 = 0; t0 < len; t0 += kTile) {
      const int nk = min(kTile, len - t0);
      __syncthreads();  // the previous tile is consumed
      for (int idx = tid; idx < kTile * (D / 4); idx += blockDim.x) {
        const int j = idx / (D / 4), c4 = idx % (D / 4);
        float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
        if (j < nk) {
          const int64_t row = base + t0 + j;
          kv = __ldg(reinterpret_cast<const float4*>(a.bank_k + row * D) + c4);
          vv = __ldg(reinterpret_cast<const float4*>(a.bank_v + row * D) + c4);
        }
        ks[j][4 * c4 + 0] = kv.x;
        ks[j][4 * c4 + 1] = kv.y;
        ks[j][4 * c4 + 2] = kv.z;
        ks[j][4 * c4 + 3] = kv.w;
        *reinterpret_cast<float4*>(&vs[j][4 * c4]) = vv;
      }
      __syncthreads();
      consume(nk, false, t0);
    }
  }
  // the local context up to this CTA's last row, Global RoPE at k_off + u
  const int64_t lrow0 = ((int64_t)b * a.n_kv_heads + h) * a.local_len;
  for (int t0 = 0; a.with_local && t0 <= i_last; t0 += kTile) {
    const int nk = min(kTile, i_last + 1 - t0);
    __syncthreads();
    for (int idx = tid; idx < kTile * (D / 2); idx += blockDim.x) {
      const int j = idx / (D / 2), dd = idx % (D / 2);
      float kx = 0.f, ky = 0.f, vx = 0.f, vy = 0.f;
      if (j < nk) {
        const int u = t0 + j;
        const float* kr = a.local_k + (lrow0 + u) * D;
        const float* vr = a.local_v + (lrow0 + u) * D;
        const float2 cs = a.gtab[(int64_t)u * (D / 2) + dd];
        const float x = kr[dd], y = kr[dd + D / 2];
        kx = x * cs.x - y * cs.y;
        ky = y * cs.x + x * cs.y;
        vx = vr[dd];
        vy = vr[dd + D / 2];
      }
      ks[j][dd] = kx;
      ks[j][dd + D / 2] = ky;
      vs[j][dd] = vx;
      vs[j][dd + D / 2] = vy;
    }
    __syncthreads();
    consume(nk, true, t0);
  }

#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    const int r = r0 + warp * kRowsPerWarp + rr;
    if (r >= rows) continue;
    const int t = blk * a.route_block + r / G;
    const int hq = h * G + r % G;
    const int64_t orow = ((int64_t)b * a.n_q_heads + hq) * a.q_tokens + t;
    const float inv = l[rr] > 0.f ? 1.0f / l[rr] : 0.f;
#pragma unroll
    for (int e = 0; e < DL; ++e) a.out[orow * D + lane + 32 * e] = o[rr][e] * inv;
    if (a.lse_out && lane == 0)
      a.lse_out[orow] = l[rr] > 0.f ? (m[rr] + log2f(l[rr])) * 0.693147180559945309f : -INFINITY;
  }
}

}  // namespace

int attend_f32_rows() { return kRows; }

cudaError_t launch_attend_f32(const AttendF32Args& a, int head_dim, cudaStream_t s) {
  if (a.top_k < 1 || a.top_k > kMaxTopK) return cudaErrorInvalidValue;
  const int rows = (a.n_q_heads / a.n_kv_heads) * a.route_block;
  const int nblk = a.q_tokens / a.route_block;
  dim3 grid((rows + kRows - 1) / kRows, a.batch * nblk * a.n_kv_heads);
  if (head_dim == 128)
    attend_f32_kernel<128><<<grid, kWarps * 32, 0, s>>>(a);
  else
    attend_f32_kernel<64><<<grid, kWarps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace msa
