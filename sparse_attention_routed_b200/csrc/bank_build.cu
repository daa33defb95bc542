// bank_build: chunk-mean pooling of the per-token routing keys into K_r
// (fp32) with 1/||K_r||, and document-wise (Parallel) RoPE applied in place to
// the bank keys.
//   Pooling: "MSA架构：突破大模型记忆瓶颈的稀疏注意力技术", §2.1 item 2 and §3.1
//   (256-token chunk means); a ragged last chunk averages its actual tokens.
//   Parallel RoPE: same page §2.2; "MSA (Memory Sparse Attention)"
//   (robocikowo.com), Komponenty: positions restart at 0 in every document.
//
// One warp per (KV head, chunk). Both passes are pure HBM streams of 128-bit
// coalesced loads: a 128-dim bf16 row is 256 bytes = 16 lanes x 16 bytes, so a
// warp covers two rows per load instruction; the half-warp partial sums are
// combined with one shuffle.
#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

template <int D>
__global__ void __launch_bounds__(256) bank_build_kernel(BankBuildArgs a) {
  constexpr int LANES_PER_ROW = D / 8;          // 16-byte vectors per row
  constexpr int ROWS_PER_ITER = 32 / LANES_PER_ROW;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= a.n_chunks * a.n_kv_heads) return;
  const int h = warp / a.n_chunks;
  const int c = warp % a.n_chunks;
  const int64_t tok0 = a.chunk_tok[c] - a.tok_base;
  const int len = a.chunk_len[c];
  const int pos0 = a.chunk_pos[c];

  // ---- pooling: sum the chunk's rows in fp32, divide by its actual length
  if (a.r != nullptr) {
    const int sub = lane / LANES_PER_ROW;   // which row of the pair/quad
    const int vec = lane % LANES_PER_ROW;   // which 8 dims
    const uint16_t* base = a.r + h * a.r_head_stride + tok0 * D + vec * 8;
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    int r = sub;
    for (; r + 3 * ROWS_PER_ITER < len; r += 4 * ROWS_PER_ITER) {
      uint4 w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        w[u] = __ldcs(reinterpret_cast<const uint4*>(base + (int64_t)(r + u * ROWS_PER_ITER) * D));
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc[0] += bf16_lo(w[u].x); acc[1] += bf16_hi(w[u].x);
        acc[2] += bf16_lo(w[u].y); acc[3] += bf16_hi(w[u].y);
        acc[4] += bf16_lo(w[u].z); acc[5] += bf16_hi(w[u].z);
        acc[6] += bf16_lo(w[u].w); acc[7] += bf16_hi(w[u].w);
      }
    }
    for (; r < len; r += ROWS_PER_ITER) {
      uint4 w = __ldcs(reinterpret_cast<const uint4*>(base + (int64_t)r * D));
      acc[0] += bf16_lo(w.x); acc[1] += bf16_hi(w.x);
      acc[2] += bf16_lo(w.y); acc[3] += bf16_hi(w.y);
      acc[4] += bf16_lo(w.z); acc[5] += bf16_hi(w.z);
      acc[6] += bf16_lo(w.w); acc[7] += bf16_hi(w.w);
    }
#pragma unroll
    for (int off = LANES_PER_ROW; off < 32; off <<= 1)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
    const float inv_len = 1.0f / (float)len;
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      acc[j] *= inv_len;
      ss += acc[j] * acc[j];
    }
#pragma unroll
    for (int off = 1; off < LANES_PER_ROW; off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const int64_t gc = a.chunk0 + c;
    if (lane < LANES_PER_ROW) {
      float4* dst = reinterpret_cast<float4*>(a.k_r + (h * a.nch_total + gc) * D + vec * 8);
      dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
    const float inv = 1.0f / fmaxf(sqrtf(ss), 1e-30f);
    if (lane == 0) a.k_r_inv[h * a.nch_total + gc] = inv;
    if (lane < LANES_PER_ROW) {
      // normalised key split into bf16 hi + lo for the tensor-core router
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float x0 = acc[2 * j] * inv, x1 = acc[2 * j + 1] * inv;
        hi[j] = pack_bf16(x0, x1);
        lo[j] = pack_bf16(x0 - bf16_lo(hi[j]), x1 - bf16_hi(hi[j]));
      }
      const int64_t o = (h * a.nch_total + gc) * D + vec * 8;
      *reinterpret_cast<uint4*>(a.k_hat_hi + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(a.k_hat_lo + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  }

  // ---- Parallel RoPE in place: pair (i, i + D/2) turned by pos * theta_i
  if (a.k != nullptr) {
    constexpr int HALF_VECS = D / 16;             // 16-byte vectors per half row
    constexpr int RROWS = 32 / HALF_VECS;         // rows per warp iteration
    const int sub = lane / HALF_VECS;
    const int vec = lane % HALF_VECS;
    uint16_t* base = a.k + h * a.k_head_stride + tok0 * D + vec * 8;
    for (int r = sub; r < len; r += RROWS) {
      uint4* lo_p = reinterpret_cast<uint4*>(base + (int64_t)r * D);
      uint4* hi_p = reinterpret_cast<uint4*>(base + (int64_t)r * D + D / 2);
      uint4 x = *lo_p, y = *hi_p;
      const float4* cs = reinterpret_cast<const float4*>(a.rope_tab + (int64_t)(pos0 + r) * (D / 2) + vec * 8);
      uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
      uint32_t xo[4], yo[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float4 t = __ldg(cs + j);  // (cos_i, sin_i, cos_{i+1}, sin_{i+1})
        float x0 = bf16_lo(xs[j]), x1 = bf16_hi(xs[j]);
        float y0 = bf16_lo(ys[j]), y1 = bf16_hi(ys[j]);
        xo[j] = pack_bf16(x0 * t.x - y0 * t.y, x1 * t.z - y1 * t.w);
        yo[j] = pack_bf16(y0 * t.x + x0 * t.y, y1 * t.z + x1 * t.w);
      }
      *lo_p = make_uint4(xo[0], xo[1], xo[2], xo[3]);
      *hi_p = make_uint4(yo[0], yo[1], yo[2], yo[3]);
    }
  }
}

// The same build for fp32 banks: routing keys and bank keys in fp32, RoPE'd keys
// stored back in fp32. One warp per (KV head, chunk), 16-byte float4 loads (a
// 128-dim row is 32 lanes, a 64-dim row 16).
template <int D>
__global__ void __launch_bounds__(256) bank_build_f32_kernel(BankBuildArgs a) {
  constexpr int LANES_PER_ROW = D / 4;
  constexpr int ROWS_PER_ITER = 32 / LANES_PER_ROW;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= a.n_chunks * a.n_kv_heads) return;
  const int h = warp / a.n_chunks;
  const int c = warp % a.n_chunks;
  const int64_t tok0 = a.chunk_tok[c] - a.tok_base;
  const int len = a.chunk_len[c];
  const int pos0 = a.chunk_pos[c];

  if (a.r32 != nullptr) {
    const int sub = lane / LANES_PER_ROW;
    const int vec = lane % LANES_PER_ROW;
    const float* base = a.r32 + h * a.r_head_stride + tok0 * D + vec * 4;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int r = sub; r < len; r += ROWS_PER_ITER) {
      const float4 v = __ldcs(reinterpret_cast<const float4*>(base + (int64_t)r * D));
      acc[0] += v.x; acc[1] += v.y; acc[2] += v.z; acc[3] += v.w;
    }
#pragma unroll
    for (int off = LANES_PER_ROW; off < 32; off <<= 1)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
    const float inv_len = 1.0f / (float)len;
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      acc[j] *= inv_len;
      ss += acc[j] * acc[j];
    }
#pragma unroll
    for (int off = 1; off < LANES_PER_ROW; off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const int64_t gc = a.chunk0 + c;
    const float inv = 1.0f / fmaxf(sqrtf(ss), 1e-30f);
    if (lane < LANES_PER_ROW) {
      const int64_t o = (h * a.nch_total + gc) * D + vec * 4;
      *reinterpret_cast<float4*>(a.k_r + o) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      uint32_t hi[2], lo[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float x0 = acc[2 * j] * inv, x1 = acc[2 * j + 1] * inv;
        hi[j] = pack_bf16(x0, x1);
        lo[j] = pack_bf16(x0 - bf16_lo(hi[j]), x1 - bf16_hi(hi[j]));
      }
      *reinterpret_cast<uint2*>(a.k_hat_hi + o) = make_uint2(hi[0], hi[1]);
      *reinterpret_cast<uint2*>(a.k_hat_lo + o) = make_uint2(lo[0], lo[1]);
    }
    if (lane == 0) a.k_r_inv[h * a.nch_total + gc] = inv;
  }

  if (a.k32 != nullptr) {
    constexpr int HALF_VECS = D / 8;             // float4 vectors per half row
    constexpr int RROWS = 32 / HALF_VECS;
    const int sub = lane / HALF_VECS;
    const int vec = lane % HALF_VECS;
    float* base = a.k32 + h * a.k_head_stride + tok0 * D + vec * 4;
    for (int r = sub; r < len; r += RROWS) {
      float4* lo_p = reinterpret_cast<float4*>(base + (int64_t)r * D);
      float4* hi_p = reinterpret_cast<float4*>(base + (int64_t)r * D + D / 2);
      const float4 x = *lo_p, y = *hi_p;
      const float4* cs = reinterpret_cast<const float4*>(a.rope_tab + (int64_t)(pos0 + r) * (D / 2) + vec * 4);
      const float4 t0 = __ldg(cs), t1 = __ldg(cs + 1);  // (cos, sin) of dims vec*4 .. vec*4 + 3
      *lo_p = make_float4(x.x * t0.x - y.x * t0.y, x.y * t0.z - y.y * t0.w, x.z * t1.x - y.z * t1.y,
                          x.w * t1.z - y.w * t1.w);
      *hi_p = make_float4(y.x * t0.x + x.x * t0.y, y.y * t0.z + x.y * t0.w, y.z * t1.x + x.z * t1.y,
                          y.w * t1.z + x.w * t1.w);
    }
  }
}

}  // namespace

cudaError_t launch_bank_build(const BankBuildArgs& a, cudaStream_t s) {
  if (a.n_chunks <= 0) return cudaSuccess;
  const int64_t warps = (int64_t)a.n_chunks * a.n_kv_heads;
  const int blocks = (int)((warps + 7) / 8);
  const bool f32 = a.r32 != nullptr || a.k32 != nullptr;
  if (f32) {
    if (a.head_dim == 128)
      bank_build_f32_kernel<128><<<blocks, 256, 0, s>>>(a);
    else
      bank_build_f32_kernel<64><<<blocks, 256, 0, s>>>(a);
  } else if (a.head_dim == 128) {
    bank_build_kernel<128><<<blocks, 256, 0, s>>>(a);
  } else {
    bank_build_kernel<64><<<blocks, 256, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace msa
