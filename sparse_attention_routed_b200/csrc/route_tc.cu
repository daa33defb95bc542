// router_score for many routing rows (prefill: 64-token blocks, block-mean
// q_r) on the tcgen05 tensor cores, accumulators in TMEM, K_r tiles by TMA.
//   "MSA架构：突破大模型记忆瓶颈的稀疏注意力技术", §2.1 item 1 (cosine top-k
//   router over the compressed routing keys); "MSA (Memory Sparse Attention)"
//   (robocikowo.com), Komponenty (Router), Złożoność obliczeniowa (scoring the
//   query against every chunk of the bank is the router's cost).
//
// score(row, chunk) = cos(q_r[row], K_r[chunk]) = q^ . k^ with both sides
// normalised and split into a bf16 high part and a bf16 remainder, the product
// taken as q_lo.k_hi + q_hi.k_lo + q_hi.k_hi (about 16 significant bits on each
// side; the dropped lo.lo term is below 2^-16 relative). With the bf16 K_r
// variant only k^_hi is streamed and the product is q_lo.k_hi + q_hi.k_hi. A
// document's score is the max over its chunks.
//
// One CTA per (range of whole documents, KV head, pass of up to 128 rows):
//   warp 0     TMA: 128-chunk tiles of k^_hi and k^_lo into a 2-stage ring.
//   warp 1     allocates 256 TMEM columns; one lane issues, per tile,
//              D = Q^ K^T (M = 128 rows, N = 128 chunks, K = 128, three
//              products per K step) into one of two accumulators.
//   warps 2-5  first write q^_hi / q^_lo of the pass's rows into shared memory
//              (128-byte swizzled, K-major); then, one thread per row (TMEM
//              lane = row), read each tile's 128 chunk scores with tcgen05.ld in
//              chunk order and keep a running max over the current document,
//              storing it when the document ends. All threads of the CTA cross
//              the same document boundaries, so control flow stays uniform.
// Every mbarrier parity wait targets the phase right after one the same waiter
// saw complete.
#include <algorithm>
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int RT_THREADS = 192;
constexpr int RT_M = 128;                 // routing rows per pass (padded with zeros)
constexpr int RT_N = 128;                 // chunks per tile
constexpr int RT_D = 128;                 // route dim
constexpr int RT_STAGES = 2;
constexpr int RT_BOX = 128 * 128;         // one 64-dim box of a 128-row tile (16 KB)
constexpr int RT_TILE = 2 * RT_BOX;       // 128 rows x 128 dims bf16 (32 KB)
constexpr int OFF_AHI = 0;
constexpr int OFF_ALO = RT_TILE;
constexpr int OFF_B0 = 2 * RT_TILE;       // stage s: hi at OFF_B0 + 2 s RT_TILE, lo right after
constexpr int OFF_BAR = OFF_B0 + RT_STAGES * 2 * RT_TILE;
constexpr int N_BAR = 4 * 2;              // b_full[2], b_empty[2], d_full[2], d_empty[2]
constexpr int OFF_TMEM = OFF_BAR + N_BAR * 8;
constexpr size_t RT_SMEM = 1024 + OFF_TMEM + 16;
static_assert(RT_SMEM <= 232448, "shared memory");

__global__ void __launch_bounds__(RT_THREADS, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tm_hi, const __grid_constant__ CUtensorMap tm_lo,
                    const RouteArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* b_full = bars + 0;
  uint64_t* b_empty = bars + 2;
  uint64_t* d_full = bars + 4;
  uint64_t* d_empty = bars + 6;   // one arrival per epilogue warp
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const int row0 = blockIdx.z * RT_M;
  const int nrows = min(RT_M, a.rows - row0);
  // this CTA's documents [d0, d1) and their chunks [c0, c1)
  const int d0 = (int)((int64_t)blockIdx.x * a.n_docs / gridDim.x);
  const int d1 = (int)((int64_t)(blockIdx.x + 1) * a.n_docs / gridDim.x);
  const int c0 = a.chunk_off[d0], c1 = a.chunk_off[d1];
  const int T = (c1 - c0 + RT_N - 1) / RT_N;
  const uint32_t sbase = smem_addr(sm);

  if (tid == 0) {
    for (int i = 0; i < N_BAR; ++i) mbar_init(&bars[i], i >= 6 ? 4 : 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_base_s, 2 * RT_N);
  if (warp >= 2) {
    // q^ = q_r / |q_r| as bf16 hi + lo, K-major with the 128-byte swizzle; warp w
    // writes rows 32 (w % 4) .. +31, one coalesced 512-byte row at a time (lane l
    // takes dims 4 l .. 4 l + 3)
#pragma unroll 4
    for (int i = 0; i < 32; ++i) {
      const int r = (warp & 3) * 32 + i;
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < nrows) {
        const int64_t qi = (int64_t)(row0 + r) * a.n_kv_heads + h;
        const float inv = a.q_r_inv[qi];
        x = reinterpret_cast<const float4*>(a.q_r + qi * RT_D)[lane];
        x.x *= inv;
        x.y *= inv;
        x.z *= inv;
        x.w *= inv;
      }
      const uint32_t h0 = pack_bf16(x.x, x.y), h1 = pack_bf16(x.z, x.w);
      const uint32_t l0 = pack_bf16(x.x - bf16_lo(h0), x.y - bf16_hi(h0));
      const uint32_t l1 = pack_bf16(x.z - bf16_lo(h1), x.w - bf16_hi(h1));
      const int kc = lane >> 1;  // 16-byte group of the 128 dims
      const uint32_t off = (kc >> 3) * RT_BOX + swz128(r, kc & 7) + (lane & 1) * 8;
      *reinterpret_cast<uint2*>(sm + OFF_AHI + off) = make_uint2(h0, h1);
      *reinterpret_cast<uint2*>(sm + OFF_ALO + off) = make_uint2(l0, l1);
    }
    fence_proxy_async();  // the tensor cores read q^ through the async proxy
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_s;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tm_hi);
      prefetch_tensormap(&tm_lo);
      const uint64_t pol = l2_policy_evict_first();  // K_r is streamed once per step
      for (int t = 0; t < T; ++t) {
        const int st = t % RT_STAGES;
        if (t >= RT_STAGES && !mbar_wait_bounded(&b_empty[st], ((t - RT_STAGES) / RT_STAGES) & 1, a.err)) break;
        // rows past c1 belong to other CTAs (or past the end: zero-filled) and are ignored
        const int y = (int)((int64_t)h * a.nch + c0 + t * RT_N);
        uint8_t* dst = sm + OFF_B0 + st * 2 * RT_TILE;
        mbar_arrive_expect_tx(&b_full[st], a.kr_bf16 ? RT_TILE : 2 * RT_TILE);
        tma_load_2d(dst, &tm_hi, 0, y, &b_full[st], pol);
        tma_load_2d(dst + RT_BOX, &tm_hi, 64, y, &b_full[st], pol);
        if (!a.kr_bf16) {
          tma_load_2d(dst + RT_TILE, &tm_lo, 0, y, &b_full[st], pol);
          tma_load_2d(dst + RT_TILE + RT_BOX, &tm_lo, 64, y, &b_full[st], pol);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(RT_M, RT_N, false);
      // shared memory addresses stay below 2^18: K-step offsets add to the 14-bit start field
      const uint64_t ahi = umma_desc_sw128(sbase + OFF_AHI, 16, 1024);
      const uint64_t alo = umma_desc_sw128(sbase + OFF_ALO, 16, 1024);
      for (int t = 0; t < T; ++t) {
        const int st = t % RT_STAGES, buf = t & 1;
        if (!mbar_wait_bounded(&b_full[st], (t / RT_STAGES) & 1, a.err)) break;
        if (t >= 2 && !mbar_wait_bounded(&d_empty[buf], ((t - 2) >> 1) & 1, a.err)) break;
        tc_fence_after();
        const uint64_t bhi = umma_desc_sw128(sbase + OFF_B0 + st * 2 * RT_TILE, 16, 1024);
        const uint64_t blo = umma_desc_sw128(sbase + OFF_B0 + st * 2 * RT_TILE + RT_TILE, 16, 1024);
        const uint32_t dt = tmem + buf * RT_N;
#pragma unroll
        for (int ks = 0; ks < RT_D / 16; ++ks) {
          const uint64_t o = (uint64_t)(((ks >> 2) * RT_BOX + (ks & 3) * 32) >> 4);
          umma_bf16_ss(dt, alo + o, bhi + o, idesc, ks > 0 ? 1u : 0u);
          if (!a.kr_bf16) umma_bf16_ss(dt, ahi + o, blo + o, idesc, 1u);
          umma_bf16_ss(dt, ahi + o, bhi + o, idesc, 1u);
        }
        umma_commit(&d_full[buf]);
        umma_commit(&b_empty[st]);
      }
    }
  } else {
    // ------------------------------------------------------------ per-document max
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    float* out = a.doc_scores + ((int64_t)(row0 + r) * a.n_kv_heads + h) * a.n_docs;
    const bool valid = r < nrows;
    int doc = d0;
    int next = a.chunk_off[d0 + 1];  // first chunk of the next document
    float run = -INFINITY;
    for (int t = 0; t < T; ++t) {
      const int buf = t & 1;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&d_full[buf], (t >> 1) & 1, a.err))) break;
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < RT_N / 32; ++q) {
        uint32_t v[32];
        tmem_ld32(tl + buf * RT_N + q * 32, v);
        tmem_wait_ld();
        // columns [0, gv) of this group lie in [c0, c1); take them one document
        // segment at a time with predicated (fully unrolled) maxima
        const int g0 = c0 + t * RT_N + q * 32;
        const int gv = min(32, c1 - g0);
        int start = 0;
        while (start < gv) {
          const int end = min(gv, next - g0);  // the current document covers [start, end)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (e >= start && e < end) run = fmaxf(run, __uint_as_float(v[e]));
          start = end;
          if (g0 + end == next) {  // the document ends here
            if (valid) out[doc] = run;
            ++doc;
            run = -INFINITY;
            next = doc < d1 ? a.chunk_off[doc + 1] : INT_MAX;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[buf]);
    }
    if (valid && doc < d1) out[doc] = run;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 2 * RT_N);
}

}  // namespace

bool route_tc_supported(int route_dim, int rows) { return route_dim == RT_D && rows > 16; }
int route_tc_tile_rows() { return RT_N; }

cudaError_t launch_route_tc(const RouteArgs& a, const RouteMaps& m, int sms, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RT_SMEM);
  if (e != cudaSuccess) return e;
  const int per_head = std::max(1, std::min(a.n_docs, sms / a.n_kv_heads));  // one wave (1 CTA per SM)
  dim3 grid(per_head, a.n_kv_heads, (a.rows + RT_M - 1) / RT_M);
  route_tc_kernel<<<grid, RT_THREADS, RT_SMEM, s>>>(m.k_hat_hi128, m.k_hat_lo128, a);
  return cudaGetLastError();
}

}  // namespace msa
