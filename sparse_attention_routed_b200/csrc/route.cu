// Routing: q_r block means, cosine scores against every chunk of K_r with the
// per-document max, and the top-k document selection.
//   Router: "MSA架构：突破大模型记忆瓶颈的稀疏注意力技术", §2.1 item 1 (cosine
//   top-k router); "MSA (Memory Sparse Attention)" (robocikowo.com), Komponenty
//   (Router / Routing Projector) and Złożoność obliczeniowa (scoring the whole
//   bank is the bottleneck, so the router is an HBM stream over K_r).
//   Top-k: robocikowo.com, Hiperparametry (Top-k documents).
#include "common.cuh"
#include "internal.h"
#include "pdl.cuh"

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
    const int64_t off =
        (((int64_t)b * a.n_kv_heads + h) * a.q_tokens + (int64_t)blk * a.route_block) * a.route_dim + i;
    float s = 0.f;
    if (a.qr32) {
      for (int t = 0; t < a.route_block; ++t) s += a.qr32[off + (int64_t)t * a.route_dim];
    } else {
      for (int t = 0; t < a.route_block; ++t) s += __uint_as_float((uint32_t)a.qr[off + (int64_t)t * a.route_dim] << 16);
    }
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
// Scoring the whole bank is the step's bottleneck (robocikowo.com, Złożoność
// obliczeniowa): K_r is the one large stream, at 2 multiply-adds per byte for
// 8 query rows -- more than the fp32 FMA pipes sustain at HBM speed -- so the
// contraction runs on tensor cores:
//   S^T[chunk, row] = sum_d Khat[chunk, d] * Qhat[row, d],
// with Khat = K_r/|K_r| and Qhat = q_r/|q_r| each split into bf16 hi + lo and
// the products lo*hi + hi*lo + hi*hi accumulated in fp32 by mma.sync m16n8k16
// (chunks as M, query rows as N). The score is then the cosine itself. With
// LO = false (the bf16 K_r variant) only Khat_hi is streamed, half the bytes,
// and the score is Khat_hi . Qhat (the query keeps its hi + lo split).
// Khat tiles of RITEM chunks arrive by 2-D TMA (128-byte swizzle) into a ring
// whose slots each consumer warp owns. The grid is one wave of resident CTAs;
// CTA (x, h) owns the documents of KV head h whose first chunk lies in the x-th
// of gridDim.x equal chunk ranges (a contiguous run of documents, found by binary
// search in chunk_off), so every CTA streams the same number of K_r bytes to
// within one document whatever the document lengths. Its j-th document goes to
// warp j % RWARPS, which keeps a running max per row over the document's chunks.
constexpr int RWARPS = 4;
constexpr int RBUFS = 2;
constexpr int RSLOTS = RWARPS * RBUFS;
constexpr int RITEM = 16;            // chunks per tile (one m16 tile)
constexpr int RNT_MAX = 2;           // n-tiles of 8 query rows per pass

template <int DR, int NT>
struct RouteShape {
  static constexpr int BOXES = DR / 64;
  static constexpr int BOX_BYTES = RITEM * 128;
  static constexpr int MAT_BYTES = BOXES * BOX_BYTES;  // hi or lo tile
  static constexpr int SLOT_BYTES = 2 * MAT_BYTES;
  static constexpr int NR = NT * 8;
  static constexpr size_t bytes() {
    return 1024 + (size_t)RSLOTS * SLOT_BYTES + 2 * RSLOTS * 8 + 2 * (size_t)NR * DR * 2;
  }
};

// First document whose first chunk is >= c (chunk_off is strictly increasing, n + 1
// entries, chunk_off[n] = nch >= c): a 32-ary search by one warp. Each round probes 32
// evenly spaced entries of [lo, hi], the range the answer lies in, and keeps the span
// between the last probe below c and the first at or above it, so 1024 documents take
// two rounds of loads and 32K three.
__device__ __forceinline__ int first_doc_at_warp(const int32_t* chunk_off, int n_docs, int64_t c, int lane) {
  int lo = 0, hi = n_docs;
  while (hi - lo > 31) {
    const int stride = (hi - lo + 31) / 32;
    const int q = min(lo + (lane + 1) * stride, hi);
    const uint32_t ge = __ballot_sync(0xffffffffu, chunk_off[q] >= c);  // lane 31 probes hi: never 0
    const int f = __ffs(ge) - 1;
    const int new_hi = min(lo + (f + 1) * stride, hi);
    lo = f == 0 ? lo : lo + f * stride + 1;
    hi = new_hi;
  }
  const int q = lo + lane;
  const uint32_t ge = __ballot_sync(0xffffffffu, q <= hi && chunk_off[q] >= c);
  return lo + __ffs(ge) - 1;
}

template <int DR, int NT, bool LO>
__global__ void __launch_bounds__((RWARPS + 1) * 32, 3)
    route_kernel(const __grid_constant__ CUtensorMap tm_hi, const __grid_constant__ CUtensorMap tm_lo,
                 const RouteArgs a, int row0) {
  using SH = RouteShape<DR, NT>;
  constexpr int NR = SH::NR;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + RSLOTS * SH::SLOT_BYTES);
  uint64_t* empty = full + RSLOTS;
  uint16_t* qhi = reinterpret_cast<uint16_t*>(empty + RSLOTS);  // [NR][DR] bf16
  uint16_t* qlo = qhi + NR * DR;                                // [NR][DR] bf16
  const int h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nrows = min(NR, a.rows - row0);
  __shared__ int doc_range[2];
  // A programmatic dependent (the top-k) may launch and set up at once (and the
  // attention behind it run its local-context CTAs in the room left); it waits for
  // this grid to finish before it reads the scores.
  pdl_launch_dependents();

  if (tid == 0) {
    for (int s = 0; s < RSLOTS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_barrier_init();
  }
  // this CTA's documents: those starting in chunks [x * nch / X, (x + 1) * nch / X)
  if (warp < 2) {
    const int d = first_doc_at_warp(a.chunk_off, a.n_docs, (a.nch * (blockIdx.x + warp)) / gridDim.x, lane);
    if (lane == 0) doc_range[warp] = d;
  }
  __syncthreads();
  const int d0 = doc_range[0];
  const int n_mine = doc_range[1] - d0;

  if (warp == RWARPS) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_hi);
      prefetch_tensormap(&tm_lo);
      const uint64_t pol = l2_policy_evict_first();
      int qw[RWARPS] = {};  // items issued per consumer warp (constant-indexed: registers)
      bool ok = true;
      for (int j0 = 0; ok && j0 < n_mine; j0 += RWARPS) {
#pragma unroll
        for (int w = 0; w < RWARPS; ++w) {
          const int j = j0 + w;
          if (!ok || j >= n_mine) break;
          const int c1 = a.chunk_off[d0 + j + 1];
          for (int cs = a.chunk_off[d0 + j]; cs < c1; cs += RITEM) {
            const int slot = w + RWARPS * (qw[w] % RBUFS), use = qw[w] / RBUFS;
            if (use > 0 && !mbar_wait_bounded(&empty[slot], (use - 1) & 1, a.err)) {
              ok = false;
              break;
            }
            ++qw[w];
            uint8_t* dst = ring + slot * SH::SLOT_BYTES;
            const int y = (int)((int64_t)h * a.nch + cs);
            mbar_arrive_expect_tx(&full[slot], LO ? SH::SLOT_BYTES : SH::MAT_BYTES);
#pragma unroll
            for (int bx = 0; bx < SH::BOXES; ++bx) {
              tma_load_2d(dst + bx * SH::BOX_BYTES, &tm_hi, bx * 64, y, &full[slot], pol);
              if (LO) tma_load_2d(dst + SH::MAT_BYTES + bx * SH::BOX_BYTES, &tm_lo, bx * 64, y, &full[slot], pol);
            }
          }
        }
      }
      // no copy may still be landing when the CTA ends
#pragma unroll
      for (int w = 0; w < RWARPS; ++w)
        for (int q = max(0, qw[w] - RBUFS); q < qw[w]; ++q)
          mbar_wait_bounded(&full[w + RWARPS * (q % RBUFS)], (q / RBUFS) & 1, nullptr);
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  // q_r rows of this pass (the block mean of the routing queries, or given), normalised
  // and split into bf16 hi + lo, while the producer's first copies are in flight.
  for (int r = warp; r < NR; r += RWARPS) {
    float v[DR / 32];
#pragma unroll
    for (int t = 0; t < DR / 32; ++t) v[t] = 0.f;
    if (r < nrows) {
      const int row = row0 + r;
      if (a.qr != nullptr) {
        const int nblk = a.q_tokens / a.route_block;
        const int bb = row / nblk, blk = row % nblk;
        const uint16_t* src = a.qr + (((int64_t)bb * a.n_kv_heads + h) * a.q_tokens + (int64_t)blk * a.route_block) * DR;
        for (int t = 0; t < a.route_block; ++t)
#pragma unroll
          for (int u = 0; u < DR / 32; ++u) v[u] += __uint_as_float((uint32_t)src[(int64_t)t * DR + u * 32 + lane] << 16);
        const float inv_b = 1.0f / (float)a.route_block;
#pragma unroll
        for (int u = 0; u < DR / 32; ++u) v[u] *= inv_b;
      } else {
#pragma unroll
        for (int u = 0; u < DR / 32; ++u) v[u] = a.q_r[((int64_t)row * a.n_kv_heads + h) * DR + u * 32 + lane];
      }
    }
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < DR / 32; ++u) ss += v[u] * v[u];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = 1.0f / fmaxf(sqrtf(ss), 1e-30f);
#pragma unroll
    for (int u = 0; u < DR / 32; ++u) {
      const float x = v[u] * inv;
      const __nv_bfloat16 hb = __float2bfloat16_rn(x);
      const __nv_bfloat16 lb = __float2bfloat16_rn(x - __bfloat162float(hb));
      qhi[r * DR + u * 32 + lane] = *reinterpret_cast<const uint16_t*>(&hb);
      qlo[r * DR + u * 32 + lane] = *reinterpret_cast<const uint16_t*>(&lb);
    }
  }
  named_barrier_sync(1, RWARPS * 32);
  const int g = lane >> 2, c = lane & 3;
  // B fragments (k = dims, n = rows): row 8*nt + g, dims 16ks + 2c (+1), +8.
  uint32_t bh[DR / 16][NT][2], bl[DR / 16][NT][2];
#pragma unroll
  for (int ks = 0; ks < DR / 16; ++ks)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int o = (nt * 8 + g) * DR + ks * 16 + hf * 8 + 2 * c;
        bh[ks][nt][hf] = *reinterpret_cast<const uint32_t*>(qhi + o);
        bl[ks][nt][hf] = *reinterpret_cast<const uint32_t*>(qlo + o);
      }
  const int arow = (lane & 7) + ((lane >> 3) & 1) * 8;  // ldmatrix row of this lane
  int qc = 0;
  for (int j = warp; j < n_mine; j += RWARPS) {
    const int doc = d0 + j;
    const int c1 = a.chunk_off[doc + 1];
    float best[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) best[nt][0] = best[nt][1] = -INFINITY;
    bool ok = true;
    for (int cs = a.chunk_off[doc]; cs < c1; cs += RITEM) {
      const int n = min(RITEM, c1 - cs);
      const int slot = warp + RWARPS * (qc % RBUFS), use = qc / RBUFS;
      ++qc;
      if (!mbar_wait_bounded(&full[slot], use & 1, a.err)) {
        ok = false;
        break;
      }
      const uint32_t hbase = smem_addr(ring + slot * SH::SLOT_BYTES);
      const uint32_t lbase = hbase + SH::MAT_BYTES;
      float acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < DR / 16; ++ks) {
        const int col = ks * 16 + (lane >> 4) * 8;
        const uint32_t off = (col >> 6) * SH::BOX_BYTES + swz128(arow, (col & 63) >> 3);
        uint32_t ah[4], al[4];
        ldmatrix_x4(ah, hbase + off);
        if (LO) ldmatrix_x4(al, lbase + off);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (LO) mma_bf16_16816(acc[nt], al, bh[ks][nt][0], bh[ks][nt][1]);
          mma_bf16_16816(acc[nt], ah, bl[ks][nt][0], bl[ks][nt][1]);
          mma_bf16_16816(acc[nt], ah, bh[ks][nt][0], bh[ks][nt][1]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      // rows of the C tile are chunks g and g + 8; mask those past the document
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float v = fmaxf(g < n ? acc[nt][e] : -INFINITY, g + 8 < n ? acc[nt][e + 2] : -INFINITY);
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
          best[nt][e] = fmaxf(best[nt][e], v);
        }
    }
    if (!ok) break;
    if (g == 0) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int r = nt * 8 + 2 * c + e;
          if (r < nrows) a.doc_scores[((int64_t)(row0 + r) * a.n_kv_heads + h) * a.n_docs + doc] = best[nt][e];
        }
    }
  }
}

template <int DR, int NT>
cudaError_t launch_route_t(const RouteArgs& a, const RouteMaps& m, int row0, int sms, cudaStream_t s) {
  auto kern = a.kr_bf16 ? route_kernel<DR, NT, false> : route_kernel<DR, NT, true>;
  const size_t smem = RouteShape<DR, NT>::bytes();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = (int)((228 * 1024) / (smem + 1024));  // 228 KiB per SM, 1 KiB reserved per CTA
  per_sm = per_sm < 1 ? 1 : (per_sm > 3 ? 3 : per_sm);
  if (a.max_ctas_per_sm > 0 && per_sm > a.max_ctas_per_sm) per_sm = a.max_ctas_per_sm;
  // one wave of resident CTAs over the chunk ranges
  int gx = (sms * per_sm) / a.n_kv_heads;
  gx = gx < 1 ? 1 : (gx > a.n_docs ? a.n_docs : gx);
  if (gx > 65535) return cudaErrorInvalidValue;
  kern<<<dim3(gx, a.n_kv_heads), (RWARPS + 1) * 32, smem, s>>>(m.k_hat_hi, m.k_hat_lo, a, row0);
  return cudaGetLastError();
}

template <int DR>
cudaError_t launch_route_dr(const RouteArgs& a, const RouteMaps& m, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  for (int row0 = 0; row0 < a.rows; row0 += 8 * RNT_MAX) {
    const int nr = a.rows - row0;
    const cudaError_t e = nr <= 8 ? launch_route_t<DR, 1>(a, m, row0, sms, s) : launch_route_t<DR, 2>(a, m, row0, sms, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
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
  pdl_launch_dependents();
  pdl_wait();  // the scores come from the router

  uint32_t prefix = 0, mask = 0, remaining = (uint32_t)a.k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += TOPK_THREADS) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < a.n; i += TOPK_THREADS) {
      const uint32_t key = float_order_key(sc[i]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      // Suffix scan over the 256 bins (largest digit first): lane l owns bins
      // 255-8l .. 248-8l; the lane whose range crosses `remaining` picks the digit.
      uint32_t cnt[8], tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[j] = hist[255 - (tid * 8 + j)];
        tot += cnt[j];
      }
      uint32_t incl = tot;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (tid >= off) incl += v;
      }
      const uint32_t excl = incl - tot;
      if (excl < remaining && remaining <= incl) {
        uint32_t cum = excl;
        int dg = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (cum + cnt[j] >= remaining) { dg = 255 - (tid * 8 + j); break; }
          cum += cnt[j];
        }
        s_prefix = prefix | ((uint32_t)dg << shift);
        s_remaining = remaining - cum;
      }
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
    a.idx[(int64_t)row * (a.out_ld ? a.out_ld : a.k) + a.out_col + rank] = a.idx_base + ii;
    if (a.top_scores) a.top_scores[(int64_t)row * a.k + rank] = sc[ii];
  }
}

// ---------------------------------------------------------------- top-k, one warp per row
// For rows of at most 32 * VPL scores and k <= 32: lane l holds scores i * 32 + l.
// Every score becomes a distinct 64-bit key, its order key above the complement of
// its index, so the larger key is the higher score and, between equal scores, the
// lower index: the same order as the block kernel above. The k-th largest of the
// 32 lane maxima, T0, bounds the k-th largest key from below (the k lanes with the
// largest maxima each hold a key >= T0), so the k winners are among the keys >= T0.
// When at most 64 keys pass, one warp-wide bitonic network over 64 elements sorts
// them; otherwise the warp takes the maximum k times.
constexpr int TOPKW_WARPS = 4;
constexpr int TOPKW_CAP = 64;
constexpr int TOPKW_MAX_N = 32 * 64;
constexpr int TOPKW_MAX_K = 32;
// Taken by default up to k = 20: for independent scores about 30 keys then pass T0, while
// at k = 32 (T0 the smallest lane maximum) it is over 100 and the slow path runs.
constexpr int TOPKW_AUTO_MAX_K = 20;

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
  return ((uint64_t)hi << 32) | lo;
}

__device__ __forceinline__ uint64_t shfl_u64(uint64_t v, int src) {
  const uint32_t lo = __shfl_sync(0xffffffffu, (uint32_t)v, src);
  const uint32_t hi = __shfl_sync(0xffffffffu, (uint32_t)(v >> 32), src);
  return ((uint64_t)hi << 32) | lo;
}

__device__ __forceinline__ uint64_t keep(uint64_t x, uint64_t p, bool keep_max) {
  return keep_max ? (x > p ? x : p) : (x < p ? x : p);
}

// Bitonic sort of the 64 elements e = lane + 32 j (j = 0: r0, j = 1: r1), largest
// first. An element of a block that sorts downward ((e & size) == 0) keeps the
// larger of the pair when it is the pair's lower element.
__device__ __forceinline__ void warp_sort64_desc(uint64_t& r0, uint64_t& r1, int lane) {
#pragma unroll
  for (int size = 2; size <= 64; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride == 32) {  // size 64: one downward block; element lane is the lower one
        const uint64_t hi = r0 > r1 ? r0 : r1, lo = r0 > r1 ? r1 : r0;
        r0 = hi;
        r1 = lo;
      } else {
        const uint64_t p0 = shfl_xor_u64(r0, stride), p1 = shfl_xor_u64(r1, stride);
        const bool lower = (lane & stride) == 0;
        r0 = keep(r0, p0, ((lane & size) == 0) == lower);
        r1 = keep(r1, p1, (((lane + 32) & size) == 0) == lower);
      }
    }
}

template <int VPL>
__global__ void __launch_bounds__(TOPKW_WARPS * 32) topk_warp_kernel(TopkArgs a) {
  __shared__ uint64_t cand[TOPKW_WARPS][TOPKW_CAP];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int row = blockIdx.x * TOPKW_WARPS + w;
  pdl_launch_dependents();
  if (row >= a.rows) return;  // a whole warp; no block-wide barrier follows
  pdl_wait();  // the scores come from the router
  const float* sc = a.scores + (int64_t)row * a.n;
  uint64_t key[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = i * 32 + lane;
    key[i] = e < a.n ? ((uint64_t)float_order_key(sc[e]) << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)e) : 0ull;
  }
  uint64_t m = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) m = key[i] > m ? key[i] : m;
  // T0: the k-th largest lane maximum (bitonic sort of the 32 maxima across lanes).
  uint64_t s = m;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1)
      s = keep(s, shfl_xor_u64(s, stride), ((lane & size) == 0) == ((lane & stride) == 0));
  const uint64_t t0 = shfl_u64(s, a.k - 1);
  int c = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) c += key[i] >= t0;
  const int total = __reduce_add_sync(0xffffffffu, (unsigned)c);
  uint64_t mine = 0;
  if (total <= TOPKW_CAP) {
    int off = c;  // inclusive scan of the counts, then exclusive
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, off, d);
      if (lane >= d) off += v;
    }
    off -= c;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (key[i] >= t0) cand[w][off++] = key[i];
    __syncwarp();
    uint64_t r0 = lane < total ? cand[w][lane] : 0ull;
    uint64_t r1 = lane + 32 < total ? cand[w][lane + 32] : 0ull;
    warp_sort64_desc(r0, r1, lane);
    mine = r0;  // element `lane` of the sorted candidates
  } else {
    uint64_t prev = 0;
    for (int r = 0; r < a.k; ++r) {
      uint64_t lm = 0;
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if ((r == 0 || key[i] < prev) && key[i] > lm) lm = key[i];
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) {
        const uint64_t o = shfl_xor_u64(lm, d);
        lm = o > lm ? o : lm;
      }
      if (lane == r) mine = lm;
      prev = lm;
    }
  }
  if (lane < a.k) {
    const int ii = (int)(0xFFFFFFFFu - (uint32_t)mine);
    a.idx[(int64_t)row * (a.out_ld ? a.out_ld : a.k) + a.out_col + lane] = a.idx_base + ii;
    // the score's bits, back from its order key (the key is a bijection of the bits)
    const uint32_t ok = (uint32_t)(mine >> 32);
    if (a.top_scores) a.top_scores[(int64_t)row * a.k + lane] = __uint_as_float(ok & 0x80000000u ? ok & 0x7FFFFFFFu : ~ok);
  }
}

template <int VPL>
cudaError_t launch_topk_warp_t(const TopkArgs& a, cudaStream_t s) {
  return launch_maybe_pdl(topk_warp_kernel<VPL>, dim3((a.rows + TOPKW_WARPS - 1) / TOPKW_WARPS),
                          dim3(TOPKW_WARPS * 32), 0, s, a.pdl != 0, a);
}

}  // namespace

cudaError_t launch_qr_prep(const QrArgs& a, cudaStream_t s) {
  const int nblk = a.q_tokens / a.route_block;
  dim3 grid(a.batch * nblk, a.n_kv_heads);
  qr_prep_kernel<<<grid, 128, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_route(const RouteArgs& a, const RouteMaps& m, cudaStream_t s) {
  if (a.route_dim == 128) return launch_route_dr<128>(a, m, s);
  return launch_route_dr<64>(a, m, s);
}

int route_tile_rows() { return RITEM; }

bool topk_warp_supported(const TopkArgs& a) { return a.k <= TOPKW_MAX_K && a.n <= TOPKW_MAX_N; }

cudaError_t launch_topk_path(const TopkArgs& a, int path, cudaStream_t s) {
  if (a.rows < 1 || a.n < 1 || a.k < 1 || a.k > a.n || a.k > TOPK_MAX) return cudaErrorInvalidValue;
  if (path == 0) path = topk_warp_supported(a) && a.k <= TOPKW_AUTO_MAX_K ? 2 : 1;
  if (path == 1) return launch_maybe_pdl(topk_kernel, dim3(a.rows), dim3(TOPK_THREADS), 0, s, a.pdl != 0, a);
  if (path != 2 || !topk_warp_supported(a)) return cudaErrorInvalidValue;
  if (a.n <= 32 * 8) return launch_topk_warp_t<8>(a, s);
  if (a.n <= 32 * 16) return launch_topk_warp_t<16>(a, s);
  if (a.n <= 32 * 32) return launch_topk_warp_t<32>(a, s);
  return launch_topk_warp_t<64>(a, s);
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) { return launch_topk_path(a, 0, s); }

}  // namespace msa
