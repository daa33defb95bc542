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

// First document whose first chunk is >= c (chunk_off is strictly increasing, n + 1 entries).
__device__ __forceinline__ int first_doc_at(const int32_t* chunk_off, int n_docs, int64_t c) {
  int lo = 0, hi = n_docs;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (chunk_off[mid] < c) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

template <int DR, int NT, bool LO>
__global__ void __launch_bounds__((RWARPS + 1) * 32, 3)
    route_kernel(const __grid_constant__ CUtensorMap tm_hi, const __grid_constant__ CUtensorMap tm_lo,
                 const RouteArgs a, int row0) {
  using SH = RouteShape<DR, NT>;
  constexpr int NR = SH::NR;
  constexpr int THREADS = (RWARPS + 1) * 32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + RSLOTS * SH::SLOT_BYTES);
  uint64_t* empty = full + RSLOTS;
  // fp32 q_r rows live in the ring until the split below (before any TMA is issued)
  float* qs = reinterpret_cast<float*>(ring);                   // [NR][DR] fp32
  static_assert(SH::NR * DR * 4 <= RSLOTS * SH::SLOT_BYTES, "q_r scratch must fit in the ring");
  uint16_t* qhi = reinterpret_cast<uint16_t*>(empty + RSLOTS);  // [NR][DR] bf16
  uint16_t* qlo = qhi + NR * DR;                                // [NR][DR] bf16
  const int h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nrows = min(NR, a.rows - row0);

  if (tid == 0) {
    for (int s = 0; s < RSLOTS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_barrier_init();
  }
  // this CTA's documents: those starting in chunks [x * nch / X, (x + 1) * nch / X)
  const int d0 = first_doc_at(a.chunk_off, a.n_docs, (a.nch * blockIdx.x) / gridDim.x);
  const int d1 = first_doc_at(a.chunk_off, a.n_docs, (a.nch * (blockIdx.x + 1)) / gridDim.x);
  const int n_mine = d1 - d0;
  // ---- query rows of this pass: q_r (block mean) in fp32
  if (a.qr != nullptr) {
    const int nblk = a.q_tokens / a.route_block;
    const float inv_b = 1.0f / (float)a.route_block;
    for (int i = tid; i < NR * DR; i += THREADS) {
      const int r = i / DR, dd = i % DR;
      float v = 0.f;
      if (r < nrows) {
        const int row = row0 + r, bb = row / nblk, blk = row % nblk;
        const uint16_t* src =
            a.qr + (((int64_t)bb * a.n_kv_heads + h) * a.q_tokens + (int64_t)blk * a.route_block) * DR + dd;
        for (int t = 0; t < a.route_block; ++t) v += __uint_as_float((uint32_t)src[(int64_t)t * DR] << 16);
        v *= inv_b;
      }
      qs[i] = v;
    }
  } else {
    for (int i = tid; i < NR * DR; i += THREADS) {
      const int r = i / DR;
      qs[i] = (r < nrows) ? a.q_r[((int64_t)(row0 + r) * a.n_kv_heads + h) * DR + (i % DR)] : 0.f;
    }
  }
  __syncthreads();
  // ---- normalise and split into bf16 hi + lo
  for (int r = warp; r < NR; r += THREADS / 32) {
    float ss = 0.f;
    for (int i = lane; i < DR; i += 32) ss += qs[r * DR + i] * qs[r * DR + i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = 1.0f / fmaxf(sqrtf(ss), 1e-30f);
    for (int i = lane; i < DR; i += 32) {
      const float x = qs[r * DR + i] * inv;
      const __nv_bfloat16 hb = __float2bfloat16_rn(x);
      const __nv_bfloat16 lb = __float2bfloat16_rn(x - __bfloat162float(hb));
      qhi[r * DR + i] = *reinterpret_cast<const uint16_t*>(&hb);
      qlo[r * DR + i] = *reinterpret_cast<const uint16_t*>(&lb);
    }
  }
  __syncthreads();

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

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
  topk_kernel<<<a.rows, TOPK_THREADS, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace msa
