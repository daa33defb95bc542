// sparse_attend (decode): one fused softmax attention over the selected
// documents' K/V (Parallel RoPE already in the bank keys, every token visible)
// plus the causal local context (Global RoPE at k_off + u applied here).
//   "MSA (Memory Sparse Attention)" (robocikowo.com), Komponenty (Memory Sparse
//   Attention Layer: append the top-k documents' K/V to the local context),
//   Pułapki implementacyjne (Global RoPE with a k-offset for the active query
//   context), Paradygmat wykonania (only the k selected documents take part).
//
// Design (B200, HBM-bound):
//  * Problem p = (sequence, routing block, KV head). Its key list is the tiles
//    of TILE keys of each selected document followed by the local tiles up to
//    the last query's position. The list is cut into n_splits equal ranges,
//    one CTA each (split-KV), so ragged documents balance by construction.
//    With n_local_splits > 0 the local tiles get splits of their own, whose
//    CTAs never read the selection: launched as a programmatic dependent of the
//    top-k, with those CTAs first, they stream the local context beside the
//    router, and only the document CTAs wait for the selection.
//  * One producer lane streams K and V tiles with 2-D TMA loads (128-byte
//    swizzle, evict-first L2 policy) into a ring of WARPS x BUFS slots; consumer
//    warp w owns slots w, w + WARPS, ... and takes relative tiles w, w + WARPS, ...
//  * The problem's query rows (G heads x Bq tokens <= 16) are few, so the MMA
//    runs "keys as M": S^T = K Q^T with mma.sync m16n8k16 (keys fill M=16, the
//    rows sit in N=8), then O^T += V^T P^T with V^T fed by ldmatrix.trans and
//    P^T produced in registers by movmatrix.trans. Padding is at most N-side.
//  * Online softmax in the exp2 domain; the consumer warps merge in shared
//    memory, each CTA leaves (m, l, O) per row, and the last CTA of a problem
//    to finish (a wrapping atomic counter) merges all splits into the output.
#include "common.cuh"
#include "internal.h"
#include "pdl.cuh"

namespace msa {
namespace {

constexpr int kMaxTopK = 64;
constexpr int kMaxSplits = 64;
constexpr int kRowsMax = 16;

template <int D_, int TILE_, int WARPS_, int BUFS_>
struct Shape {
  static constexpr int D = D_;
  static constexpr int TILE = TILE_;                  // keys per tile
  static constexpr int WARPS = WARPS_;                // consumer warps
  static constexpr int BUFS = BUFS_;                  // ring slots per consumer warp
  static constexpr int STAGES = WARPS * BUFS;
  static constexpr int MT = TILE / 16;                // 16-key m-tiles per tile
  static constexpr int BOXES = D / 64;                // 128-byte-wide TMA boxes per row
  static constexpr int BOX_BYTES = TILE * 128;
  static constexpr int TILE_BYTES = TILE * D * 2;     // one of K or V
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
  static constexpr int THREADS = (WARPS + 1) * 32;
  // resident CTAs per SM the ring allows (227 KiB of shared memory per SM)
  static constexpr int MINB = RING_BYTES <= 70 * 1024 ? 3 : (RING_BYTES <= 108 * 1024 ? 2 : 1);
  static_assert(TILE % 16 == 0 && TILE <= 256, "tile");
};

// The shape the library launches (one place to change it; the macros exist so
// that other shapes can be compiled for measurement).
#ifndef MSA_DECODE_TILE
#define MSA_DECODE_TILE 32
#endif
#ifndef MSA_DECODE_WARPS
#define MSA_DECODE_WARPS 4
#endif
#ifndef MSA_DECODE_BUFS
#define MSA_DECODE_BUFS 1
#endif
// Cost of a local tile (Global RoPE in shared memory) relative to a bank tile,
// used to cut each problem's tile list into splits of equal cost.
#ifndef MSA_DECODE_LOCAL_W
#define MSA_DECODE_LOCAL_W 2
#endif
template <int D>
using Decode = Shape<D, MSA_DECODE_TILE, MSA_DECODE_WARPS, MSA_DECODE_BUFS>;

struct TileRef {
  int di;  // document slot (0..k-1) or k for the local context
  int tt;  // tile index inside it
};

__device__ __forceinline__ TileRef locate(const int* tile_start, int k, int j, int hint) {
  int di = hint;
  while (di < k && j >= tile_start[di + 1]) ++di;
  return {di, j - tile_start[di]};
}

// Relative tile n goes to consumer warp n % WARPS; that warp's q-th tile uses
// slot w + WARPS * (q % BUFS). Every slot is filled and drained by one producer
// and one consumer in order, so each mbarrier parity wait targets the phase
// right after one the waiter saw complete (the only case where it is unambiguous).
template <class S>
__device__ __forceinline__ void slot_of(int n, int& stage, int& use) {
  const int w = n % S::WARPS, q = n / S::WARPS;
  stage = w + S::WARPS * (q % S::BUFS);
  use = q / S::BUFS;
}

template <class S>
constexpr size_t smem_bytes(int nt) {
  // ring, or the merge scratch that reuses it
  size_t scratch = (size_t)S::WARPS * nt * 8 * (S::D + 2) * 4;
  size_t body = (size_t)S::RING_BYTES > scratch ? (size_t)S::RING_BYTES : scratch;
  return 1024 + body + 2 * S::STAGES * 8 + (kMaxTopK + 2) * 4 + kMaxTopK * 4 + kMaxTopK * 8 +
         kMaxSplits * kRowsMax * 4 + 64;
}

template <class S, int NT>
__global__ void __launch_bounds__(S::THREADS, S::MINB)
    attend_decode_kernel(const __grid_constant__ CUtensorMap tm_bk, const __grid_constant__ CUtensorMap tm_bv,
                         const __grid_constant__ CUtensorMap tm_lk, const __grid_constant__ CUtensorMap tm_lv,
                         const AttendArgs a) {
  constexpr int D = S::D, TILE = S::TILE, WARPS = S::WARPS, MT = S::MT;
  constexpr int R = NT * 8;
  static_assert((size_t)WARPS * R * (D + 2) * 4 <= (size_t)S::RING_BYTES, "merge scratch must fit in the ring");
  extern __shared__ uint8_t smem_raw[];
  // 128-byte swizzle is defined on shared-memory address bits: align the ring to 1 KiB there.
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::RING_BYTES);
  uint64_t* empty = full + S::STAGES;
  int* tile_start = reinterpret_cast<int*>(empty + S::STAGES);                 // [kMaxTopK + 2]
  int* doc_len_s = tile_start + kMaxTopK + 2;                                  // [kMaxTopK]
  long long* doc_base_s = reinterpret_cast<long long*>(doc_len_s + kMaxTopK);  // [kMaxTopK]
  float* wgt_s = reinterpret_cast<float*>(doc_base_s + kMaxTopK);              // [kMaxSplits][kRowsMax]
  int* flag_s = reinterpret_cast<int*>(wgt_s + kMaxSplits * kRowsMax);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int nblk = a.q_tokens / a.route_block;
  // CTA -> (problem, split). Launched the ordinary way: problem after problem, so that
  // the local tiles (Global RoPE in shared memory) spread evenly over the waves. As a
  // programmatic dependent: every problem's local splits first (split 0 of every
  // problem, then split 1, ...), so that they run beside the routing, then the document
  // splits problem after problem. The order moves no tile to another split.
  const int nls = a.n_local_splits;
  const int n_problems = a.batch * nblk * a.n_kv_heads;
  int p, split;
  if (!a.pdl || nls == 0) {
    p = blockIdx.x / a.n_splits;
    split = blockIdx.x % a.n_splits;
  } else if ((int)blockIdx.x < n_problems * nls) {
    split = blockIdx.x / n_problems;
    p = blockIdx.x % n_problems;
  } else {
    const int l = blockIdx.x - n_problems * nls, nds = a.n_splits - nls;
    p = l / nds;
    split = nls + l % nds;
  }
  const bool local_cta = split < nls;
  const int h = p % a.n_kv_heads;
  const int blk = (p / a.n_kv_heads) % nblk;
  const int b = p / (a.n_kv_heads * nblk);
  const int rows = G * a.route_block;
  const int i_first = a.local_len - a.q_tokens + blk * a.route_block;  // local index of row 0's token
  const int i_max = i_first + a.route_block - 1;
  const int k = a.top_k;

  if (tid == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_barrier_init();
  }
  if (!local_cta) pdl_wait();  // the selection comes from the top-k
  if (tid < k && !local_cta) {
    const int j = a.sel[(int64_t)p * k + tid];  // a global index on a shard bank
    const int jl = j - a.doc_lo;
    int len = 0;
    long long base = 0;
    if (jl >= 0 && jl < a.n_docs) {
      len = a.doc_len[jl];
      base = a.sel_base ? (long long)a.sel_base[(int64_t)p * k + tid] : (long long)h * a.kv_rows + a.doc_row[jl];
    } else if (j < 0 || j >= a.n_docs_index) {
      atomicCAS(a.err, 0, kErrInvalidArg);
    }
    doc_len_s[tid] = len;
    doc_base_s[tid] = base;
  }
  __syncthreads();
  const int local_tiles = a.with_local ? (i_max + 1 + TILE - 1) / TILE : 0;
  if (tid == 0) {
    // A local CTA sees a list of local tiles only; a document CTA with splits of
    // its own for the local context sees the document tiles only.
    int acc = 0;
    for (int d = 0; d < k; ++d) {
      tile_start[d] = acc;
      acc += local_cta ? 0 : (doc_len_s[d] + TILE - 1) / TILE;
    }
    tile_start[k] = acc;
    tile_start[k + 1] = acc + (local_cta || nls == 0 ? local_tiles : 0);
  }
  __syncthreads();
  const int Tb = tile_start[k], T = tile_start[k + 1];
  int t0, t1;
  if (nls > 0) {
    const int s0 = local_cta ? split : split - nls, ns = local_cta ? nls : a.n_splits - nls;
    t0 = (int)(((long long)T * s0) / ns);
    t1 = (int)(((long long)T * (s0 + 1)) / ns);
  } else {
    // split boundaries in cost units: bank tiles cost 1, local tiles LOCAL_W
    constexpr int LW = MSA_DECODE_LOCAL_W;
    const long long cost = (long long)Tb + (long long)LW * (T - Tb);
    auto tile_at = [&](long long cpos) -> int {
      return cpos <= Tb ? (int)cpos : Tb + (int)((cpos - Tb + LW - 1) / LW);
    };
    t0 = tile_at((cost * split) / a.n_splits);
    t1 = tile_at((cost * (split + 1)) / a.n_splits);
  }
  const int ntiles = t1 - t0;

  if (warp == WARPS) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && ntiles > 0) {
      prefetch_tensormap(&tm_bk);
      prefetch_tensormap(&tm_bv);
      prefetch_tensormap(&tm_lk);
      prefetch_tensormap(&tm_lv);
      const uint64_t pol = l2_policy_evict_first();
      int hint = 0;
      int issued = 0;
      auto tile_coord = [&](const TileRef& tr, const CUtensorMap*& mk, const CUtensorMap*& mv, int& y) {
        if (tr.di < k) {
          mk = &tm_bk; mv = &tm_bv;
          y = (int)(doc_base_s[tr.di] + (long long)tr.tt * TILE);
        } else {
          mk = &tm_lk; mv = &tm_lv;
          y = (b * a.n_kv_heads + h) * a.local_len + tr.tt * TILE;
        }
      };
      for (int n = 0; n < ntiles; ++n) {
        int stage, use;
        slot_of<S>(n, stage, use);
        if (use > 0 && !mbar_wait_bounded(&empty[stage], (use - 1) & 1, a.err)) break;
        const TileRef tr = locate(tile_start, k, t0 + n, hint);
        hint = tr.di;
        const CUtensorMap *mk, *mv;
        int y;
        tile_coord(tr, mk, mv, y);
        uint8_t* kdst = ring + stage * S::STAGE_BYTES;
        uint8_t* vdst = kdst + S::TILE_BYTES;
        mbar_arrive_expect_tx(&full[stage], S::STAGE_BYTES);
#pragma unroll
        for (int bx = 0; bx < S::BOXES; ++bx) {
          tma_load_2d(kdst + bx * S::BOX_BYTES, mk, bx * 64, y, &full[stage], pol);
          tma_load_2d(vdst + bx * S::BOX_BYTES, mv, bx * 64, y, &full[stage], pol);
        }
        ++issued;
      }
      // No copy may still be landing when the CTA ends: wait for the last fill
      // of every slot (consumers normally have already).
      for (int n = max(0, issued - S::STAGES); n < issued; ++n) {
        int stage, use;
        slot_of<S>(n, stage, use);
        mbar_wait_bounded(&full[stage], use & 1, nullptr);
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int g = lane >> 2, c = lane & 3;
  // Query fragments (B operand of S^T = K Q^T): row 8*nt + g, dims
  // 16*ks + 2c + {0,1} and 16*ks + 8 + 2c + {0,1}; Global RoPE at k_off + i.
  uint32_t qf[D / 16][NT][2];
  int lim[NT][2];  // causal limit (local index) of this thread's two columns per n-tile
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int r = nt * 8 + 2 * c + e;
      lim[nt][e] = (r < rows) ? i_first + r / G : i_max;
    }
    const int r = nt * 8 + g;
    if (r < rows) {
      const int t = blk * a.route_block + r / G;
      const int hq = h * G + r % G;
      const int i = a.local_len - a.q_tokens + t;
      const uint16_t* qrow = a.q + (((int64_t)b * a.n_q_heads + hq) * a.q_tokens + t) * D;
      const float2* cs = a.gtab + (int64_t)i * (D / 2);
#pragma unroll
      for (int ks = 0; ks < D / 32; ++ks) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float xo[2], yo[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int d0 = 16 * ks + 8 * hf + 2 * c + e;
            const float x = __uint_as_float((uint32_t)qrow[d0] << 16);
            const float y = __uint_as_float((uint32_t)qrow[d0 + D / 2] << 16);
            const float2 t2 = __ldg(cs + d0);
            xo[e] = x * t2.x - y * t2.y;
            yo[e] = y * t2.x + x * t2.y;
          }
          qf[ks][nt][hf] = pack_bf16(xo[0], xo[1]);
          qf[ks + D / 32][nt][hf] = pack_bf16(yo[0], yo[1]);
        }
      }
    } else {
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) qf[ks][nt][0] = qf[ks][nt][1] = 0u;
    }
  }

  float m_run[NT][2], l_run[NT][2];
  float acc[D / 16][NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
    for (int md = 0; md < D / 16; ++md)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[md][nt][e] = 0.f;
  }

  // Global RoPE of a local tile: lane l rotates the 8 pairs of 16-byte chunk l % PC
  // (PC = D / 16 chunks per half row) of keys l / PC + STEP * i, STEP = 32 / PC.
  constexpr int kPairChunks = D / 16;
  constexpr int kStep = 32 / kPairChunks;
  const int rch = lane % kPairChunks, rr0 = lane / kPairChunks;
  int hint = 0;
  for (int n = warp; n < ntiles; n += WARPS) {
    int stage, use;
    slot_of<S>(n, stage, use);
    const TileRef tr = locate(tile_start, k, t0 + n, hint);
    hint = tr.di;
    const bool local = tr.di >= k;
    const int key0 = tr.tt * TILE;
    // the lane's first key's (cos, sin) from the table (fetched into L1 before the wait);
    // the later keys' by rotating STEP positions at a time (gstep)
    const float4* cs_src = reinterpret_cast<const float4*>(a.gtab + (int64_t)(key0 + rr0) * (D / 2) + rch * 8);
    if (local && key0 + rr0 < a.local_len) asm volatile("prefetch.global.L1 [%0];" ::"l"(cs_src));
    if (!mbar_wait_bounded(&full[stage], use & 1, a.err)) break;
    uint8_t* kt = ring + stage * S::STAGE_BYTES;
    uint8_t* vt = kt + S::TILE_BYTES;
    const int nvalid = local ? 0 : min(TILE, doc_len_s[tr.di] - key0);

    if (local) {
      // Global RoPE of the local keys, in shared memory: pair (i, i + D/2)
      // lives in the same swizzled slot of chunk i/8 and chunk (i + D/2)/8.
      float4 st[4], cs[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) st[j] = __ldg(reinterpret_cast<const float4*>(a.gstep + rch * 8) + j);
      if (key0 + rr0 < a.local_len) {
#pragma unroll
        for (int j = 0; j < 4; ++j) cs[j] = __ldg(cs_src + j);
      }
#pragma unroll 1
      for (int it = 0; it < TILE / kStep; ++it) {
        const int r = rr0 + kStep * it, ch = rch;
        const int u = key0 + r;
        if (u >= a.local_len) break;
        uint8_t* px;
        uint8_t* py;
        if constexpr (D == 128) {
          px = kt + swz128(r, ch);
          py = kt + S::BOX_BYTES + swz128(r, ch);
        } else {
          px = kt + swz128(r, ch);
          py = kt + swz128(r, ch + 4);
        }
        uint4 xv = *reinterpret_cast<uint4*>(px), yv = *reinterpret_cast<uint4*>(py);
        uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w}, ys[4] = {yv.x, yv.y, yv.z, yv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 t4 = cs[j];
          const float x0 = bf16_lo(xs[j]), x1 = bf16_hi(xs[j]);
          const float y0 = bf16_lo(ys[j]), y1 = bf16_hi(ys[j]);
          xs[j] = pack_bf16(x0 * t4.x - y0 * t4.y, x1 * t4.z - y1 * t4.w);
          ys[j] = pack_bf16(y0 * t4.x + x0 * t4.y, y1 * t4.z + x1 * t4.w);
          cs[j] = make_float4(t4.x * st[j].x - t4.y * st[j].y, t4.y * st[j].x + t4.x * st[j].y,
                              t4.z * st[j].z - t4.w * st[j].w, t4.w * st[j].z + t4.z * st[j].w);
        }
        *reinterpret_cast<uint4*>(px) = make_uint4(xs[0], xs[1], xs[2], xs[3]);
        *reinterpret_cast<uint4*>(py) = make_uint4(ys[0], ys[1], ys[2], ys[3]);
      }
      __syncwarp();
    }

    // ---- S^T = K Q^T : MT m-tiles of 16 keys x NT n-tiles of 8 rows; even and
    // odd k-steps accumulate separately (two short mma dependency chains).
    float s[MT][NT][4];
    const uint32_t kbase = smem_addr(kt);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      float s2[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[mt][nt][e] = s2[nt][e] = 0.f;
      const int row = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const int col = ks * 16 + (lane >> 4) * 8;
        const uint32_t addr = kbase + (col >> 6) * S::BOX_BYTES + swz128(row, (col & 63) >> 3);
        uint32_t af[4];
        ldmatrix_x4(af, addr);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (ks & 1) mma_bf16_16816(s2[nt], af, qf[ks][nt][0], qf[ks][nt][1]);
          else mma_bf16_16816(s[mt][nt], af, qf[ks][nt][0], qf[ks][nt][1]);
        }
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[mt][nt][e] += s2[nt][e];
    }

    // ---- mask, scale, online softmax (per column = query row)
    float alpha[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int kk = mt * 16 + g + hf * 8;
            const bool vis = local ? (key0 + kk <= lim[nt][e]) : (kk < nvalid);
            float v = s[mt][nt][hf * 2 + e] * a.scale_log2;
            v = vis ? v : -INFINITY;
            s[mt][nt][hf * 2 + e] = v;
            mx[e] = fmaxf(mx[e], v);
          }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 4));
        mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 8));
        mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 16));
        const float m_new = fmaxf(m_run[nt][e], mx[e]);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        alpha[nt][e] = exp2f(m_run[nt][e] - m_use);
        m_run[nt][e] = m_new;
        float sum = 0.f;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const float pv = exp2f(s[mt][nt][hf * 2 + e] - m_use);
            s[mt][nt][hf * 2 + e] = pv;
            sum += pv;
          }
        l_run[nt][e] = l_run[nt][e] * alpha[nt][e] + sum;
      }
#pragma unroll
      for (int md = 0; md < D / 16; ++md) {
        acc[md][nt][0] *= alpha[nt][0];
        acc[md][nt][1] *= alpha[nt][1];
        acc[md][nt][2] *= alpha[nt][0];
        acc[md][nt][3] *= alpha[nt][1];
      }
    }

    // ---- P^T fragments: transpose each 8x8 (keys x rows) block with movmatrix
    uint32_t pb[MT][NT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        pb[mt][nt][0] = movmatrix_trans(pack_bf16(s[mt][nt][0], s[mt][nt][1]));
        pb[mt][nt][1] = movmatrix_trans(pack_bf16(s[mt][nt][2], s[mt][nt][3]));
      }

    // ---- O^T += V^T P^T
    const uint32_t vbase = smem_addr(vt);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int key = mt * 16 + (lane & 7) + (lane >> 4) * 8;
#pragma unroll
      for (int md = 0; md < D / 16; ++md) {
        const int dim = md * 16 + ((lane >> 3) & 1) * 8;
        const uint32_t addr = vbase + (dim >> 6) * S::BOX_BYTES + swz128(key, (dim & 63) >> 3);
        uint32_t af[4];
        ldmatrix_x4_trans(af, addr);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[md][nt], af, pb[mt][nt][0], pb[mt][nt][1]);
      }
    }

    if (local) fence_proxy_async();  // generic writes above precede the next TMA into this stage
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
  }

  // ------------------------------------------------------------ CTA merge
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float v = l_run[nt][e];
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      l_run[nt][e] = v;
    }
  constexpr int CT = WARPS * 32;  // consumer threads
  named_barrier_sync(1, CT);      // every consumer is done reading the ring
  float* sc_o = reinterpret_cast<float*>(ring);            // [WARPS][R][D]
  float* sc_m = sc_o + WARPS * R * D;                      // [WARPS][R]
  float* sc_l = sc_m + WARPS * R;                          // [WARPS][R]
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int r = nt * 8 + 2 * c + e;
#pragma unroll
      for (int md = 0; md < D / 16; ++md) {
        sc_o[(warp * R + r) * D + md * 16 + g] = acc[md][nt][e];
        sc_o[(warp * R + r) * D + md * 16 + g + 8] = acc[md][nt][e + 2];
      }
      if (g == 0) {
        sc_m[warp * R + r] = m_run[nt][e];
        sc_l[warp * R + r] = l_run[nt][e];
      }
    }
  named_barrier_sync(1, CT);
  const int64_t slot = (int64_t)p * a.n_splits + split;
  for (int idx = tid; idx < rows * D; idx += CT) {
    const int r = idx / D, dim = idx % D;
    float mstar = -INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) mstar = fmaxf(mstar, sc_m[w * R + r]);
    float o = 0.f, l = 0.f;
    if (mstar != -INFINITY) {
#pragma unroll
      for (int w = 0; w < WARPS; ++w) {
        const float f = exp2f(sc_m[w * R + r] - mstar);
        o += f * sc_o[(w * R + r) * D + dim];
        l += f * sc_l[w * R + r];
      }
    }
    a.part_o[(slot * rows + r) * D + dim] = o;
    if (dim == 0) {
      a.part_ml[(slot * rows + r) * 2 + 0] = mstar;
      a.part_ml[(slot * rows + r) * 2 + 1] = l;
    }
  }

  // ------------------------------------------------------------ split merge
  // The last CTA of this problem to get here combines every split. Writers
  // fence before the counter bump; the last one fences before reading.
  __threadfence();
  named_barrier_sync(1, CT);
  if (tid == 0) {
    const unsigned old = atomicInc(reinterpret_cast<unsigned*>(a.counters + p), (unsigned)(a.n_splits - 1));
    *flag_s = (old == (unsigned)(a.n_splits - 1));
  }
  named_barrier_sync(1, CT);
  if (!*flag_s) return;
  __threadfence();
  const int nS = a.n_splits;
  // Every split's (m, l) of every row into shared memory at once (the ring is free by
  // now): one round of loads instead of two dependent chains of nS per row.
  const float2* pm = reinterpret_cast<const float2*>(a.part_ml) + (int64_t)p * nS * rows;
  float2* ml_s = reinterpret_cast<float2*>(ring);  // [nS][rows]
  for (int i = tid; i < nS * rows; i += CT) ml_s[i] = __ldcg(pm + i);
  named_barrier_sync(1, CT);
  for (int i = tid; i < rows; i += CT) {
    float M = -INFINITY;
    for (int sp = 0; sp < nS; ++sp) M = fmaxf(M, ml_s[sp * rows + i].x);
    float L = 0.f;
    for (int sp = 0; sp < nS; ++sp) {
      const float m = ml_s[sp * rows + i].x;
      const float f = (m == -INFINITY) ? 0.f : exp2f(m - M);
      wgt_s[sp * kRowsMax + i] = f;
      L += f * ml_s[sp * rows + i].y;
    }
    const float inv = (L > 0.f) ? 1.0f / L : 0.f;
    for (int sp = 0; sp < nS; ++sp) wgt_s[sp * kRowsMax + i] *= inv;
    if (a.lse_out)
      a.lse_out[((int64_t)b * a.n_q_heads + h * G + i % G) * a.q_tokens + blk * a.route_block + i / G] =
          L > 0.f ? (M + log2f(L)) * 0.693147180559945309f : -INFINITY;
  }
  named_barrier_sync(1, CT);
  // Outputs in items of 4 dims: a thread owns up to 4 items and keeps 4 splits x 4 items
  // of loads in flight; each output still sums the splits in order, split 0 first.
  constexpr int D4 = D / 4;
  const int n4 = rows * D4;
  const float4* po = reinterpret_cast<const float4*>(a.part_o) + (int64_t)p * nS * n4;
  for (int base = 0; base < n4; base += 4 * CT) {
    float4 o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) o[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sp0 = 0; sp0 < nS; sp0 += 4) {
      float4 x[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int item = base + j * CT + tid;
          x[u][j] = (sp0 + u < nS && item < n4) ? __ldcg(po + (int64_t)(sp0 + u) * n4 + item)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (sp0 + u >= nS) break;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int item = base + j * CT + tid;
          const float w = wgt_s[(sp0 + u) * kRowsMax + (item < n4 ? item / D4 : 0)];
          o[j].x += w * x[u][j].x;
          o[j].y += w * x[u][j].y;
          o[j].z += w * x[u][j].z;
          o[j].w += w * x[u][j].w;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int item = base + j * CT + tid;
      if (item >= n4) continue;
      const int r = item / D4, dim = (item % D4) * 4;
      const int t = blk * a.route_block + r / G;
      const int hq = h * G + r % G;
      float* dst = a.out + (((int64_t)b * a.n_q_heads + hq) * a.q_tokens + t) * D + dim;
      dst[0] = o[j].x;
      dst[1] = o[j].y;
      dst[2] = o[j].z;
      dst[3] = o[j].w;
    }
  }
}

template <class S, int NT>
cudaError_t launch_decode_t(const AttendArgs& a, const AttendMaps& m, cudaStream_t s) {
  auto kern = attend_decode_kernel<S, NT>;
  const size_t smem = smem_bytes<S>(NT);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int nblk = a.q_tokens / a.route_block;
  const long long ctas = (long long)a.n_splits * a.batch * nblk * a.n_kv_heads;
  if (ctas > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  return launch_maybe_pdl(kern, dim3((unsigned)ctas), dim3(S::THREADS), smem, s, a.pdl != 0, m.bank_k, m.bank_v,
                          m.loc_k, m.loc_v, a);
}

}  // namespace

int attend_tile_rows() { return Decode<128>::TILE; }
int attend_max_splits() { return kMaxSplits; }

int attend_ctas_per_sm(int head_dim) {
  const size_t per = head_dim == 128 ? smem_bytes<Decode<128>>(2) : smem_bytes<Decode<64>>(2);
  const size_t total = 227 * 1024;
  int n = (int)(total / (per + 1024));
  return n < 1 ? 1 : n;
}

cudaError_t launch_attend_decode(const AttendArgs& a, const AttendMaps& m, int head_dim, cudaStream_t s) {
  const int rows = (a.n_q_heads / a.n_kv_heads) * a.route_block;
  if (a.n_splits < 1 || a.n_splits > kMaxSplits || rows > kRowsMax) return cudaErrorInvalidValue;
  if (a.n_local_splits < 0 || a.n_local_splits >= a.n_splits || (a.n_local_splits > 0 && !a.with_local))
    return cudaErrorInvalidValue;
  if (head_dim == 128) {
    if (rows <= 8) return launch_decode_t<Decode<128>, 1>(a, m, s);
    return launch_decode_t<Decode<128>, 2>(a, m, s);
  }
  if (rows <= 8) return launch_decode_t<Decode<64>, 1>(a, m, s);
  return launch_decode_t<Decode<64>, 2>(a, m, s);
}

}  // namespace msa
