// Backward of sparse_attend for a fixed selection (top-k routing is not
// differentiated): gradients of sum(dO * O) with respect to the queries, the
// selected documents' keys and values and the local keys and values.
//   "MSA (Memory Sparse Attention)" (robocikowo.com), Komponenty (Memory Sparse
//   Attention Layer: trained end to end on the step's selection), Pułapki
//   implementacyjne (Global RoPE with a k-offset, Parallel RoPE of the bank).
//
// With s_j = q_rot . k_j / sqrt(d), p = softmax(s), O = sum_j p_j v_j:
//   dv_j = p_j dO,  dp_j = dO . v_j,  ds_j = p_j (dp_j - dO . O),
//   dq_rot = sum_j ds_j k_j / sqrt(d),  dk_j = ds_j q_rot / sqrt(d),
// and the rotated quantities go back through RoPE's adjoint (the turn by the
// negative angle).
//
// bwd_dq_kernel: a CTA owns 64 query rows of one problem (4 warps of 16 rows)
// and streams the problem's key list twice through a TMA ring. Pass 1 is the
// forward (online softmax and O) for each row's log-sum-exp and D = dO . O;
// pass 2 rebuilds P, forms dP = dO V^T and dS, and accumulates dQ += dS K, all
// with mma.sync m16n8k16 in the FlashAttention-2 register layout.
//
// bwd_dkdv_kernel: keys as M. A CTA owns a run of key tiles of one problem; it
// keeps the problem's RoPE'd queries and dO (bf16) in shared memory, and each of
// its 4 warps takes 16 keys of a 64-key tile: for every 16 rows it forms
// S^T = K Q^T, P^T, dP^T = V dO^T and dS^T, and accumulates dV += P^T dO and
// dK += dS^T Q. A tile's dK (turned back through the RoPE adjoint) and dV are
// added to the outputs with vector atomics, since the same document (and the
// same local context) serves several problems.
#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int BT = 64;               // keys per tile
constexpr int BW = 4;                // consumer warps of the dQ kernel (16 rows each)
constexpr int BROWS = BW * 16;       // rows per dQ CTA
constexpr int BSTAGES = 4;
constexpr int BMAX_TOPK = 64;
constexpr float kLn2 = 0.693147180559945309f;

template <int D>
struct BShape {
  static constexpr int BOXES = D / 64;
  static constexpr int BOX_BYTES = BT * 128;
  static constexpr int TILE_BYTES = BT * D * 2;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int RING_BYTES = BSTAGES * STAGE_BYTES;
  static constexpr size_t TAB_BYTES = (BMAX_TOPK + 2) * 4 + BMAX_TOPK * 4 + BMAX_TOPK * 8;
  static constexpr size_t SMEM = 1024 + RING_BYTES + 2 * BSTAGES * 8 + TAB_BYTES;
};

// The selected documents of problem p (length, first row in the K/V maps) and
// the tile list: the documents' tiles in selection order, then the local tiles
// up to local index i_max. Called by every thread of the CTA.
__device__ __forceinline__ int build_tiles(const AttendArgs& a, int p, int h, int i_max, int* tile_start,
                                           int* doc_len_s, long long* doc_base_s) {
  const int k = a.top_k;
  const int tid = threadIdx.x;
  if (tid < k) {
    const int j = a.sel[(int64_t)p * k + tid];
    int len = 0;
    long long base = 0;
    if (j >= 0 && j < a.n_docs) {
      len = a.doc_len[j];
      base = (long long)h * a.kv_rows + a.doc_row[j];
    } else {
      atomicCAS(a.err, 0, kErrInvalidArg);
    }
    doc_len_s[tid] = len;
    doc_base_s[tid] = base;
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int d = 0; d < k; ++d) {
      tile_start[d] = acc;
      acc += (doc_len_s[d] + BT - 1) / BT;
    }
    tile_start[k] = acc;
    tile_start[k + 1] = acc + (i_max + 1 + BT - 1) / BT;
  }
  __syncthreads();
  return tile_start[k + 1];
}

// Key tile n of the problem: first row in the K/V tensor maps; local tiles use
// the local maps. `di` is a cursor that only moves forward.
__device__ __forceinline__ int tile_row(const AttendArgs& a, int n, int b, int h, const int* tile_start,
                                        const long long* doc_base_s, int& di, bool& local) {
  while (di < a.top_k && n >= tile_start[di + 1]) ++di;
  local = di >= a.top_k;
  const int tt = n - tile_start[di];
  return local ? (b * a.n_kv_heads + h) * a.local_len + tt * BT : (int)(doc_base_s[di] + (long long)tt * BT);
}

template <int D>
__global__ void __launch_bounds__((BW + 1) * 32, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_bk, const __grid_constant__ CUtensorMap tm_bv,
                  const __grid_constant__ CUtensorMap tm_lk, const __grid_constant__ CUtensorMap tm_lv,
                  const AttendBwdArgs g) {
  using S = BShape<D>;
  const AttendArgs& a = g.a;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + S::RING_BYTES);
  uint64_t* empty = full + BSTAGES;
  int* tile_start = reinterpret_cast<int*>(empty + BSTAGES);
  int* doc_len_s = tile_start + BMAX_TOPK + 2;
  long long* doc_base_s = reinterpret_cast<long long*>(doc_len_s + BMAX_TOPK);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int p = blockIdx.y;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int nblk = a.q_tokens / a.route_block;
  const int h = p % a.n_kv_heads;
  const int blk = (p / a.n_kv_heads) % nblk;
  const int b = p / (a.n_kv_heads * nblk);
  const int rows = G * a.route_block;               // rows of the problem, ordered (head, token)
  const int row0 = blockIdx.x * BROWS;
  const int i_first = a.local_len - a.q_tokens + blk * a.route_block;
  const int r_end = min(row0 + BROWS, rows) - 1;
  const int i_max = i_first + (r_end / a.route_block != row0 / a.route_block ? a.route_block - 1
                                                                              : r_end % a.route_block);
  if (tid == 0) {
    for (int s = 0; s < BSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], BW);
    }
    fence_barrier_init();
  }
  const int T = build_tiles(a, p, h, i_max, tile_start, doc_len_s, doc_base_s);

  if (warp == BW) {
    // ------------------------------------------------------------ producer: the key list, twice
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_last();
      int di = 0, issued = 0;
      for (int n = 0; n < 2 * T; ++n) {
        if (n == T) di = 0;
        const int stage = n % BSTAGES, use = n / BSTAGES;
        if (use > 0 && !mbar_wait_bounded(&empty[stage], (use - 1) & 1, a.err)) break;
        bool local;
        const int y = tile_row(a, n % T, b, h, tile_start, doc_base_s, di, local);
        const CUtensorMap* mk = local ? &tm_lk : &tm_bk;
        const CUtensorMap* mv = local ? &tm_lv : &tm_bv;
        uint8_t* kdst = ring + stage * S::STAGE_BYTES;
        mbar_arrive_expect_tx(&full[stage], S::STAGE_BYTES);
#pragma unroll
        for (int bx = 0; bx < S::BOXES; ++bx) {
          tma_load_2d(kdst + bx * S::BOX_BYTES, mk, bx * 64, y, &full[stage], pol);
          tma_load_2d(kdst + S::TILE_BYTES + bx * S::BOX_BYTES, mv, bx * 64, y, &full[stage], pol);
        }
        ++issued;
      }
      for (int n = max(0, issued - BSTAGES); n < issued; ++n)
        mbar_wait_bounded(&full[n % BSTAGES], (n / BSTAGES) & 1, nullptr);
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int gq = lane >> 2, c = lane & 3;
  int lim[2], rr[2];
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    rr[hf] = min(row0 + 16 * warp + gq + 8 * hf, rows - 1);
    lim[hf] = i_first + rr[hf] % a.route_block;
  }
  const float* dorow[2];
  int64_t orow[2];
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int hq = h * G + rr[hf] / a.route_block;
    const int t = blk * a.route_block + rr[hf] % a.route_block;
    orow[hf] = ((int64_t)b * a.n_q_heads + hq) * a.q_tokens + t;
    dorow[hf] = g.dout + orow[hf] * D;
  }
  // A fragments of the RoPE'd queries (rows gq, gq + 8)
  uint32_t qa[D / 16][4];
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const uint16_t* qrow = g.q_rot + orow[hf] * D;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
      for (int half = 0; half < 2; ++half)
        qa[ks][hf + 2 * half] = *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 * half + 2 * c);
  }
  int warp_lim_max = max(lim[0], lim[1]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) warp_lim_max = max(warp_lim_max, __shfl_xor_sync(0xffffffffu, warp_lim_max, off));

  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float acc[D / 8][4];  // pass 1: O; pass 2: dQ (rotated)
#pragma unroll
  for (int nd = 0; nd < D / 8; ++nd) acc[nd][0] = acc[nd][1] = acc[nd][2] = acc[nd][3] = 0.f;
  uint32_t doa[D / 16][4];  // pass 2: A fragments of dO
  float lse2[2] = {0.f, 0.f}, drow[2] = {0.f, 0.f};
  const float inv_sqrt_d = a.scale_log2 * kLn2;

  int di = 0;
  for (int n = 0; n < 2 * T; ++n) {
    const bool pass2 = n >= T;
    if (n == T) {
      // ---- row statistics from pass 1, then the dO fragments for pass 2
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float l = l_run[hf];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        lse2[hf] = m_run[hf] + log2f(l);
        const float inv = l > 0.f ? 1.0f / l : 0.f;
        float dsum = 0.f;
#pragma unroll
        for (int nd = 0; nd < D / 8; ++nd) {
          const float2 dv = *reinterpret_cast<const float2*>(dorow[hf] + nd * 8 + 2 * c);
          dsum += (acc[nd][2 * hf] * dv.x + acc[nd][2 * hf + 1] * dv.y) * inv;
        }
        dsum += __shfl_xor_sync(0xffffffffu, dsum, 1);
        dsum += __shfl_xor_sync(0xffffffffu, dsum, 2);
        drow[hf] = dsum;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const float2 dv = *reinterpret_cast<const float2*>(dorow[hf] + 16 * ks + 8 * half + 2 * c);
            doa[ks][hf + 2 * half] = pack_bf16(dv.x, dv.y);
          }
      }
#pragma unroll
      for (int nd = 0; nd < D / 8; ++nd) acc[nd][0] = acc[nd][1] = acc[nd][2] = acc[nd][3] = 0.f;
      di = 0;
    }
    const int stage = n % BSTAGES, use = n / BSTAGES;
    if (!mbar_wait_bounded(&full[stage], use & 1, a.err)) break;
    const int tn = pass2 ? n - T : n;
    while (di < a.top_k && tn >= tile_start[di + 1]) ++di;
    const bool local = di >= a.top_k;
    const int key0 = (tn - tile_start[di]) * BT;
    const int nvalid = local ? BT : min(BT, doc_len_s[di] - key0);
    const bool skip = local && key0 > warp_lim_max;
    if (!skip) {
      const uint32_t kbase = smem_addr(ring + stage * S::STAGE_BYTES);
      const uint32_t vbase = kbase + S::TILE_BYTES;
      // ---- S = Q K^T
      float sc[BT / 8][4];
#pragma unroll
      for (int nt = 0; nt < BT / 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
        for (int np = 0; np < BT / 16; ++np) {
          const int mi = lane >> 3;
          const int key = 16 * np + (mi >> 1) * 8 + (lane & 7);
          const int dim = 16 * ks + (mi & 1) * 8;
          uint32_t bf[4];
          ldmatrix_x4(bf, kbase + (dim >> 6) * S::BOX_BYTES + swz128(key, (dim & 63) >> 3));
          mma_bf16_16816(sc[2 * np], qa[ks], bf[0], bf[1]);
          mma_bf16_16816(sc[2 * np + 1], qa[ks], bf[2], bf[3]);
        }
      // ---- mask and scale
#pragma unroll
      for (int nt = 0; nt < BT / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kk = nt * 8 + 2 * c + (e & 1);
          const int hf = e >> 1;
          const bool vis = local ? (key0 + kk <= lim[hf]) : (kk < nvalid);
          sc[nt][e] = vis ? sc[nt][e] * a.scale_log2 : -INFINITY;
        }
      if (!pass2) {
        // ---- online softmax and O += P V (the forward)
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < BT / 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) mx[e >> 1] = fmaxf(mx[e >> 1], sc[nt][e]);
        float alpha[2];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          mx[hf] = fmaxf(mx[hf], __shfl_xor_sync(0xffffffffu, mx[hf], 1));
          mx[hf] = fmaxf(mx[hf], __shfl_xor_sync(0xffffffffu, mx[hf], 2));
          const float m_new = fmaxf(m_run[hf], mx[hf]);
          const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
          alpha[hf] = exp2f(m_run[hf] - m_use);
          m_run[hf] = m_new;
          mx[hf] = m_use;
        }
        float sum[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < BT / 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float pv = exp2f(sc[nt][e] - mx[e >> 1]);
            sc[nt][e] = pv;
            sum[e >> 1] += pv;
          }
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) l_run[hf] = l_run[hf] * alpha[hf] + sum[hf];
#pragma unroll
        for (int nd = 0; nd < D / 8; ++nd) {
          acc[nd][0] *= alpha[0];
          acc[nd][1] *= alpha[0];
          acc[nd][2] *= alpha[1];
          acc[nd][3] *= alpha[1];
        }
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk) {
          uint32_t pa[4];
          pa[0] = pack_bf16(sc[2 * kk][0], sc[2 * kk][1]);
          pa[1] = pack_bf16(sc[2 * kk][2], sc[2 * kk][3]);
          pa[2] = pack_bf16(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
          pa[3] = pack_bf16(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
          for (int np = 0; np < D / 16; ++np) {
            const int mi = lane >> 3;
            const int key = 16 * kk + (mi & 1) * 8 + (lane & 7);
            const int dim = 16 * np + (mi >> 1) * 8;
            uint32_t bf[4];
            ldmatrix_x4_trans(bf, vbase + (dim >> 6) * S::BOX_BYTES + swz128(key, (dim & 63) >> 3));
            mma_bf16_16816(acc[2 * np], pa, bf[0], bf[1]);
            mma_bf16_16816(acc[2 * np + 1], pa, bf[2], bf[3]);
          }
        }
      } else {
        // ---- P from the row statistics; dP = dO V^T; dS = P (dP - D) / sqrt(d); dQ += dS K
        float dp[BT / 8][4];
#pragma unroll
        for (int nt = 0; nt < BT / 8; ++nt) dp[nt][0] = dp[nt][1] = dp[nt][2] = dp[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
          for (int np = 0; np < BT / 16; ++np) {
            const int mi = lane >> 3;
            const int key = 16 * np + (mi >> 1) * 8 + (lane & 7);
            const int dim = 16 * ks + (mi & 1) * 8;
            uint32_t bf[4];
            ldmatrix_x4(bf, vbase + (dim >> 6) * S::BOX_BYTES + swz128(key, (dim & 63) >> 3));
            mma_bf16_16816(dp[2 * np], doa[ks], bf[0], bf[1]);
            mma_bf16_16816(dp[2 * np + 1], doa[ks], bf[2], bf[3]);
          }
#pragma unroll
        for (int nt = 0; nt < BT / 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int hf = e >> 1;
            const float pv = exp2f(sc[nt][e] - lse2[hf]);  // 0 where masked
            sc[nt][e] = pv * (dp[nt][e] - drow[hf]) * inv_sqrt_d;
          }
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk) {
          uint32_t pa[4];
          pa[0] = pack_bf16(sc[2 * kk][0], sc[2 * kk][1]);
          pa[1] = pack_bf16(sc[2 * kk][2], sc[2 * kk][3]);
          pa[2] = pack_bf16(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
          pa[3] = pack_bf16(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
          for (int np = 0; np < D / 16; ++np) {
            const int mi = lane >> 3;
            const int key = 16 * kk + (mi & 1) * 8 + (lane & 7);
            const int dim = 16 * np + (mi >> 1) * 8;
            uint32_t bf[4];
            ldmatrix_x4_trans(bf, kbase + (dim >> 6) * S::BOX_BYTES + swz128(key, (dim & 63) >> 3));
            mma_bf16_16816(acc[2 * np], pa, bf[0], bf[1]);
            mma_bf16_16816(acc[2 * np + 1], pa, bf[2], bf[3]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
  }

  // ---- dQ through the Global-RoPE adjoint; the row statistics for the dK/dV kernel
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int r = row0 + 16 * warp + gq + 8 * hf;
    if (r >= rows) continue;
    const int i = i_first + r % a.route_block;
    const float2* cs = a.gtab + (int64_t)i * (D / 2);
    float* dst = g.dq + orow[hf] * D;
#pragma unroll
    for (int nd = 0; nd < D / 16; ++nd)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int d0 = nd * 8 + 2 * c + e;  // first-half dim; its partner is d0 + D/2 (fragment nd + D/16)
        const float2 t2 = __ldg(cs + d0);
        const float x = acc[nd][2 * hf + e], y = acc[nd + D / 16][2 * hf + e];
        dst[d0] = x * t2.x + y * t2.y;
        dst[d0 + D / 2] = y * t2.x - x * t2.y;
      }
    if (c == 0) {
      g.lse2[(int64_t)p * rows + r] = lse2[hf];
      g.drow[(int64_t)p * rows + r] = drow[hf];
    }
  }
}

constexpr int KW = 4;                // consumer warps of the dK/dV kernel (16 keys each)
constexpr int KSTAGES = 2;
constexpr int KROWS = 256;           // query rows per dK/dV CTA (a slice of the problem's rows)
constexpr int KGROUP = 16;           // key tiles per dK/dV CTA

template <int D>
struct KShape {
  static constexpr int BOXES = D / 64;
  static constexpr int BOX_BYTES = BT * 128;
  static constexpr int TILE_BYTES = BT * D * 2;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int RING_BYTES = KSTAGES * STAGE_BYTES;
  static constexpr int QBOX = KROWS * 128;          // one 64-dim box of the row slice
  static constexpr int QBYTES = KROWS * D * 2;      // RoPE'd queries (and, after them, dO) of the slice
  static constexpr size_t OFF_Q = RING_BYTES;
  static constexpr size_t OFF_DO = OFF_Q + QBYTES;
  static constexpr size_t OFF_ST = OFF_DO + QBYTES;  // lse2[KROWS], drow[KROWS], lim[KROWS]
  static constexpr size_t OFF_BAR = OFF_ST + 3 * KROWS * 4;
  static constexpr size_t OFF_TAB = OFF_BAR + 2 * KSTAGES * 8;
  static constexpr size_t SMEM = 1024 + OFF_TAB + BShape<D>::TAB_BYTES;
};

template <int D>
__global__ void __launch_bounds__((KW + 1) * 32, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_bk, const __grid_constant__ CUtensorMap tm_bv,
                    const __grid_constant__ CUtensorMap tm_lk, const __grid_constant__ CUtensorMap tm_lv,
                    const AttendBwdArgs g) {
  using S = KShape<D>;
  const AttendArgs& a = g.a;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  float* lse_s = reinterpret_cast<float*>(sm + S::OFF_ST);
  float* drow_s = lse_s + KROWS;
  int* lim_s = reinterpret_cast<int*>(drow_s + KROWS);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + S::OFF_BAR);
  uint64_t* empty = full + KSTAGES;
  int* tile_start = reinterpret_cast<int*>(sm + S::OFF_TAB);
  int* doc_len_s = tile_start + BMAX_TOPK + 2;
  long long* doc_base_s = reinterpret_cast<long long*>(doc_len_s + BMAX_TOPK);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int p = blockIdx.z;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int nblk = a.q_tokens / a.route_block;
  const int h = p % a.n_kv_heads;
  const int blk = (p / a.n_kv_heads) % nblk;
  const int b = p / (a.n_kv_heads * nblk);
  const int rows = G * a.route_block;
  const int r0 = blockIdx.y * KROWS;                 // this CTA's row slice [r0, r0 + nr)
  const int nr = min(KROWS, rows - r0);
  const int i_first = a.local_len - a.q_tokens + blk * a.route_block;
  // the latest local index any row of the problem reaches (the tile list is the problem's)
  const int i_max = i_first + a.route_block - 1;
  if (tid == 0) {
    for (int s = 0; s < KSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], KW);
    }
    fence_barrier_init();
  }
  const int T = build_tiles(a, p, h, i_max, tile_start, doc_len_s, doc_base_s);
  const int t0 = blockIdx.x * KGROUP, t1 = min(T, t0 + KGROUP);
  if (t0 >= t1 || nr <= 0) return;  // uniform over the CTA

  // ---- the slice's RoPE'd queries and dO (bf16) in 128-byte-swizzled boxes, and its row statistics
  for (int u = tid; u < KROWS * (D / 8); u += blockDim.x) {
    const int r = u / (D / 8), v = u % (D / 8);  // row, 16-byte group
    const uint32_t off = (v >> 3) * S::QBOX + swz128(r, v & 7);
    uint4 qv = make_uint4(0, 0, 0, 0), dv = make_uint4(0, 0, 0, 0);
    if (r < nr) {
      const int R = r0 + r;
      const int hq = h * G + R / a.route_block;
      const int t = blk * a.route_block + R % a.route_block;
      const int64_t orow = ((int64_t)b * a.n_q_heads + hq) * a.q_tokens + t;
      qv = *reinterpret_cast<const uint4*>(g.q_rot + orow * D + v * 8);
      const float4 d0 = *reinterpret_cast<const float4*>(g.dout + orow * D + v * 8);
      const float4 d1 = *reinterpret_cast<const float4*>(g.dout + orow * D + v * 8 + 4);
      dv = make_uint4(pack_bf16(d0.x, d0.y), pack_bf16(d0.z, d0.w), pack_bf16(d1.x, d1.y), pack_bf16(d1.z, d1.w));
    }
    *reinterpret_cast<uint4*>(sm + S::OFF_Q + off) = qv;
    *reinterpret_cast<uint4*>(sm + S::OFF_DO + off) = dv;
  }
  for (int r = tid; r < KROWS; r += blockDim.x) {
    const bool ok = r < nr;
    lse_s[r] = ok ? g.lse2[(int64_t)p * rows + r0 + r] : INFINITY;  // padding rows: P = 0
    drow_s[r] = ok ? g.drow[(int64_t)p * rows + r0 + r] : 0.f;
    lim_s[r] = ok ? i_first + (r0 + r) % a.route_block : -1;
  }
  __syncthreads();

  if (warp == KW) {
    // ------------------------------------------------------------ producer: tiles [t0, t1)
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int di = 0, issued = 0;
      for (int n = t0; n < t1; ++n) {
        const int q = n - t0, stage = q % KSTAGES, use = q / KSTAGES;
        if (use > 0 && !mbar_wait_bounded(&empty[stage], (use - 1) & 1, a.err)) break;
        bool local;
        const int y = tile_row(a, n, b, h, tile_start, doc_base_s, di, local);
        const CUtensorMap* mk = local ? &tm_lk : &tm_bk;
        const CUtensorMap* mv = local ? &tm_lv : &tm_bv;
        uint8_t* kdst = sm + stage * S::STAGE_BYTES;
        mbar_arrive_expect_tx(&full[stage], S::STAGE_BYTES);
#pragma unroll
        for (int bx = 0; bx < S::BOXES; ++bx) {
          tma_load_2d(kdst + bx * S::BOX_BYTES, mk, bx * 64, y, &full[stage], pol);
          tma_load_2d(kdst + S::TILE_BYTES + bx * S::BOX_BYTES, mv, bx * 64, y, &full[stage], pol);
        }
        ++issued;
      }
      for (int q = max(0, issued - KSTAGES); q < issued; ++q)
        mbar_wait_bounded(&full[q % KSTAGES], (q / KSTAGES) & 1, nullptr);
    }
    return;
  }

  // ------------------------------------------------------------ consumers: 16 keys per warp
  const int gq = lane >> 2, c = lane & 3, mi = lane >> 3;
  const uint32_t qs = smem_addr(sm + S::OFF_Q), dos = smem_addr(sm + S::OFF_DO);
  const float inv_sqrt_d = a.scale_log2 * kLn2;
  int di = 0;
  for (int n = t0; n < t1; ++n) {
    const int q = n - t0, stage = q % KSTAGES, use = q / KSTAGES;
    if (!mbar_wait_bounded(&full[stage], use & 1, a.err)) break;
    while (di < a.top_k && n >= tile_start[di + 1]) ++di;
    const bool local = di >= a.top_k;
    const int key0 = (n - tile_start[di]) * BT;
    const int nvalid = local ? min(BT, a.local_len - key0) : min(BT, doc_len_s[di] - key0);
    const uint32_t kbase = smem_addr(sm + stage * S::STAGE_BYTES);
    const uint32_t vbase = kbase + S::TILE_BYTES;
    float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd)
#pragma unroll
      for (int e = 0; e < 4; ++e) dk[nd][e] = dv[nd][e] = 0.f;
    // this warp's keys: kw + gq and kw + gq + 8 of the tile
    const int kw = 16 * warp;
    int kpos[2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) kpos[hf] = key0 + kw + gq + 8 * hf;  // local index (local tiles)
    for (int rc = 0; rc < nr; rc += 16) {
      // ---- S^T = K Q^T and dP^T = V dO^T for 16 keys x 16 rows
      float st[2][4], dpt[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) st[nt][e] = dpt[nt][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t ka[4], va[4], bq[4], bd[4];
        {
          const int key = kw + (lane & 15);
          const int dim = 16 * ks + (lane >> 4) * 8;
          const uint32_t o = (dim >> 6) * S::BOX_BYTES + swz128(key, (dim & 63) >> 3);
          ldmatrix_x4(ka, kbase + o);
          ldmatrix_x4(va, vbase + o);
        }
        {
          const int row = rc + (mi >> 1) * 8 + (lane & 7);
          const int dim = 16 * ks + (mi & 1) * 8;
          const uint32_t o = (dim >> 6) * S::QBOX + swz128(row, (dim & 63) >> 3);
          ldmatrix_x4(bq, qs + o);
          ldmatrix_x4(bd, dos + o);
        }
        mma_bf16_16816(st[0], ka, bq[0], bq[1]);
        mma_bf16_16816(st[1], ka, bq[2], bq[3]);
        mma_bf16_16816(dpt[0], va, bd[0], bd[1]);
        mma_bf16_16816(dpt[1], va, bd[2], bd[3]);
      }
      // ---- P^T and dS^T (element e: key kw + gq + 8 (e >> 1), row rc + 8 nt + 2 c + (e & 1))
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int row = rc + 8 * nt + 2 * c + (e & 1);
          const int kk = kw + gq + 8 * (e >> 1);
          const bool vis = (kk < nvalid) && (!local || key0 + kk <= lim_s[row]);
          const float pv = vis ? exp2f(st[nt][e] * a.scale_log2 - lse_s[row]) : 0.f;
          st[nt][e] = pv;
          dpt[nt][e] = pv * (dpt[nt][e] - drow_s[row]) * inv_sqrt_d;
        }
      // ---- dV += P^T dO and dK += dS^T Q (k = the 16 rows)
      uint32_t pa[4], sa[4];
      pa[0] = pack_bf16(st[0][0], st[0][1]);
      pa[1] = pack_bf16(st[0][2], st[0][3]);
      pa[2] = pack_bf16(st[1][0], st[1][1]);
      pa[3] = pack_bf16(st[1][2], st[1][3]);
      sa[0] = pack_bf16(dpt[0][0], dpt[0][1]);
      sa[1] = pack_bf16(dpt[0][2], dpt[0][3]);
      sa[2] = pack_bf16(dpt[1][0], dpt[1][1]);
      sa[3] = pack_bf16(dpt[1][2], dpt[1][3]);
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {
        const int row = rc + (mi & 1) * 8 + (lane & 7);
        const int dim = 16 * np + (mi >> 1) * 8;
        const uint32_t o = (dim >> 6) * S::QBOX + swz128(row, (dim & 63) >> 3);
        uint32_t bdo[4], bq[4];
        ldmatrix_x4_trans(bdo, dos + o);
        ldmatrix_x4_trans(bq, qs + o);
        mma_bf16_16816(dv[2 * np], pa, bdo[0], bdo[1]);
        mma_bf16_16816(dv[2 * np + 1], pa, bdo[2], bdo[3]);
        mma_bf16_16816(dk[2 * np], sa, bq[0], bq[1]);
        mma_bf16_16816(dk[2 * np + 1], sa, bq[2], bq[3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
    // ---- add this tile's dK (through the RoPE adjoint) and dV to the outputs
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int kk = kw + gq + 8 * hf;
      if (kk >= nvalid) continue;
      float* dkr;
      float* dvr;
      const float2* cs;
      if (local) {
        const int64_t row = ((int64_t)b * a.n_kv_heads + h) * a.local_len + key0 + kk;
        dkr = g.dk_loc + row * D;
        dvr = g.dv_loc + row * D;
        cs = a.gtab + (int64_t)(key0 + kk) * (D / 2);           // Global RoPE at k_off + u
      } else {
        const int64_t row = doc_base_s[di] + key0 + kk;       // h * kv_rows + document row
        dkr = g.dk_bank + row * D;
        dvr = g.dv_bank + row * D;
        cs = g.ptab + (int64_t)(key0 + kk) * (D / 2);          // Parallel RoPE at the position in the document
      }
#pragma unroll
      for (int nd = 0; nd < D / 16; ++nd) {
        const int d0 = nd * 8 + 2 * c;  // dims d0, d0 + 1 and their partners d0 + D/2, d0 + D/2 + 1
        const float2 ta = __ldg(cs + d0), tb = __ldg(cs + d0 + 1);
        const float x0 = dk[nd][2 * hf], x1 = dk[nd][2 * hf + 1];
        const float y0 = dk[nd + D / 16][2 * hf], y1 = dk[nd + D / 16][2 * hf + 1];
        atomicAdd(reinterpret_cast<float2*>(dkr + d0), make_float2(x0 * ta.x + y0 * ta.y, x1 * tb.x + y1 * tb.y));
        atomicAdd(reinterpret_cast<float2*>(dkr + d0 + D / 2),
                  make_float2(y0 * ta.x - x0 * ta.y, y1 * tb.x - x1 * tb.y));
        atomicAdd(reinterpret_cast<float2*>(dvr + d0), make_float2(dv[nd][2 * hf], dv[nd][2 * hf + 1]));
        atomicAdd(reinterpret_cast<float2*>(dvr + d0 + D / 2),
                  make_float2(dv[nd + D / 16][2 * hf], dv[nd + D / 16][2 * hf + 1]));
      }
    }
  }
}

template <int D>
cudaError_t launch_dq_t(const AttendBwdArgs& g, const AttendMaps& m, cudaStream_t s) {
  auto kern = bwd_dq_kernel<D>;
  const size_t smem = BShape<D>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const AttendArgs& a = g.a;
  const int nblk = a.q_tokens / a.route_block;
  const int rows = (a.n_q_heads / a.n_kv_heads) * a.route_block;
  dim3 grid((rows + BROWS - 1) / BROWS, a.batch * nblk * a.n_kv_heads);
  kern<<<grid, (BW + 1) * 32, smem, s>>>(m.bank_k, m.bank_v, m.loc_k, m.loc_v, g);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_dkdv_t(const AttendBwdArgs& g, const AttendMaps& m, int max_tiles, cudaStream_t s) {
  auto kern = bwd_dkdv_kernel<D>;
  const size_t smem = KShape<D>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const AttendArgs& a = g.a;
  const int nblk = a.q_tokens / a.route_block;
  const int rows = (a.n_q_heads / a.n_kv_heads) * a.route_block;
  dim3 grid((max_tiles + KGROUP - 1) / KGROUP, (rows + KROWS - 1) / KROWS, a.batch * nblk * a.n_kv_heads);
  kern<<<grid, (KW + 1) * 32, smem, s>>>(m.bank_k, m.bank_v, m.loc_k, m.loc_v, g);
  return cudaGetLastError();
}

}  // namespace

int attend_bwd_tile_rows() { return BT; }

cudaError_t launch_attend_bwd_dq(const AttendBwdArgs& g, const AttendMaps& m, int head_dim, cudaStream_t s) {
  if (head_dim == 128) return launch_dq_t<128>(g, m, s);
  return launch_dq_t<64>(g, m, s);
}

// max_tiles: an upper bound of any problem's tile count (CTAs past a problem's
// list return at once)
cudaError_t launch_attend_bwd_dkdv(const AttendBwdArgs& g, const AttendMaps& m, int head_dim, int max_tiles,
                                   cudaStream_t s) {
  if (head_dim == 128) return launch_dkdv_t<128>(g, m, max_tiles, s);
  return launch_dkdv_t<64>(g, m, max_tiles, s);
}

}  // namespace msa
