// sparse_attend (prefill): the same routed attention as attend_decode for
// problems with many query rows (G heads x Bq tokens > 16), e.g. 64-token
// routing blocks with 4 query heads per KV head = 256 rows.
//   "MSA (Memory Sparse Attention)" (robocikowo.com), Komponenty (Memory Sparse
//   Attention Layer), Pułapki implementacyjne (Global RoPE with a k-offset),
//   Paradygmat wykonania (only the k selected documents take part).
//
// Design: a CTA owns 128 query rows of one problem (sequence, routing block,
// KV head) -- 8 consumer warps of 16 rows -- and streams the problem's whole
// key list (selected documents' tiles, then the local tiles up to its last
// row's position) through a TMA ring that all consumer warps read (an empty
// barrier counts the 8 warps). Per 64-key tile each warp computes
// S = Q K^T and O += P V with mma.sync m16n8k16 in the FlashAttention-2
// register layout (the S accumulator fragments are the P operand fragments).
// The local keys arrive already turned by Global RoPE (rope_rows_kernel);
// queries are turned while their fragments are built.
#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int PT = 64;               // keys per tile
constexpr int PW = 8;                // consumer warps (16 rows each)
constexpr int PROWS = PW * 16;       // rows per CTA
constexpr int PSTAGES = 4;
constexpr int PMAX_TOPK = 64;

template <int D>
struct PShape {
  static constexpr int BOXES = D / 64;
  static constexpr int BOX_BYTES = PT * 128;
  static constexpr int TILE_BYTES = PT * D * 2;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int RING_BYTES = PSTAGES * STAGE_BYTES;
  static constexpr size_t SMEM = 1024 + RING_BYTES + 2 * PSTAGES * 8 + (PMAX_TOPK + 2) * 4 + PMAX_TOPK * 4 +
                                 PMAX_TOPK * 8;
};

// Global RoPE of a [rows, d] tensor into a workspace copy: row r sits at local
// index offset + r % period (local keys: period Lc, offset 0; queries: period
// Tq, offset Lc - Tq), i.e. at position k_off + that index.
__global__ void rope_rows_kernel(const uint16_t* __restrict__ lk, uint16_t* __restrict__ out,
                                 const float2* __restrict__ gtab, int64_t rows, int period, int offset, int d) {
  const int half_vecs = d / 16;  // 16-byte vectors per half row
  const int64_t unit = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (unit >= rows * half_vecs) return;
  const int64_t row = unit / half_vecs;
  const int vec = (int)(unit % half_vecs);
  const int u = offset + (int)(row % period);
  const uint4 x = *reinterpret_cast<const uint4*>(lk + row * d + vec * 8);
  const uint4 y = *reinterpret_cast<const uint4*>(lk + row * d + d / 2 + vec * 8);
  const float4* cs = reinterpret_cast<const float4*>(gtab + (int64_t)u * (d / 2) + vec * 8);
  uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 t = __ldg(cs + j);
    const float x0 = bf16_lo(xs[j]), x1 = bf16_hi(xs[j]);
    const float y0 = bf16_lo(ys[j]), y1 = bf16_hi(ys[j]);
    xs[j] = pack_bf16(x0 * t.x - y0 * t.y, x1 * t.z - y1 * t.w);
    ys[j] = pack_bf16(y0 * t.x + x0 * t.y, y1 * t.z + x1 * t.w);
  }
  *reinterpret_cast<uint4*>(out + row * d + vec * 8) = make_uint4(xs[0], xs[1], xs[2], xs[3]);
  *reinterpret_cast<uint4*>(out + row * d + d / 2 + vec * 8) = make_uint4(ys[0], ys[1], ys[2], ys[3]);
}

template <int D>
__global__ void __launch_bounds__((PW + 1) * 32, 1)
    attend_prefill_kernel(const __grid_constant__ CUtensorMap tm_bk, const __grid_constant__ CUtensorMap tm_bv,
                          const __grid_constant__ CUtensorMap tm_lk, const __grid_constant__ CUtensorMap tm_lv,
                          const AttendArgs a) {
  using S = PShape<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + S::RING_BYTES);
  uint64_t* empty = full + PSTAGES;
  int* tile_start = reinterpret_cast<int*>(empty + PSTAGES);
  int* doc_len_s = tile_start + PMAX_TOPK + 2;
  long long* doc_base_s = reinterpret_cast<long long*>(doc_len_s + PMAX_TOPK);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int p = blockIdx.y;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int nblk = a.q_tokens / a.route_block;
  const int h = p % a.n_kv_heads;
  const int blk = (p / a.n_kv_heads) % nblk;
  const int b = p / (a.n_kv_heads * nblk);
  const int rows = G * a.route_block;               // rows of the problem, ordered (head, token)
  const int row0 = blockIdx.x * PROWS;              // this CTA's first row
  const int i_first = a.local_len - a.q_tokens + blk * a.route_block;
  // rows are ordered (head, token): the CTA's latest token is the block's last
  // one if its row range crosses a head boundary, else that of its last row
  const int r_end = min(row0 + PROWS, rows) - 1;
  const int i_max = i_first + (r_end / a.route_block != row0 / a.route_block ? a.route_block - 1
                                                                              : r_end % a.route_block);
  const int k = a.top_k;

  if (tid < k) {
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
  if (tid == 0) {
    for (int s = 0; s < PSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], PW);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int d = 0; d < k; ++d) {
      tile_start[d] = acc;
      acc += (doc_len_s[d] + PT - 1) / PT;
    }
    tile_start[k] = acc;
    tile_start[k + 1] = acc + (a.with_local ? (i_max + 1 + PT - 1) / PT : 0);
  }
  __syncthreads();
  const int T = tile_start[k + 1];

  if (warp == PW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_bk);
      prefetch_tensormap(&tm_bv);
      prefetch_tensormap(&tm_lk);
      prefetch_tensormap(&tm_lv);
      const uint64_t pol = l2_policy_evict_last();  // the other CTAs of this problem re-read these tiles
      int di = 0, issued = 0;
      for (int n = 0; n < T; ++n) {
        const int stage = n % PSTAGES, use = n / PSTAGES;
        if (use > 0 && !mbar_wait_bounded(&empty[stage], (use - 1) & 1, a.err)) break;
        while (di < k && n >= tile_start[di + 1]) ++di;
        const int tt = n - tile_start[di];
        const CUtensorMap *mk, *mv;
        int y;
        if (di < k) {
          mk = &tm_bk; mv = &tm_bv;
          y = (int)(doc_base_s[di] + (long long)tt * PT);
        } else {
          mk = &tm_lk; mv = &tm_lv;
          y = (b * a.n_kv_heads + h) * a.local_len + tt * PT;
        }
        uint8_t* kdst = ring + stage * S::STAGE_BYTES;
        mbar_arrive_expect_tx(&full[stage], S::STAGE_BYTES);
#pragma unroll
        for (int bx = 0; bx < S::BOXES; ++bx) {
          tma_load_2d(kdst + bx * S::BOX_BYTES, mk, bx * 64, y, &full[stage], pol);
          tma_load_2d(kdst + S::TILE_BYTES + bx * S::BOX_BYTES, mv, bx * 64, y, &full[stage], pol);
        }
        ++issued;
      }
      for (int n = max(0, issued - PSTAGES); n < issued; ++n)
        mbar_wait_bounded(&full[n % PSTAGES], (n / PSTAGES) & 1, nullptr);
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int g = lane >> 2, c = lane & 3;
  // rows of this warp: row0 + 16*warp + {g, g+8}; row -> (head hq, token t)
  int lim[2];
  uint32_t qa[D / 16][4];  // A fragments of Q (rows g, g+8; dims 16ks + 2c.., +8)
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int r = min(row0 + 16 * warp + g + 8 * hf, rows - 1);
    lim[hf] = i_first + r % a.route_block;
  }
  {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int r = min(row0 + 16 * warp + g + 8 * hf, rows - 1);
      const int hq = h * G + r / a.route_block;
      const int t = blk * a.route_block + r % a.route_block;
      const int i = a.local_len - a.q_tokens + t;
      const uint16_t* qrow = a.q + (((int64_t)b * a.n_q_heads + hq) * a.q_tokens + t) * D;
      const float2* cs = a.gtab + (int64_t)i * (D / 2);
#pragma unroll
      for (int ks = 0; ks < D / 32; ++ks) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float xo[2], yo[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int d0 = 16 * ks + 8 * half + 2 * c + e;
            const float x = __uint_as_float((uint32_t)qrow[d0] << 16);
            const float y = __uint_as_float((uint32_t)qrow[d0 + D / 2] << 16);
            const float2 t2 = __ldg(cs + d0);
            xo[e] = x * t2.x - y * t2.y;
            yo[e] = y * t2.x + x * t2.y;
          }
          // a[0]: row g, cols 0-7; a[1]: row g+8, cols 0-7; a[2]: row g, cols 8-15; a[3]: row g+8, cols 8-15
          qa[ks][hf + 2 * half] = pack_bf16(xo[0], xo[1]);
          qa[ks + D / 32][hf + 2 * half] = pack_bf16(yo[0], yo[1]);
        }
      }
    }
  }

  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float o[D / 8][4];
#pragma unroll
  for (int nd = 0; nd < D / 8; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
  // largest causal limit over the warp's 16 rows (warp-uniform: it gates mma.sync)
  int warp_lim_max = max(lim[0], lim[1]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) warp_lim_max = max(warp_lim_max, __shfl_xor_sync(0xffffffffu, warp_lim_max, off));

  int di = 0;
  for (int n = 0; n < T; ++n) {
    const int stage = n % PSTAGES, use = n / PSTAGES;
    if (!mbar_wait_bounded(&full[stage], use & 1, a.err)) break;
    while (di < k && n >= tile_start[di + 1]) ++di;
    const bool local = di >= k;
    const int key0 = (n - tile_start[di]) * PT;
    const int nvalid = local ? PT : min(PT, doc_len_s[di] - key0);
    // a local tile entirely past every row of this warp contributes nothing
    const bool skip = local && key0 > warp_lim_max;
    if (!skip) {
      const uint32_t kbase = smem_addr(ring + stage * S::STAGE_BYTES);
      const uint32_t vbase = kbase + S::TILE_BYTES;
      // ---- S = Q K^T: 8 n-tiles of 8 keys
      float sc[PT / 8][4];
#pragma unroll
      for (int nt = 0; nt < PT / 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
        for (int np = 0; np < PT / 16; ++np) {  // pairs of n-tiles per ldmatrix.x4
          const int mi = lane >> 3;
          const int key = 16 * np + (mi >> 1) * 8 + (lane & 7);
          const int dim = 16 * ks + (mi & 1) * 8;
          uint32_t bf[4];
          ldmatrix_x4(bf, kbase + (dim >> 6) * S::BOX_BYTES + swz128(key, (dim & 63) >> 3));
          mma_bf16_16816(sc[2 * np], qa[ks], bf[0], bf[1]);
          mma_bf16_16816(sc[2 * np + 1], qa[ks], bf[2], bf[3]);
        }
      }
      // ---- mask, scale, online softmax (rows g and g+8)
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < PT / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kk = nt * 8 + 2 * c + (e & 1);
          const int hf = e >> 1;
          const bool vis = local ? (key0 + kk <= lim[hf]) : (kk < nvalid);
          const float v = vis ? sc[nt][e] * a.scale_log2 : -INFINITY;
          sc[nt][e] = v;
          mx[hf] = fmaxf(mx[hf], v);
        }
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
      for (int nt = 0; nt < PT / 8; ++nt)
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
        o[nd][0] *= alpha[0];
        o[nd][1] *= alpha[0];
        o[nd][2] *= alpha[1];
        o[nd][3] *= alpha[1];
      }
      // ---- O += P V: 4 k-steps of 16 keys, D/8 n-tiles of 8 dims
#pragma unroll
      for (int kk = 0; kk < PT / 16; ++kk) {
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
          mma_bf16_16816(o[2 * np], pa, bf[0], bf[1]);
          mma_bf16_16816(o[2 * np + 1], pa, bf[2], bf[3]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
  }

  // ---- normalise and store: rows g (o[..][0,1]) and g+8 (o[..][2,3])
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    float l = l_run[hf];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const float inv = l > 0.f ? 1.0f / l : 0.f;
    const int r = row0 + 16 * warp + g + 8 * hf;
    if (r >= rows) continue;
    const int hq = h * G + r / a.route_block;
    const int t = blk * a.route_block + r % a.route_block;
    if (a.lse_out && c == 0)
      a.lse_out[((int64_t)b * a.n_q_heads + hq) * a.q_tokens + t] =
          l > 0.f ? (m_run[hf] + log2f(l)) * 0.693147180559945309f : -INFINITY;
    float* dst = a.out + (((int64_t)b * a.n_q_heads + hq) * a.q_tokens + t) * D;
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd)
      *reinterpret_cast<float2*>(dst + nd * 8 + 2 * c) = make_float2(o[nd][2 * hf] * inv, o[nd][2 * hf + 1] * inv);
  }
}

template <int D>
cudaError_t launch_prefill_t(const AttendArgs& a, const AttendMaps& m, cudaStream_t s) {
  auto kern = attend_prefill_kernel<D>;
  const size_t smem = PShape<D>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int nblk = a.q_tokens / a.route_block;
  const int rows = (a.n_q_heads / a.n_kv_heads) * a.route_block;
  dim3 grid((rows + PROWS - 1) / PROWS, a.batch * nblk * a.n_kv_heads);
  kern<<<grid, (PW + 1) * 32, smem, s>>>(m.bank_k, m.bank_v, m.loc_k, m.loc_v, a);
  return cudaGetLastError();
}

}  // namespace

int attend_prefill_tile_rows() { return PT; }

cudaError_t launch_rope_rows(const uint16_t* in, uint16_t* out, const float2* gtab, int64_t rows, int period,
                             int offset, int head_dim, cudaStream_t s) {
  const int64_t units = rows * (head_dim / 16);
  const int blocks = (int)((units + 255) / 256);
  rope_rows_kernel<<<blocks, 256, 0, s>>>(in, out, gtab, rows, period, offset, head_dim);
  return cudaGetLastError();
}

cudaError_t launch_attend_prefill(const AttendArgs& a, const AttendMaps& m, int head_dim, cudaStream_t s) {
  if (head_dim == 128) return launch_prefill_t<128>(a, m, s);
  return launch_prefill_t<64>(a, m, s);
}

}  // namespace msa
