// sparse_attend (prefill) on the 5th-generation tensor cores: tcgen05.mma with
// accumulators in tensor memory (TMEM), operands staged by TMA.
//   "MSA (Memory Sparse Attention)" (robocikowo.com), Komponenty (Memory Sparse
//   Attention Layer), Pułapki implementacyjne (Global RoPE with a k-offset),
//   Paradygmat wykonania (only the k selected documents take part).
//
// One CTA owns 128 query rows of one problem (sequence, 64- or 128-token
// routing block, KV head; rows ordered head-major) and walks the problem's key
// list in tiles of 128 keys: the selected documents' tiles, then the local
// tiles up to its last row's position.
//   warp 0     TMA producer: the query tile once (queries pre-turned by Global
//              RoPE), then K and V tiles into two separate 3-slot rings, in
//              the order K_0, K_1, V_0, K_2, V_1, ...: a K slot frees as soon
//              as its S MMA completes, a V slot only after its P V, so the
//              loads of the next keys never wait behind the softmax.
//   warp 1     allocates 512 TMEM columns; one lane issues, per tile j,
//              S_j = Q K_j^T (M = N = K = 128, into one of two S buffers, once
//              both P V of tile j-2, which read P over that buffer, completed)
//              and then, for tile j-1, O_0 += P_0 V[0:64) and O_1 += P_1
//              V[64:128) (P read from TMEM as the A operand, V from shared
//              memory as an MN-major operand), each as soon as its warpgroup
//              has written P; every group is committed to an mbarrier.
//   warps 2-9  softmax, two warpgroups; warpgroup h owns keys [64 h, 64 h + 64)
//              of every tile and keeps, per row (TMEM lane = row), its own
//              reference max, running sum and output accumulator O_h over
//              those keys, so the two never wait for each other inside the
//              key loop. Each thread reads its 64 S values with tcgen05.ld,
//              masks (document tails, causal local keys), and writes
//              P = exp2(S * scale - m) as packed bf16 pairs over the S columns
//              it has just read. m moves only when the half-row max rises by
//              more than 2^8; then the row of O_h is rescaled in TMEM (after
//              the previous P V into it). At the end the two halves' (m, l, O)
//              are merged per row -- exact, as a softmax over the union of
//              two key sets -- and each warpgroup writes 64 of the 128 dims.
// Every mbarrier parity wait targets the phase right after one the same waiter
// saw complete, so no wait can be satisfied by an older phase.
#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int TN = 128;               // keys per tile
constexpr int TM = 128;               // query rows per CTA
constexpr int TD = 128;               // head dim
constexpr int TMEM_COLS = 512;        // S0 [0,128) S1 [128,256) O_0 [256,384) O_1 [384,512)
constexpr int O_COL = 256;            // O_h = O_COL + 128 h
constexpr int NSLOT = 3;              // depth of the K ring and of the V ring
constexpr int THREADS = 320;           // producer, MMA, 8 softmax warps
constexpr int BOX = TN * 128;         // one 64-element-wide box of a 128-row tile (16 KB)
constexpr int TILE = 2 * BOX;         // 128 x 128 bf16 (32 KB)
constexpr int TOPK_MAX = 64;
constexpr float kLazy = 8.0f;         // rescale O only when a row max grows by more than 2^8
#ifndef MSA_PF_POLY
#define MSA_PF_POLY 1                 // of every 4 key pairs, how many take exp2 on the FMA pipe
#endif
constexpr int kPolyPairs = MSA_PF_POLY;
#ifndef MSA_PF_OPTIMISTIC
#define MSA_PF_OPTIMISTIC 1
#endif
// Full half-tiles skip the row-max pass: P is taken against the current
// reference max and the tile is kept while every P stays below 2^64 (bf16 and
// the fp32 accumulators hold such values with their full relative precision);
// otherwise, and for the first and the masked tiles, the exact path runs.
constexpr bool kOptimistic = MSA_PF_OPTIMISTIC != 0;
#ifndef MSA_PF_FAST_POLY
#define MSA_PF_FAST_POLY 0            // of every 4 key pairs of the fast path, how many take the polynomial
#endif
constexpr int kFastPoly = MSA_PF_FAST_POLY;
#ifndef MSA_PF_PMAX
#define MSA_PF_PMAX 18446744073709551616.f  // 2^64
#endif
constexpr float kPMax = MSA_PF_PMAX;

// max(a, b, c) in one instruction.
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// shared memory layout (offsets from a 1 KiB-aligned base)
constexpr int OFF_Q = 0;
constexpr int OFF_K0 = OFF_Q + TILE;              // K[s] = OFF_K0 + s * TILE
constexpr int OFF_V0 = OFF_K0 + NSLOT * TILE;     // V[s] = OFF_V0 + s * TILE
constexpr int OFF_BAR = OFF_V0 + NSLOT * TILE;
constexpr int N_BAR = 12 + 4 * NSLOT;
constexpr int OFF_TMEM = OFF_BAR + N_BAR * 8;
constexpr int OFF_TAB = OFF_TMEM + 16;
constexpr size_t SMEM_BYTES = 1024 + OFF_TAB + (TOPK_MAX + 2) * 4 + TOPK_MAX * 4 + TOPK_MAX * 8;
static_assert(SMEM_BYTES <= 232448, "shared memory");

__global__ void __launch_bounds__(THREADS, 1)
    attend_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_bk,
                             const __grid_constant__ CUtensorMap tm_bv, const __grid_constant__ CUtensorMap tm_lk,
                             const __grid_constant__ CUtensorMap tm_lv, const AttendArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* s_full = bars + 1;     // [buffer]
  uint64_t* s_free = bars + 3;     // [buffer]  both P V that read P over the buffer completed
  uint64_t* p_full = bars + 5;     // [warpgroup * 2 + buffer]  one arrival per warp of the warpgroup
  uint64_t* pv_done = bars + 9;    // [warpgroup]  one phase per tile
  uint64_t* o_done = bars + 11;    // one phase: every MMA of the CTA has completed
  uint64_t* k_full = bars + 12;    // [NSLOT] each
  uint64_t* k_empty = k_full + NSLOT;
  uint64_t* v_full = k_empty + NSLOT;
  uint64_t* v_empty = v_full + NSLOT;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
  int* abort_s = reinterpret_cast<int*>(sm + OFF_TMEM + 4);   // set when a wait expired: softmax warps stop together

  int* tile_start = reinterpret_cast<int*>(sm + OFF_TAB);
  int* doc_len_s = tile_start + TOPK_MAX + 2;
  long long* doc_base_s = reinterpret_cast<long long*>(doc_len_s + TOPK_MAX);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int p = blockIdx.y;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int Bq = a.route_block;
  const int nblk = a.q_tokens / Bq;
  const int h = p % a.n_kv_heads;
  const int blk = (p / a.n_kv_heads) % nblk;
  const int b = p / (a.n_kv_heads * nblk);
  const int row0 = blockIdx.x * TM;  // rows ordered (head, token); 128 | G * Bq
  const int i_first = a.local_len - a.q_tokens + blk * Bq;
  const int r_end = row0 + TM - 1;
  const int i_max = i_first + (r_end / Bq != row0 / Bq ? Bq - 1 : r_end % Bq);
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
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int d = 0; d < k; ++d) {
      tile_start[d] = acc;
      acc += (doc_len_s[d] + TN - 1) / TN;
    }
    tile_start[k] = acc;
    tile_start[k + 1] = acc + (a.with_local ? (i_max + 1 + TN - 1) / TN : 0);
  }
  __syncthreads();
  const int T = tile_start[k + 1];
  if (T == 0) {
    // no key of this CTA's rows lives here (a shard without the local context and
    // without any of the problem's selected documents): softmax over nothing
    for (int idx = tid; idx < TM * TD; idx += THREADS) {
      const int R = row0 + idx / TD;
      const int hq = h * G + R / Bq;
      const int t = blk * Bq + R % Bq;
      const int64_t orow = ((int64_t)b * a.n_q_heads + hq) * a.q_tokens + t;
      a.out[orow * TD + idx % TD] = 0.f;
      if (a.lse_out && idx % TD == 0) a.lse_out[orow] = -INFINITY;
    }
    return;
  }
  if (tid == 0) {
    // p_full collects one arrival per warp of a warpgroup; the rest one arrival each
    for (int i = 0; i < N_BAR; ++i) mbar_init(&bars[i], (i >= 5 && i <= 8) ? 4 : 1);
    fence_barrier_init();
    *abort_s = 0;
  }
  if (warp == 1) tmem_alloc(tmem_base_s, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_s;
  const uint32_t sbase = smem_addr(sm);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_bk);
      prefetch_tensormap(&tm_bv);
      prefetch_tensormap(&tm_lk);
      prefetch_tensormap(&tm_lv);
      const uint64_t pol = l2_policy_evict_last();  // the problem's other CTAs read the same tiles
      // query tile: two 64-row segments x two 64-dim boxes
      mbar_arrive_expect_tx(q_full, TILE);
#pragma unroll
      for (int sg = 0; sg < 2; ++sg) {
        const int r = row0 + 64 * sg;
        const int hq = h * G + r / Bq;
        const int y = (int)(((int64_t)b * a.n_q_heads + hq) * a.q_tokens + (int64_t)blk * Bq + r % Bq);
#pragma unroll
        for (int dh = 0; dh < 2; ++dh)
          tma_load_2d(sm + OFF_Q + dh * BOX + sg * (64 * 128), &tm_q, dh * 64, y, q_full, pol);
      }
      // key tile n -> (tensor map pair, first row); tiles are visited in order, so
      // one cursor per ring suffices
      auto coord = [&](int n, int& di, bool& local) -> int {
        while (di < k && n >= tile_start[di + 1]) ++di;
        local = di >= k;
        const int tt = n - tile_start[di];
        return local ? (b * a.n_kv_heads + h) * a.local_len + tt * TN : (int)(doc_base_s[di] + (long long)tt * TN);
      };
      int dk = 0, dv = 0;
      auto load = [&](int n, bool is_v, int& di) -> bool {
        const int st = n % NSLOT, use = n / NSLOT;
        uint64_t* empty = is_v ? v_empty : k_empty;
        uint64_t* full = is_v ? v_full : k_full;
        if (use > 0 && !mbar_wait_bounded(&empty[st], (use - 1) & 1, a.err)) return false;
        bool local;
        const int y = coord(n, di, local);
        const CUtensorMap* m = is_v ? (local ? &tm_lv : &tm_bv) : (local ? &tm_lk : &tm_bk);
        uint8_t* dst = sm + (is_v ? OFF_V0 : OFF_K0) + st * TILE;
        mbar_arrive_expect_tx(&full[st], TILE);
        tma_load_2d(dst, m, 0, y, &full[st], pol);
        tma_load_2d(dst + BOX, m, 64, y, &full[st], pol);
        return true;
      };
      // K runs one tile ahead of V: K_n is needed for S_n, V_n only after the softmax of tile n
      bool ok = true;
      for (int n = 0; ok && n <= T; ++n) {
        if (n < T) ok = load(n, false, dk);
        if (ok && n >= 1) ok = load(n - 1, true, dv);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = umma_idesc_bf16(TM, TN, false);
      const uint32_t idesc_pv = umma_idesc_bf16(TM, TD, true);
      bool ok = mbar_wait_bounded(q_full, 0, a.err);
      const uint64_t qdesc = umma_desc_sw128(sbase + OFF_Q, 16, 1024);
      const uint64_t kdesc0 = umma_desc_sw128(sbase + OFF_K0, 16, 1024);
      // O_h += P_h V_i[64 h, 64 h + 64) for both warpgroups h of tile i
      auto issue_pv = [&](int i) -> bool {
        if (!mbar_wait_bounded(&v_full[i % NSLOT], (i / NSLOT) & 1, a.err)) return false;
        const uint32_t vb = sbase + OFF_V0 + (i % NSLOT) * TILE;
        const uint64_t vdesc = umma_desc_sw128(vb, BOX, 1024);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait_bounded(&p_full[h * 2 + (i & 1)], (i >> 1) & 1, a.err)) return false;
          tc_fence_after();
          const uint32_t pt = tmem + (i & 1) * TN + h * (TN / 2);  // P_h over S_h's first 32 columns
#pragma unroll
          for (int kk = 0; kk < TN / 32; ++kk) {
            const uint64_t bd = vdesc + (uint64_t)(((h * 4 + kk) * 2048) >> 4);
            umma_bf16_ts(tmem + O_COL + h * TD, pt + kk * 8, bd, idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&pv_done[h]);
        }
        umma_commit(&v_empty[i % NSLOT]);
        umma_commit(&s_free[i & 1]);
        return true;
      };
      for (int j = 0; ok && j < T; ++j) {
        const int st = j % NSLOT;
        if (!mbar_wait_bounded(&k_full[st], (j / NSLOT) & 1, a.err)) break;
        if (j >= 2 && !mbar_wait_bounded(&s_free[j & 1], ((j - 2) >> 1) & 1, a.err)) break;
        tc_fence_after();
        // shared memory addresses stay below 2^18, so the 14-bit start field
        // of a descriptor never carries: offsets add to it directly
        const uint64_t kdesc = kdesc0 + (uint64_t)((st * TILE) >> 4);
#pragma unroll
        for (int ks = 0; ks < TD / 16; ++ks) {
          const uint32_t off = (ks >> 2) * BOX + (ks & 3) * 32;
          umma_bf16_ss(tmem + (j & 1) * TN, qdesc + (uint64_t)(off >> 4), kdesc + (uint64_t)(off >> 4),
                       idesc_qk, ks > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[j & 1]);
        umma_commit(&k_empty[st]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && T > 0 && issue_pv(T - 1)) umma_commit(o_done);
    }
  } else {
    // ------------------------------------------------------------ softmax
    // warps 2..9 = two warpgroups; warpgroup wg owns keys [64 wg, 64 wg + 64)
    // of every tile; warp w reads TMEM lanes 32 (w % 4) .. +31 (its rows).
    const int wg = (warp - 2) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                  // row inside the CTA tile = TMEM lane
    const int R = row0 + r;                        // row of the problem
    const int g = R / Bq, t_in = R % Bq;
    const int lim = i_first + t_in;                // causal limit among local keys
    const int c0 = wg * (TN / 2);                  // this warpgroup's first key / S column
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    const uint32_t ocol = tl + O_COL + wg * TD;    // this warpgroup's O
    float m_ref = -INFINITY, l = 0.f;
    int di = 0;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      // S_j was issued only after both P V of tile j-2 completed: its columns are free for P_j
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s_full[j & 1], (j >> 1) & 1, a.err));
      if (!ok) break;
      tc_fence_after();
      while (di < k && j >= tile_start[di + 1]) ++di;
      const bool local = di >= k;
      const int key0 = (j - tile_start[di]) * TN;
      const int nvalid = local ? TN : min(TN, doc_len_s[di] - key0);
      const int vis_end = local ? max(0, min(TN, lim - key0 + 1)) : nvalid;  // keys [0, vis_end) are visible
      const uint32_t scol = tl + (j & 1) * TN + c0;
      uint32_t v0[32], v1[32];  // S of keys c0 .. c0+31 and c0+32 .. c0+63
      tmem_ld32(scol, v0);
      tmem_ld32(scol + 32, v1);
      tmem_wait_ld();
#define SV(e) __uint_as_float((e) < 32 ? v0[(e) & 31] : v1[(e) & 31])
      // every key of this half visible for every row of the warp: no per-key masks
      const bool full = __all_sync(0xffffffffu, vis_end >= c0 + TN / 2);
      bool need = false;  // the reference max moved (O and l rescaled by alpha)
      float alpha = 1.f;
      bool done = false;
      if (kOptimistic && full && __all_sync(0xffffffffu, m_ref != -INFINITY)) {
        // fast path: P = exp2(S * scale - m_ref) with the current reference, no max pass
        const float2 sc2 = make_float2(a.scale_log2, a.scale_log2), nm2 = make_float2(-m_ref, -m_ref);
        float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t pk[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const int e = hh * 32 + 2 * u;
            const bool poly = (u & 3) >= 4 - kFastPoly;
            const float2 x = __ffma2_rn(make_float2(SV(e), SV(e + 1)), sc2, nm2);
            // ex2: +inf past 2^128; the polynomial: 2^64 at most
            const float2 pp = poly ? exp2_poly3x2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
            ls[u & 1] = __fadd2_rn(ls[u & 1], pp);
            pk[u] = pack_bf16(pp.x, pp.y);
          }
          tmem_st16(scol + hh * 16, pk);
        }
        const float lt = (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y);
        done = __all_sync(0xffffffffu, lt < kPMax);  // false for +inf and NaN as well
        if (done) l += lt;
      }
      if (!done) {
        // exact path: the (masked) half-row max, the lazy reference update, P over the S columns
        float mt;
        if (full) {
          float m4[4] = {SV(0), SV(1), SV(2), SV(3)};
#pragma unroll
          for (int pr = 2; pr < TN / 4; ++pr) m4[pr & 3] = max3f(m4[pr & 3], SV(2 * pr), SV(2 * pr + 1));
          mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * a.scale_log2;
        } else {
          mt = -INFINITY;
#pragma unroll
          for (int e = 0; e < TN / 2; ++e)
            if (c0 + e < vis_end) mt = fmaxf(mt, SV(e));
          mt = (mt == -INFINITY) ? mt : mt * a.scale_log2;
        }
        const float m_new = fmaxf(m_ref, mt);
        need = m_new > m_ref + kLazy;  // also true when m_ref = -inf and the half-tile has a key
        if (need) {
          alpha = exp2f(m_ref - m_new);  // 0 when m_ref = -inf
          l *= alpha;
          m_ref = m_new;
        }
        // P = exp2(S * scale - m_ref) as bf16 pairs over this half's first 32 S columns (already read)
        const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
        const float2 sc2 = make_float2(a.scale_log2, a.scale_log2), nm2 = make_float2(-m_use, -m_use);
        float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t pk[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const int e = hh * 32 + 2 * u;
            const bool poly = (u & 3) >= 4 - kPolyPairs;
            const float2 x = __ffma2_rn(make_float2(SV(e), SV(e + 1)), sc2, nm2);
            float2 pp = poly ? exp2_poly3x2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
            if (!full) {
              pp.x = (c0 + e < vis_end) ? pp.x : 0.f;
              pp.y = (c0 + e + 1 < vis_end) ? pp.y : 0.f;
            }
            ls[u & 1] = __fadd2_rn(ls[u & 1], pp);
            pk[u] = pack_bf16(pp.x, pp.y);
          }
          tmem_st16(scol + hh * 16, pk);
        }
        l += (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y);
      }
#undef SV
      // this warpgroup's P V of tile j-1 (issued a whole tile ago, so normally long
      // complete): waited at every tile, phase after phase, before O_wg may be rescaled
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait_bounded(&pv_done[wg], (j - 1) & 1, a.err))) {
        ok = false;
        break;
      }
      if (__any_sync(0xffffffffu, need && j > 0)) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < TD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(ocol + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(ocol + c * 32, o);
        }
      }
      tmem_wait_st();  // P (and any rescaled O) is in TMEM before the MMA may read it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[wg * 2 + (j & 1)]);
    }
    // ---- epilogue: once every P V has completed (o_done has a single phase, so
    // its wait is unambiguous), merge the two halves' (m, l, O) of each row
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(o_done, 0, a.err));
    if (!ok) *abort_s = 1;
    tc_fence_after();
    // (m, l) through this half's first two columns of S buffer 0, free once its P V completed
    tmem_st1(tl + c0, __float_as_uint(m_ref));
    tmem_st1(tl + c0 + 1, __float_as_uint(l));
    tmem_wait_st();
    tc_fence_before();
    named_barrier_sync(1, 2 * 4 * 32);
    tc_fence_after();
    if (!*abort_s && T > 0) {
      const uint32_t pc = tl + (c0 ^ (TN / 2));
      const float m_o = __uint_as_float(tmem_ld1(pc));
      const float l_o = __uint_as_float(tmem_ld1(pc + 1));
      tmem_wait_ld();
      const float mA = wg ? m_o : m_ref, lA = wg ? l_o : l;  // keys [0, 64) of every tile
      const float mB = wg ? m_ref : m_o, lB = wg ? l : l_o;  // keys [64, 128)
      const float mm = fmaxf(mA, mB);
      const float fA = mA == -INFINITY ? 0.f : exp2f(mA - mm);
      const float fB = mB == -INFINITY ? 0.f : exp2f(mB - mm);
      const float lt = lA * fA + lB * fB;
      const float inv = lt > 0.f ? 1.0f / lt : 0.f;
      const float wA = fA * inv, wB = fB * inv;
      const int hq = h * G + g;
      const int t = blk * Bq + t_in;
      if (a.lse_out && wg == 0)
        a.lse_out[((int64_t)b * a.n_q_heads + hq) * a.q_tokens + t] =
            lt > 0.f ? (mm + log2f(lt)) * 0.693147180559945309f : -INFINITY;
      // this warpgroup writes dims [64 wg, 64 wg + 64) of its rows
      float* dst = a.out + (((int64_t)b * a.n_q_heads + hq) * a.q_tokens + t) * TD + c0;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t oa[32], ob[32];
        tmem_ld32(tl + O_COL + c0 + cc * 32, oa);
        tmem_ld32(tl + O_COL + TD + c0 + cc * 32, ob);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + cc * 32 + e) =
              make_float4(__uint_as_float(oa[e]) * wA + __uint_as_float(ob[e]) * wB,
                          __uint_as_float(oa[e + 1]) * wA + __uint_as_float(ob[e + 1]) * wB,
                          __uint_as_float(oa[e + 2]) * wA + __uint_as_float(ob[e + 2]) * wB,
                          __uint_as_float(oa[e + 3]) * wA + __uint_as_float(ob[e + 3]) * wB);
      }
    }
  }
  // ---- teardown: every role is done with TMEM and shared memory
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace

bool attend_prefill_tc_supported(int head_dim, int group, int route_block) {
  return head_dim == TD && (route_block == 64 || route_block == 128) && (group * route_block) % TM == 0;
}
int attend_prefill_tc_tile_rows() { return TN; }

cudaError_t launch_attend_prefill_tc(const AttendArgs& a, const AttendMaps& m, const CUtensorMap& q_map,
                                     cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(attend_prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int nblk = a.q_tokens / a.route_block;
  const int rows = (a.n_q_heads / a.n_kv_heads) * a.route_block;
  dim3 grid(rows / TM, a.batch * nblk * a.n_kv_heads);
  attend_prefill_tc_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(q_map, m.bank_k, m.bank_v, m.loc_k, m.loc_v, a);
  return cudaGetLastError();
}

}  // namespace msa
