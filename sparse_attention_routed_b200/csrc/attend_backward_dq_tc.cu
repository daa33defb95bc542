// dQ of sparse_attend on the 5th-generation tensor cores, for a fixed selection
// and given each row's log-sum-exp and D = dO . O.
//   "MSA (Memory Sparse Attention)" (robocikowo.com), Komponenty (Memory Sparse
//   Attention Layer: trained end to end on the step's selection), Pułapki
//   implementacyjne (Global RoPE with a k-offset).
//
// With s = q_rot . k / sqrt(d), p = exp(s - lse) over the row's key set and
// dp = dO . v: dq_rot = sum over keys of p (dp - D) k / sqrt(d), turned back
// through the Global RoPE adjoint at the row's position.
//
// One CTA owns 128 query rows of one problem (sequence, routing block, KV head;
// rows ordered head-major) and walks the problem's key list in tiles of 128 keys
// (the selected documents' tiles, then the local tiles up to its last row):
//   warp 0     TMA producer: the RoPE'd query tile and the dO tile once, then
//              K_j (three-slot ring: S_j and dQ_j read it) and V_j (two slots:
//              only dP_j reads it).
//   warp 1     allocates all 512 TMEM columns -- S [0,128), dP[2] [128,384),
//              dQ [384,512) -- and issues, per tile j, S_j = Q K_j^T (once the
//              elementwise warps have read S_{j-1}), dP_j = dO V_j^T (once
//              dQ_{j-2} freed its buffer) and dQ += dS_{j-1} K_{j-1} (dS read
//              from TMEM as the A operand, K_{j-1} as an MN-major operand).
//   warps 2-9  two warpgroups; warpgroup w owns keys [64 w, 64 w + 64) of every
//              tile and a thread owns one row (its TMEM lane): it reads its S
//              values, frees S, then forms P = exp2(S scale - lse) (zero for
//              keys past a document and for local keys after the row's
//              position) and dS = P (dP - D) / sqrt(d) and writes dS as packed
//              bf16 over the dP columns it read. At the end they apply the
//              RoPE adjoint to dQ and write it.
// Every mbarrier parity wait targets the phase right after one the same waiter
// saw complete, so no wait can be satisfied by an older phase.
#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int TN = 128;               // keys per tile
constexpr int TM = 128;               // query rows per CTA
constexpr int TD = 128;               // head dim
constexpr int KSLOT = 3;
constexpr int VSLOT = 2;
constexpr int THREADS = 320;
constexpr int BOX = TN * 128;         // 64 dims of a 128-row tile (16 KB)
constexpr int TILE = 2 * BOX;         // 128 x 128 bf16 (32 KB)
constexpr int TOPK_MAX = 64;
constexpr int TMEM_COLS = 512;
constexpr int S_COL = 0;
constexpr int DP_COL = 128;           // dP[buf] = DP_COL + 128 buf (dS over its columns)
constexpr int DQ_COL = 384;

constexpr int OFF_Q = 0;
constexpr int OFF_DO = OFF_Q + TILE;
constexpr int OFF_K0 = OFF_DO + TILE;             // K[s] = OFF_K0 + s * TILE
constexpr int OFF_V0 = OFF_K0 + KSLOT * TILE;     // V[s] = OFF_V0 + s * TILE
constexpr int OFF_BAR = OFF_V0 + VSLOT * TILE;
constexpr int N_BAR = 1 + 2 * KSLOT + 2 * VSLOT + 1 + 1 + 2 + 4 + 2 + 1;
constexpr int OFF_TMEM = OFF_BAR + N_BAR * 8;
constexpr int OFF_TAB = OFF_TMEM + 16;
constexpr size_t SMEM_BYTES = 1024 + OFF_TAB + (TOPK_MAX + 2) * 4 + TOPK_MAX * 4 + TOPK_MAX * 8;
static_assert(SMEM_BYTES <= 232448, "shared memory");

// Shared-memory descriptors as two 32-bit halves (see umma_desc_sw128): lo = start >> 4 |
// (LBO >> 4) << 16, hi = SBO 1024 B | version 1 | 128-byte swizzle. Shared-memory
// addresses stay below 2^18, so adding an offset >> 4 to lo never carries.
constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
__device__ __forceinline__ uint32_t desc_lo(uint32_t addr, uint32_t lbo) { return (addr >> 4) | ((lbo >> 4) << 16); }

__device__ __forceinline__ void mma_ss(uint32_t d, uint32_t alo, uint32_t blo, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\tsetp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 da, {%1, %3};\n\tmov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %4, p;\n\t}" ::"r"(d),
      "r"(alo), "r"(blo), "r"(kDescHi), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint32_t blo, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %5, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "r"(blo), "r"(kDescHi), "r"(acc), "r"(idesc)
      : "memory");
}

__global__ void __launch_bounds__(THREADS, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_bk, const __grid_constant__ CUtensorMap tm_bv,
                     const __grid_constant__ CUtensorMap tm_lk, const __grid_constant__ CUtensorMap tm_lv,
                     const AttendBwdArgs g) {
  const AttendArgs& a = g.a;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* q_full = bars;                     // the query and dO tiles
  uint64_t* k_full = q_full + 1;               // [KSLOT]
  uint64_t* k_empty = k_full + KSLOT;          // [KSLOT] dQ_j (the last reader of K_j) completed
  uint64_t* v_full = k_empty + KSLOT;          // [VSLOT]
  uint64_t* v_empty = v_full + VSLOT;          // [VSLOT] dP_j completed
  uint64_t* s_full = v_empty + VSLOT;          // one phase per tile: S_j is in TMEM
  uint64_t* s_read = s_full + 1;               // one phase per tile: every elementwise warp has read S_j
  uint64_t* dp_full = s_read + 1;              // [buf] dP_j is in TMEM
  uint64_t* ds_full = dp_full + 2;             // [buf * 2 + warpgroup] one arrival per warp of the warpgroup
  uint64_t* dp_free = ds_full + 4;             // [buf] dQ_j completed: the buffer (dS_j) is free
  uint64_t* dq_done = dp_free + 2;             // one phase: every MMA of the CTA has completed
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
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
  const int rows = G * Bq;
  const int row0 = blockIdx.x * TM;  // rows ordered (head, token); 128 | G * Bq
  const int i_first = a.local_len - a.q_tokens + blk * Bq;
  const int r_end = row0 + TM - 1;
  const int i_max = i_first + (r_end / Bq != row0 / Bq ? Bq - 1 : r_end % Bq);
  const int k = a.top_k;

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
  if (tid == 0) {
    for (int i = 0; i < N_BAR; ++i) {
      uint32_t cnt = 1;
      if (bars + i == s_read) cnt = 8;
      if (bars + i >= ds_full && bars + i < dp_free) cnt = 4;
      mbar_init(&bars[i], cnt);
    }
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_base_s, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0) {
    int acc = 0;
    for (int d = 0; d < k; ++d) {
      tile_start[d] = acc;
      acc += (doc_len_s[d] + TN - 1) / TN;
    }
    tile_start[k] = acc;
    tile_start[k + 1] = acc + (i_max + 1 + TN - 1) / TN;
  }
  __syncthreads();
  const int T = tile_start[k + 1];
  const uint32_t tmem = *tmem_base_s;
  const uint32_t sbase = smem_addr(sm);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_do);
      prefetch_tensormap(&tm_bk);
      prefetch_tensormap(&tm_bv);
      prefetch_tensormap(&tm_lk);
      prefetch_tensormap(&tm_lv);
      const uint64_t pol = l2_policy_evict_last();  // the problem's other CTAs read the same tiles
      mbar_arrive_expect_tx(q_full, 2 * TILE);
#pragma unroll
      for (int sg = 0; sg < 2; ++sg) {
        const int r = row0 + 64 * sg;
        const int hq = h * G + r / Bq;
        const int y = (int)(((int64_t)b * a.n_q_heads + hq) * a.q_tokens + (int64_t)blk * Bq + r % Bq);
#pragma unroll
        for (int dh = 0; dh < 2; ++dh) {
          tma_load_2d(sm + OFF_Q + dh * BOX + sg * (64 * 128), &tm_q, dh * 64, y, q_full, pol);
          tma_load_2d(sm + OFF_DO + dh * BOX + sg * (64 * 128), &tm_do, dh * 64, y, q_full, pol);
        }
      }
      int di = 0;
      bool ok = true;
      for (int n = 0; ok && n < T; ++n) {
        while (di < k && n >= tile_start[di + 1]) ++di;
        const bool local = di >= k;
        const int tt = n - tile_start[di];
        const int y = local ? (b * a.n_kv_heads + h) * a.local_len + tt * TN : (int)(doc_base_s[di] + (long long)tt * TN);
        const int ks = n % KSLOT, ku = n / KSLOT, vs = n % VSLOT, vu = n / VSLOT;
        if (ku > 0 && !mbar_wait_bounded(&k_empty[ks], (ku - 1) & 1, a.err)) { ok = false; break; }
        uint8_t* kd = sm + OFF_K0 + ks * TILE;
        mbar_arrive_expect_tx(&k_full[ks], TILE);
        tma_load_2d(kd, local ? &tm_lk : &tm_bk, 0, y, &k_full[ks], pol);
        tma_load_2d(kd + BOX, local ? &tm_lk : &tm_bk, 64, y, &k_full[ks], pol);
        if (vu > 0 && !mbar_wait_bounded(&v_empty[vs], (vu - 1) & 1, a.err)) { ok = false; break; }
        uint8_t* vd = sm + OFF_V0 + vs * TILE;
        mbar_arrive_expect_tx(&v_full[vs], TILE);
        tma_load_2d(vd, local ? &tm_lv : &tm_bv, 0, y, &v_full[vs], pol);
        tma_load_2d(vd + BOX, local ? &tm_lv : &tm_bv, 64, y, &v_full[vs], pol);
      }
      // leave no copy in flight
      mbar_wait_bounded(q_full, 0, nullptr);
      for (int n = T > KSLOT ? T - KSLOT : 0; n < T; ++n) mbar_wait_bounded(&k_full[n % KSLOT], (n / KSLOT) & 1, nullptr);
      for (int n = T > VSLOT ? T - VSLOT : 0; n < T; ++n) mbar_wait_bounded(&v_full[n % VSLOT], (n / VSLOT) & 1, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = umma_idesc_bf16(TM, TN, false);   // S, dP: 128 rows x 128 keys
      const uint32_t idesc_q = umma_idesc_bf16(TM, TD, true);    // dQ: 128 rows x 128 dims, B MN-major
      bool ok = mbar_wait_bounded(q_full, 0, a.err);
      const uint32_t qlo = desc_lo(sbase + OFF_Q, 16), olo = desc_lo(sbase + OFF_DO, 16);
      // dQ += dS_i K_i, half by half as the warpgroups finish
      auto issue_dq = [&](int i) -> bool {
        const uint32_t buf = i & 1;
        const uint32_t klo = desc_lo(sbase + OFF_K0 + (i % KSLOT) * TILE, BOX);
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (!mbar_wait_bounded(&ds_full[buf * 2 + w], (i >> 1) & 1, a.err)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int kg = 4 * w + kk;                                 // keys 16 kg .. 16 kg + 15
            mma_ts(tmem + DQ_COL, tmem + DP_COL + buf * 128 + 64 * w + 8 * kk, klo + kg * (2048 >> 4), idesc_q,
                   (i > 0 || kg > 0) ? 1u : 0u);
          }
        }
        umma_commit(&dp_free[buf]);
        umma_commit(&k_empty[i % KSLOT]);
        return true;
      };
      for (int j = 0; ok && j < T; ++j) {
        const int ks = j % KSLOT, vs = j % VSLOT;
        if (!mbar_wait_bounded(&k_full[ks], (j / KSLOT) & 1, a.err)) { ok = false; break; }
        if (j >= 1 && !mbar_wait_bounded(s_read, (j - 1) & 1, a.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kklo = desc_lo(sbase + OFF_K0 + ks * TILE, 16);
#pragma unroll
        for (int kd = 0; kd < TD / 16; ++kd) {
          const uint32_t off = ((kd >> 2) * BOX + (kd & 3) * 32) >> 4;
          mma_ss(tmem + S_COL, qlo + off, kklo + off, idesc_s, kd > 0 ? 1u : 0u);
        }
        umma_commit(s_full);
        if (!mbar_wait_bounded(&v_full[vs], (j / VSLOT) & 1, a.err)) { ok = false; break; }
        if (j >= 2 && !mbar_wait_bounded(&dp_free[j & 1], ((j - 2) >> 1) & 1, a.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t vlo = desc_lo(sbase + OFF_V0 + vs * TILE, 16);
#pragma unroll
        for (int kd = 0; kd < TD / 16; ++kd) {
          const uint32_t off = ((kd >> 2) * BOX + (kd & 3) * 32) >> 4;
          mma_ss(tmem + DP_COL + (j & 1) * 128, olo + off, vlo + off, idesc_s, kd > 0 ? 1u : 0u);
        }
        umma_commit(&dp_full[j & 1]);
        umma_commit(&v_empty[vs]);
        if (j >= 1 && !issue_dq(j - 1)) { ok = false; break; }
      }
      if (ok && T > 0 && issue_dq(T - 1)) umma_commit(dq_done);
    }
  } else {
    // ------------------------------------------------------------ elementwise warps
    const int wg = (warp - 2) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                  // row inside the CTA tile = TMEM lane
    const int R = row0 + r;                        // row of the problem
    const int gq = R / Bq, t_in = R % Bq;
    const int lim = i_first + t_in;                // causal limit among local keys
    const int c0 = wg * (TN / 2);                  // this warpgroup's first key of every tile
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    const float lse = g.lse2[(int64_t)p * rows + R];
    const float drow = g.drow[(int64_t)p * rows + R];
    const float scale_log2 = a.scale_log2;
    const float inv_sqrt_d = a.scale_log2 * 0.693147180559945309f;
    int di = 0;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(s_full, j & 1, a.err));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[64];
      tmem_ld32(tl + S_COL + c0, *reinterpret_cast<uint32_t(*)[32]>(sv));
      tmem_ld32(tl + S_COL + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_read);
      while (di < k && j >= tile_start[di + 1]) ++di;
      const bool local = di >= k;
      const int key0 = (j - tile_start[di]) * TN;
      const int nvalid = local ? TN : min(TN, doc_len_s[di] - key0);
      const int vis_end = local ? max(0, min(TN, lim - key0 + 1)) : nvalid;  // keys [0, vis_end) are visible
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&dp_full[j & 1], (j >> 1) & 1, a.err));
      if (!ok) break;
      tc_fence_after();
      const uint32_t dcol = tl + DP_COL + (j & 1) * 128 + c0;
      // every key of this half visible for every row of the warp: no per-key masks
      const bool dense = __all_sync(0xffffffffu, vis_end >= c0 + TN / 2);
      const float2 sc2 = make_float2(scale_log2, scale_log2), nl2 = make_float2(-lse, -lse);
      const float2 nd2 = make_float2(-drow, -drow), c2 = make_float2(inv_sqrt_d, inv_sqrt_d);
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        uint32_t dv[32], pk[16];
        tmem_ld32(dcol + 32 * rr, dv);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int kk = 32 * rr + e;
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[kk]), __uint_as_float(sv[kk + 1])), sc2, nl2);
          float2 pe = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          if (!dense) {
            pe.x = (c0 + kk < vis_end) ? pe.x : 0.f;
            pe.y = (c0 + kk + 1 < vis_end) ? pe.y : 0.f;
          }
          const float2 dd = __fadd2_rn(make_float2(__uint_as_float(dv[e]), __uint_as_float(dv[e + 1])), nd2);
          const float2 ds2 = __fmul2_rn(__fmul2_rn(pe, dd), c2);
          pk[e >> 1] = pack_bf16(ds2.x, ds2.y);
        }
        tmem_st16(dcol + 16 * rr, pk);           // columns already read (this pass of 32 keys or the last)
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ds_full[(j & 1) * 2 + wg]);
    }
    // ---- epilogue: dQ through the Global-RoPE adjoint at the row's position
    if (ok && T > 0) ok = __all_sync(0xffffffffu, mbar_wait_bounded(dq_done, 0, a.err));
    if (ok && T > 0) {
      tc_fence_after();
      uint32_t xa[32], ya[32];
      tmem_ld32(tl + DQ_COL + 32 * wg, xa);
      tmem_ld32(tl + DQ_COL + 64 + 32 * wg, ya);
      tmem_wait_ld();
      const float2* cs = a.gtab + (int64_t)lim * (TD / 2) + 32 * wg;
      const int hq = h * G + gq;
      const int t = blk * Bq + t_in;
      float* dst = g.dq + (((int64_t)b * a.n_q_heads + hq) * a.q_tokens + t) * TD + 32 * wg;
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        float lo[4], hi[4];
#pragma unroll
        for (int f = 0; f < 4; ++f) {
          const float2 c2 = __ldg(cs + e + f);
          const float x = __uint_as_float(xa[e + f]), y = __uint_as_float(ya[e + f]);
          lo[f] = x * c2.x + y * c2.y;
          hi[f] = y * c2.x - x * c2.y;
        }
        *reinterpret_cast<float4*>(dst + e) = make_float4(lo[0], lo[1], lo[2], lo[3]);
        *reinterpret_cast<float4*>(dst + 64 + e) = make_float4(hi[0], hi[1], hi[2], hi[3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// dO in bf16, D = dO . O and the log-sum-exp in the backward's units (log2, rows
// of a problem) for every query row (one warp per row of 128 dims).
__global__ void bwd_prep_kernel(const float* __restrict__ dout, const float* __restrict__ out,
                                const float* __restrict__ lse, uint16_t* __restrict__ dout_bf,
                                float* __restrict__ drow, float* __restrict__ lse2, int64_t n_rows,
                                int n_q_heads, int n_kv_heads, int q_tokens, int route_block) {
  const int lane = threadIdx.x & 31;
  const int64_t wpb = blockDim.x >> 5;
  for (int64_t row = blockIdx.x * wpb + (threadIdx.x >> 5); row < n_rows; row += (int64_t)gridDim.x * wpb) {
    const float4 d = *reinterpret_cast<const float4*>(dout + row * TD + 4 * lane);
    const float4 o = *reinterpret_cast<const float4*>(out + row * TD + 4 * lane);
    *reinterpret_cast<uint2*>(dout_bf + row * TD + 4 * lane) = make_uint2(pack_bf16(d.x, d.y), pack_bf16(d.z, d.w));
    float s = d.x * o.x + d.y * o.y + d.z * o.z + d.w * o.w;
#pragma unroll
    for (int o2 = 16; o2; o2 >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o2);
    if (lane == 0) {
      // row = (b, hq, t) -> problem p = (b, t / Bq, hq / G) and row (hq % G) * Bq + t % Bq inside it
      const int t = (int)(row % q_tokens);
      const int hq = (int)((row / q_tokens) % n_q_heads);
      const int64_t bb = row / ((int64_t)q_tokens * n_q_heads);
      const int G = n_q_heads / n_kv_heads, nblk = q_tokens / route_block;
      const int64_t p = (bb * nblk + t / route_block) * n_kv_heads + hq / G;
      const int64_t pr = p * (G * route_block) + (hq % G) * route_block + t % route_block;
      drow[pr] = s;
      lse2[pr] = lse[row] * 1.4426950408889634f;
    }
  }
}

}  // namespace

cudaError_t launch_attend_bwd_dq_tc(const AttendBwdArgs& g, const AttendMaps& m, const CUtensorMap& q_map,
                                    const CUtensorMap& do_map, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const AttendArgs& a = g.a;
  if (a.top_k > TOPK_MAX) return cudaErrorInvalidValue;
  const int nblk = a.q_tokens / a.route_block;
  const int rows = (a.n_q_heads / a.n_kv_heads) * a.route_block;
  dim3 grid(rows / TM, a.batch * nblk * a.n_kv_heads);
  bwd_dq_tc_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(q_map, do_map, m.bank_k, m.bank_v, m.loc_k, m.loc_v, g);
  return cudaGetLastError();
}

cudaError_t launch_attend_bwd_prep(const float* dout, const float* out, const float* lse, uint16_t* dout_bf,
                                   float* drow, float* lse2, int batch, int n_q_heads, int n_kv_heads, int q_tokens,
                                   int route_block, int sms, cudaStream_t s) {
  const int64_t n_rows = (int64_t)batch * n_q_heads * q_tokens;
  const int64_t want = (n_rows + 7) / 8;
  const int blocks = (int)std::min<int64_t>(want, (int64_t)sms * 16);
  bwd_prep_kernel<<<blocks < 1 ? 1 : blocks, 256, 0, s>>>(dout, out, lse, dout_bf, drow, lse2, n_rows, n_q_heads,
                                                          n_kv_heads, q_tokens, route_block);
  return cudaGetLastError();
}

}  // namespace msa
