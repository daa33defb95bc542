// dK and dV of sparse_attend on the 5th-generation tensor cores, for a fixed
// selection (top-k routing is not differentiated).
//   "MSA (Memory Sparse Attention)" (robocikowo.com), Komponenty (Memory Sparse
//   Attention Layer: trained end to end on the step's selection), Pułapki
//   implementacyjne (Global RoPE with a k-offset, Parallel RoPE of the bank).
//
// With s = q_rot . k / sqrt(d), p = softmax over the row's key set, dp = dO . v
// and D = dO . O per row: dv_j = sum over rows of p_j dO, and
// dk_j = sum over rows of p_j (dp_j - D) q_rot / sqrt(d), turned back through
// the RoPE adjoint (the rotation by the negative angle).
//
// Work is organised by key tile, not by problem: an item is 128 keys of one
// selected document of one KV head (or of one sequence's local context), and
// its CTA visits every query row that attends those keys -- the rows of every
// problem (sequence, routing block, KV head) whose selection holds the document
// (an index built by bwd_index_kernel), or, for local keys, of every routing
// block at or after the keys. dK and dV of the item stay in TMEM across all
// those rows and leave once, so no two CTAs add to the same gradient row.
//
// Persistent CTAs, one per SM, take items round-robin. Per CTA:
//   warp 0     TMA producer: an item's K and V tiles (two-slot ring), then its
//              query chunks: 64 rows of RoPE'd queries and of dO (bf16) and the
//              rows' log-sum-exp and D (three-slot ring).
//   warp 1     allocates all 512 TMEM columns and issues, per chunk c,
//              S^T = K Q^T and dP^T = V dO^T (M = 128 keys, N = 64 rows, K = d)
//              into one of two buffers, then, for chunk c-1, dV += P^T dO and
//              dK += dS^T Q (A = P^T / dS^T read from TMEM, B = dO / Q as
//              MN-major shared-memory operands, K = the 64 rows).
//   warps 2-9  two warpgroups, one per half of the chunk's rows; a thread owns
//              one key (its TMEM lane): it reads S^T and dP^T, forms
//              P = exp2(S scale - lse) and dS = P (dP - D) / sqrt(d) (zero for
//              keys past the document, and for local keys after the row's
//              position), and writes both back as packed bf16 over the columns
//              it read. At the end of an item they stage its dV in the item's
//              K/V slot (64 KB) and take its dK into registers -- TMEM is free
//              for the next item from here; the dK follows into the slot two
//              chunks into the next item, once the dV has left it.
//   warps 10-11 reducers: turn the staged dK through the RoPE adjoint in
//              place (64 keys each), and warp 10 adds each staged half to the
//              gradients with TMA reduce-add (the additions run in L2) and
//              frees the slot; the waits for those copies fall on it alone.
// Every mbarrier parity wait targets the phase right after one the same waiter
// saw complete, so no wait can be satisfied by an older phase.
#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int KT = 128;               // keys per item
constexpr int RC = 64;                // query rows per chunk
constexpr int DH = 128;               // head dim
constexpr int KBOX = KT * 128;        // 64 dims of the key tile (16 KB)
constexpr int KTILE = 2 * KBOX;       // 128 x 128 bf16 (32 KB)
constexpr int CBOX = RC * 128;        // 64 dims of a chunk (8 KB)
constexpr int CTILE = 2 * CBOX;       // 64 x 128 bf16 (16 KB)
constexpr int KVSLOT = 2;
constexpr int CSLOT = 3;
constexpr int THREADS = 384;          // producer, MMA, 8 elementwise warps, 2 reducer warps
constexpr int TMEM_COLS = 512;
constexpr int S_COL = 0;              // S^T[buf]  = S_COL + 64 buf   (P^T over its columns)
constexpr int DP_COL = 128;           // dP^T[buf] = DP_COL + 64 buf  (dS^T over its columns)
constexpr int DV_COL = 256;
constexpr int DK_COL = 384;

// shared memory layout (offsets from a 1 KiB-aligned base)
constexpr int OFF_KV = 0;                                  // slot s: K at OFF_KV + s * 2 KTILE, V after it
constexpr int OFF_C = OFF_KV + KVSLOT * 2 * KTILE;         // slot c: Q at OFF_C + c * 2 CTILE, dO after it
constexpr int OFF_ST = OFF_C + CSLOT * 2 * CTILE;          // slot c: lse2[64], D[64] at OFF_ST + c * 512
constexpr int OFF_BAR = OFF_ST + CSLOT * 2 * RC * 4;
constexpr int N_BAR = 2 * KVSLOT + 2 * CSLOT + 2 + 2 + 4 + 6;
constexpr int OFF_TMEM = OFF_BAR + N_BAR * 8;

// One item: 128 keys and the problems whose rows attend them.
struct Item {
  bool local;
  int b, h, t;          // sequence (local items), KV head, tile index inside the document / local context
  int nvalid;           // keys of the tile inside the document / local context
  int kv_row;           // first row of the tile in the K/V tensor maps (and in the gradient maps)
  const int* plist;     // bank items: the problems that selected the document (ascending)
  int np;               // number of problems
  int blk0;             // local items: the first routing block whose rows reach the tile
};

// Items [0, NL) are the local tiles (b, h, t); the rest are the bank tiles of the
// selection index, head by head (pre[h] = tiles of the heads before h).
__device__ __forceinline__ int4 item_record(const AttendBwdArgs& g, int idx, int NL, int total, const int* pre,
                                            int n_kv_heads) {
  if (idx < NL || idx >= total) return make_int4(0, 0, 0, 0);
  const int j = idx - NL;
  int h = 0;
  while (h + 1 < n_kv_heads && pre[h + 1] <= j) ++h;
  return __ldg(g.idx_items + (int64_t)h * g.idx_item_cap + (j - pre[h]));
}

__device__ __forceinline__ bool make_item(const AttendBwdArgs& g, int idx, int NL, int LT, const int* pre, int4 rec,
                                          Item& it) {
  const AttendArgs& a = g.a;
  const int nblk = a.q_tokens / a.route_block;
  if (idx < NL) {
    it.local = true;
    it.t = idx % LT;
    it.h = (idx / LT) % a.n_kv_heads;
    it.b = idx / (LT * a.n_kv_heads);
    const int u0 = it.t * KT;
    it.nvalid = min(KT, a.local_len - u0);
    // rows of block blk sit at local indices [i_first, i_first + Bq); they see key u iff u <= index
    const int base = a.local_len - a.q_tokens;
    const int need = u0 - base - (a.route_block - 1);  // i_first(blk) >= need  <=>  last row reaches u0
    it.blk0 = need <= 0 ? 0 : (need + a.route_block - 1) / a.route_block;
    it.np = nblk - it.blk0;
    it.plist = nullptr;
    it.kv_row = (it.b * a.n_kv_heads + it.h) * a.local_len + u0;
    return it.np > 0 && it.nvalid > 0;
  }
  const int j = idx - NL;
  int h = 0;
  while (h + 1 < a.n_kv_heads && pre[h + 1] <= j) ++h;
  it.local = false;
  it.h = h;
  it.kv_row = rec.x;
  it.t = rec.y & 0xFFFF;
  it.nvalid = rec.y >> 16;
  it.plist = g.idx_prob + (int64_t)h * g.idx_cap + rec.z;
  it.np = rec.w;
  it.b = 0;
  it.blk0 = 0;
  return it.np > 0;
}

__device__ __forceinline__ int item_problem(const AttendArgs& a, const Item& it, int i) {
  if (!it.local) return __ldg(it.plist + i);
  const int nblk = a.q_tokens / a.route_block;
  return (it.b * nblk + it.blk0 + i) * a.n_kv_heads + it.h;
}

// Shared-memory descriptors as two 32-bit halves: lo = start >> 4 | (LBO >> 4) << 16,
// hi = SBO >> 4 (1024 B) | version 1 | 128-byte swizzle. Shared-memory addresses
// stay below 2^18, so adding an offset >> 4 to lo never carries out of the start field.
constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
__device__ __forceinline__ uint32_t desc_lo(uint32_t addr, uint32_t lbo) { return (addr >> 4) | ((lbo >> 4) << 16); }

// D[tmem] (+)= A[smem] B[smem]^T with descriptors given by their low halves.
__device__ __forceinline__ void mma_ss(uint32_t d, uint32_t alo, uint32_t blo, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\tsetp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 da, {%1, %3};\n\tmov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %4, p;\n\t}" ::"r"(d),
      "r"(alo), "r"(blo), "r"(kDescHi), "r"(idesc), "r"(acc)
      : "memory");
}

// D[tmem] (+)= A[tmem] B[smem].
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint32_t blo, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %5, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "r"(blo), "r"(kDescHi), "r"(acc), "r"(idesc)
      : "memory");
}

// Element-wise add of a shared-memory box into global memory through a tensor map
// (the reduction runs in L2), tracked by the issuing thread's bulk async-group.
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(smem_addr(src))
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// 16 / 8 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// This thread's 32 fp32 values of row r into box c of the staging area: four boxes
// of [128 rows][32 floats], 128-byte swizzled as the gradient tensor maps expect.
__device__ __forceinline__ void stage_row(uint8_t* stg, int c, int r, const float (&v)[32]) {
  uint8_t* row = stg + c * (KT * 128) + r * 128;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<float4*>(row + ((j ^ (r & 7)) << 4)) = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
}

constexpr int OFF_PRE = OFF_TMEM + 16;                     // item prefix over KV heads [65]
constexpr int MAX_HKV = 64;
constexpr size_t SMEM_TOTAL = 1024 + OFF_PRE + (MAX_HKV + 1) * 4;
static_assert(SMEM_TOTAL <= 232448, "shared memory");

__global__ void __launch_bounds__(THREADS, 1)
    bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_bk, const __grid_constant__ CUtensorMap tm_bv,
                       const __grid_constant__ CUtensorMap tm_lk, const __grid_constant__ CUtensorMap tm_lv,
                       const __grid_constant__ CUtensorMap tm_dkb, const __grid_constant__ CUtensorMap tm_dvb,
                       const __grid_constant__ CUtensorMap tm_dkl, const __grid_constant__ CUtensorMap tm_dvl,
                       const AttendBwdArgs g) {
  const AttendArgs& a = g.a;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* kv_full = bars;                      // [KVSLOT]
  uint64_t* kv_empty = kv_full + KVSLOT;         // [KVSLOT]  the item's dK / dV left the slot (staging)
  uint64_t* c_full = kv_empty + KVSLOT;          // [CSLOT]
  uint64_t* c_empty = c_full + CSLOT;            // [CSLOT]
  uint64_t* s_full = c_empty + CSLOT;            // [buf]  S^T and dP^T of the buffer are in TMEM
  uint64_t* s_free = s_full + 2;                 // [buf]  the dV / dK MMAs that read the buffer completed
  uint64_t* p_full = s_free + 2;                 // [buf * 2 + half]  one arrival per warp of the warpgroup
  uint64_t* acc_full = p_full + 4;               // one phase per item: its dK / dV are complete
  uint64_t* acc_free = acc_full + 1;             // one phase per item: the elementwise warps have read them
  uint64_t* staged_v = acc_free + 1;             // one phase per item: its dV is in the staging area
  uint64_t* staged_k = staged_v + 1;             // one phase per item: its dK is in the staging area
  uint64_t* vread = staged_k + 1;                // one phase per item: its dV left the staging area
  uint64_t* rope_done = vread + 1;               // one phase per item: the second reducer warp turned its keys
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
  int* pre = reinterpret_cast<int*>(sm + OFF_PRE);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int Bq = a.route_block;
  const int nblk = a.q_tokens / Bq;
  const int rows = G * Bq;                       // rows of a problem, ordered (head, token); 64 | Bq
  const int CH = rows / RC;                      // chunks per problem
  const int LT = (a.local_len + KT - 1) / KT;
  const int NL = a.batch * a.n_kv_heads * LT;

  if (tid == 0) {
    for (int i = 0; i < N_BAR; ++i) {
      uint32_t cnt = 1;
      if (bars + i >= p_full && bars + i < acc_full) cnt = 4;
      if (bars + i == acc_free || bars + i == staged_v || bars + i == staged_k) cnt = 8;
      mbar_init(&bars[i], cnt);
    }
    fence_barrier_init();
    int acc = 0;
    for (int h = 0; h < a.n_kv_heads; ++h) {
      pre[h] = acc;
      acc += __ldg(g.idx_nitems + h);
    }
    pre[a.n_kv_heads] = acc;
  }
  if (warp == 1) tmem_alloc(tmem_base_s, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_s;
  const uint32_t sbase = smem_addr(sm);
  const int total = NL + pre[a.n_kv_heads];
  const int step = gridDim.x;
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_do);
      prefetch_tensormap(&tm_bk);
      prefetch_tensormap(&tm_bv);
      prefetch_tensormap(&tm_lk);
      prefetch_tensormap(&tm_lv);
      const uint64_t keep = l2_policy_evict_last();   // queries and dO are read by many items
      const uint64_t once = l2_policy_evict_first();  // a key tile is read by one item
      uint32_t n_it = 0, cc = 0;
      bool ok = true;
      Item it;
      int nidx = 0;
      int4 rec = item_record(g, blockIdx.x, NL, total, pre, a.n_kv_heads), nrec;
      for (int idx = blockIdx.x; ok && idx < total; idx = nidx, rec = nrec) {
        nidx = idx + step;
        nrec = item_record(g, nidx, NL, total, pre, a.n_kv_heads);
        if (!make_item(g, idx, NL, LT, pre, rec, it)) continue;
        const int s = n_it % KVSLOT, use = n_it / KVSLOT;
        if (use > 0 && !mbar_wait_bounded(&kv_empty[s], (use - 1) & 1, a.err)) { ok = false; break; }
        const CUtensorMap* mk = it.local ? &tm_lk : &tm_bk;
        const CUtensorMap* mv = it.local ? &tm_lv : &tm_bv;
        uint8_t* kd = sm + OFF_KV + s * 2 * KTILE;
        mbar_arrive_expect_tx(&kv_full[s], 2 * KTILE);
        tma_load_2d(kd, mk, 0, it.kv_row, &kv_full[s], once);
        tma_load_2d(kd + KBOX, mk, 64, it.kv_row, &kv_full[s], once);
        tma_load_2d(kd + KTILE, mv, 0, it.kv_row, &kv_full[s], once);
        tma_load_2d(kd + KTILE + KBOX, mv, 64, it.kv_row, &kv_full[s], once);
        ++n_it;
        const int nch = it.np * CH;
        for (int q = 0; q < nch; ++q, ++cc) {
          const int cs = cc % CSLOT, cu = cc / CSLOT;
          if (cu > 0 && !mbar_wait_bounded(&c_empty[cs], (cu - 1) & 1, a.err)) { ok = false; break; }
          const int p = item_problem(a, it, q / CH);
          const int r0 = (q % CH) * RC;
          const int b = p / (a.n_kv_heads * nblk), blk = (p / a.n_kv_heads) % nblk;
          const int y = (int)(((int64_t)b * a.n_q_heads + it.h * G + r0 / Bq) * a.q_tokens + (int64_t)blk * Bq +
                              r0 % Bq);
          uint8_t* cd = sm + OFF_C + cs * 2 * CTILE;
          float* st = reinterpret_cast<float*>(sm + OFF_ST + cs * 2 * RC * 4);
          mbar_arrive_expect_tx(&c_full[cs], 2 * CTILE + 2 * RC * 4);
          tma_load_2d(cd, &tm_q, 0, y, &c_full[cs], keep);
          tma_load_2d(cd + CBOX, &tm_q, 64, y, &c_full[cs], keep);
          tma_load_2d(cd + CTILE, &tm_do, 0, y, &c_full[cs], keep);
          tma_load_2d(cd + CTILE + CBOX, &tm_do, 64, y, &c_full[cs], keep);
          const int64_t so = (int64_t)p * rows + r0;
          bulk_load(st, g.lse2 + so, RC * 4, &c_full[cs], keep);
          bulk_load(st + RC, g.drow + so, RC * 4, &c_full[cs], keep);
        }
      }
      // leave no copy in flight: wait for the last fills of both rings
      for (uint32_t q = cc > (uint32_t)CSLOT ? cc - CSLOT : 0; q < cc; ++q)
        mbar_wait_bounded(&c_full[q % CSLOT], (q / CSLOT) & 1, nullptr);
      for (uint32_t q = n_it > (uint32_t)KVSLOT ? n_it - KVSLOT : 0; q < n_it; ++q)
        mbar_wait_bounded(&kv_full[q % KVSLOT], (q / KVSLOT) & 1, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = umma_idesc_bf16(KT, RC, false);   // S^T, dP^T: 128 keys x 64 rows
      const uint32_t idesc_g = umma_idesc_bf16(KT, DH, true);    // dV, dK: 128 keys x 128 dims, B MN-major
      struct Pending { uint32_t cc, n_it; bool first, last; };
      Pending pv{};
      bool have = false, ok = true;
      // dV += P^T dO and dK += dS^T Q for chunk x, half by half as the warpgroups finish
      auto grads = [&](const Pending& x) -> bool {
        if (x.first && x.n_it > 0 && !mbar_wait_bounded(acc_free, (x.n_it - 1) & 1, a.err)) return false;
        const uint32_t buf = x.cc & 1, cs = x.cc % CSLOT;
        const uint32_t qb = sbase + OFF_C + cs * 2 * CTILE;
        const uint32_t qlo = desc_lo(qb, CBOX), dlo = desc_lo(qb + CTILE, CBOX);
        const uint32_t pa = tmem + S_COL + buf * 64, sa = tmem + DP_COL + buf * 64;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          if (!mbar_wait_bounded(&p_full[buf * 2 + hh], (x.cc >> 1) & 1, a.err)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 2 * hh; kk < 2 * hh + 2; ++kk) {
            const uint32_t acol = (kk >> 1) * 32 + (kk & 1) * 8;  // rows 16 kk .. 16 kk + 15, two per column
            const uint32_t acc = (x.first && kk == 0) ? 0u : 1u;
            mma_ts(tmem + DV_COL, pa + acol, dlo + kk * (2048 >> 4), idesc_g, acc);
            mma_ts(tmem + DK_COL, sa + acol, qlo + kk * (2048 >> 4), idesc_g, acc);
          }
        }
        umma_commit(&s_free[buf]);
        umma_commit(&c_empty[cs]);
        if (x.last) umma_commit(acc_full);
        return true;
      };
      uint32_t n_it = 0, cc = 0;
      Item it;
      int nidx = 0;
      int4 rec = item_record(g, blockIdx.x, NL, total, pre, a.n_kv_heads), nrec;
      for (int idx = blockIdx.x; ok && idx < total; idx = nidx, rec = nrec) {
        nidx = idx + step;
        nrec = item_record(g, nidx, NL, total, pre, a.n_kv_heads);
        if (!make_item(g, idx, NL, LT, pre, rec, it)) continue;
        const uint32_t kvs = n_it % KVSLOT;
        if (!mbar_wait_bounded(&kv_full[kvs], (n_it / KVSLOT) & 1, a.err)) { ok = false; break; }
        const uint32_t kb = sbase + OFF_KV + kvs * 2 * KTILE;
        const uint32_t klo = desc_lo(kb, 16), vlo = desc_lo(kb + KTILE, 16);
        const int nch = it.np * CH;
        for (int q = 0; q < nch; ++q, ++cc) {
          const uint32_t cs = cc % CSLOT, buf = cc & 1;
          if (!mbar_wait_bounded(&c_full[cs], (cc / CSLOT) & 1, a.err)) { ok = false; break; }
          if (cc >= 2 && !mbar_wait_bounded(&s_free[buf], ((cc - 2) >> 1) & 1, a.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t qb = sbase + OFF_C + cs * 2 * CTILE;
          const uint32_t qlo = desc_lo(qb, 16), dlo = desc_lo(qb + CTILE, 16);
          const uint32_t sd = tmem + S_COL + buf * 64, pd = tmem + DP_COL + buf * 64;
#pragma unroll
          for (int ks = 0; ks < DH / 16; ++ks) {
            const uint32_t ko = ((ks >> 2) * KBOX + (ks & 3) * 32) >> 4, co = ((ks >> 2) * CBOX + (ks & 3) * 32) >> 4;
            mma_ss(sd, klo + ko, qlo + co, idesc_s, ks > 0 ? 1u : 0u);
            mma_ss(pd, vlo + ko, dlo + co, idesc_s, ks > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[buf]);
          if (have && !grads(pv)) { ok = false; break; }
          pv = Pending{cc, n_it, q == 0, q == nch - 1};
          have = true;
        }
        ++n_it;
      }
      if (ok && have) grads(pv);
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------ elementwise warps
    const int q4 = warp & 3;                       // TMEM lane quadrant
    const int hh = (warp - 2) >> 2;                // half of the chunk's rows / of the dims in the epilogue
    const int key = q4 * 32 + lane;                // this thread's key in the tile = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
    const float scale_log2 = a.scale_log2;
    const float inv_sqrt_d = a.scale_log2 * 0.693147180559945309f;
    uint32_t n_it = 0, cc = 0;
    bool ok = true;
    // dK of the previous item, held until the staging area is free
    float klo[32], khi[32];
    bool pend = false;
    uint32_t pend_it = 0, pend_slot = 0;
    // stage the held dK once the reducer has read the item's dV out of its slot
    auto flush_dk = [&]() -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(vread, pend_it & 1, a.err))) return false;
      uint8_t* stg = sm + OFF_KV + pend_slot * 2 * KTILE;
      stage_row(stg, hh, key, klo);
      stage_row(stg, 2 + hh, key, khi);
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(staged_k);
      pend = false;
      return true;
    };
    Item it;
    int nidx = 0;
    int4 rec = item_record(g, blockIdx.x, NL, total, pre, a.n_kv_heads), nrec;
    for (int idx = blockIdx.x; ok && idx < total; idx = nidx, rec = nrec) {
      nidx = idx + step;
      nrec = item_record(g, nidx, NL, total, pre, a.n_kv_heads);
      if (!make_item(g, idx, NL, LT, pre, rec, it)) continue;
      const bool kvalid = key < it.nvalid;
      const int u = it.t * KT + key;               // local index (local items) / position in the document
      const int nch = it.np * CH;
      for (int q = 0; q < nch; ++q, ++cc) {
        const uint32_t cs = cc % CSLOT, buf = cc & 1;
        bool w = mbar_wait_bounded(&c_full[cs], (cc / CSLOT) & 1, a.err);
        w = w && mbar_wait_bounded(&s_full[buf], (cc >> 1) & 1, a.err);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        tc_fence_after();
        // the rows' causal limit among local keys: rows of one chunk share a head and run over consecutive tokens
        int lim0 = 1 << 30;                        // bank keys: every row sees every key
        if (it.local) {
          const int blk = it.blk0 + q / CH;
          lim0 = a.local_len - a.q_tokens + blk * Bq + ((q % CH) * RC) % Bq + 32 * hh;
        }
        const float* st = reinterpret_cast<const float*>(sm + OFF_ST + cs * 2 * RC * 4) + 32 * hh;
        const uint32_t scol = lane_base + S_COL + buf * 64 + 32 * hh, dcol = lane_base + DP_COL + buf * 64 + 32 * hh;
        // rows [vstart, 32) of this half see the key: all of them (bank keys), from the row whose
        // position reaches the key (local keys), none (keys past the document or context)
        const int vstart = !kvalid ? 32 : (it.local ? max(0, u - lim0) : 0);
        const bool dense = __all_sync(0xffffffffu, vstart == 0);
        const float2 sc2 = make_float2(scale_log2, scale_log2), c2 = make_float2(inv_sqrt_d, inv_sqrt_d);
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {           // 16 rows at a time; P / dS over columns already read
          uint32_t sv[16], dv[16], pp[8], ds[8];
          tmem_ld16(scol + 16 * rr, sv);
          tmem_ld16(dcol + 16 * rr, dv);
          float4 l4[4], d4[4];                     // the rows' log-sum-exp and D
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            l4[v] = *reinterpret_cast<const float4*>(st + 16 * rr + 4 * v);
            d4[v] = *reinterpret_cast<const float4*>(st + RC + 16 * rr + 4 * v);
          }
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float4 lv = l4[j >> 2], dvv = d4[j >> 2];
            const float2 nl = (j & 2) ? make_float2(-lv.z, -lv.w) : make_float2(-lv.x, -lv.y);
            const float2 nd = (j & 2) ? make_float2(-dvv.z, -dvv.w) : make_float2(-dvv.x, -dvv.y);
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])), sc2, nl);
            float2 pe = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            if (!dense) {
              const int row = 16 * rr + j;
              pe.x = row >= vstart ? pe.x : 0.f;
              pe.y = row + 1 >= vstart ? pe.y : 0.f;
            }
            const float2 dd = __fadd2_rn(make_float2(__uint_as_float(dv[j]), __uint_as_float(dv[j + 1])), nd);
            const float2 dsv = __fmul2_rn(__fmul2_rn(pe, dd), c2);
            pp[j >> 1] = pack_bf16(pe.x, pe.y);
            ds[j >> 1] = pack_bf16(dsv.x, dsv.y);
          }
          tmem_st8(scol + 8 * rr, pp);
          tmem_st8(dcol + 8 * rr, ds);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[buf * 2 + hh]);
        // the previous item's dK goes out after this item's second chunk (its dV has had time to leave)
        if (pend && q == min(1, nch - 1) && !flush_dk()) { ok = false; break; }
      }
      if (!ok) break;
      if (pend && !flush_dk()) { ok = false; break; }
      // ---- the item's dV, dims [32 hh, 32 hh + 32) and [64 + 32 hh, 96 + 32 hh): staged in the
      // item's K/V slot for the reducer; then its dK, held in registers, and TMEM is free
      const uint32_t kvs = n_it % KVSLOT;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(acc_full, n_it & 1, a.err))) { ok = false; break; }
      tc_fence_after();
      {
        float vlo[32], vhi[32];
        tmem_ld32(lane_base + DV_COL + 32 * hh, reinterpret_cast<uint32_t(&)[32]>(vlo));
        tmem_ld32(lane_base + DV_COL + 64 + 32 * hh, reinterpret_cast<uint32_t(&)[32]>(vhi));
        tmem_wait_ld();
        // keys past the document / context hold exact zeros (P = dS = 0): adding them is harmless
        uint8_t* stg = sm + OFF_KV + kvs * 2 * KTILE;
        stage_row(stg, hh, key, vlo);
        stage_row(stg, 2 + hh, key, vhi);
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(staged_v);
      }
      tmem_ld32(lane_base + DK_COL + 32 * hh, reinterpret_cast<uint32_t(&)[32]>(klo));
      tmem_ld32(lane_base + DK_COL + 64 + 32 * hh, reinterpret_cast<uint32_t(&)[32]>(khi));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_free);
      pend = true;
      pend_it = n_it;
      pend_slot = kvs;
      ++n_it;
    }
    if (ok && pend) flush_dk();
  } else {
    // ------------------------------------------------------------ reducers: the gradients out of the staging area
    // warp 10 issues the copies (and alone waits for them); both turn dK through the RoPE adjoint,
    // warp 10 keys [0, 64) of the tile and warp 11 keys [64, 128)
    const bool lead = warp == 10;
    const int kr0 = lead ? 0 : 64;
    // offset of dim l (this lane) of a row r with r % 8 == e inside a swizzled box, minus 32 r
    int swz[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) swz[e] = (((lane >> 2) ^ e) << 2) + (lane & 3);
    uint32_t n_it = 0;
    bool ok = true;
    Item it;
    int nidx = 0;
    int4 rec = item_record(g, blockIdx.x, NL, total, pre, a.n_kv_heads), nrec;
    for (int idx = blockIdx.x; ok && idx < total; idx = nidx, rec = nrec) {
      nidx = idx + step;
      nrec = item_record(g, nidx, NL, total, pre, a.n_kv_heads);
      if (!make_item(g, idx, NL, LT, pre, rec, it)) continue;
      const uint32_t kvs = n_it % KVSLOT;
      uint8_t* stg = sm + OFF_KV + kvs * 2 * KTILE;
      const CUtensorMap* mdv = it.local ? &tm_dvl : &tm_dvb;
      const CUtensorMap* mdk = it.local ? &tm_dkl : &tm_dkb;
      if (lead) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(staged_v, n_it & 1, a.err))) { ok = false; break; }
        if (lane == 0) {
#pragma unroll
          for (int c = 0; c < 4; ++c) tma_reduce_add_2d(mdv, stg + c * (KT * 128), 32 * c, it.kv_row);
          bulk_commit();
          bulk_wait_read0();
          mbar_arrive(vread);
        }
        __syncwarp();
      }
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(staged_k, n_it & 1, a.err))) { ok = false; break; }
      // dK through the RoPE adjoint, in place: Global RoPE at k_off + u (local keys), Parallel
      // RoPE at the position u in the document (bank keys). Lane l turns the dim pairs (l, l + 64)
      // and (l + 32, l + 96) of every key. The (cos, sin) of a key come from the table every 16
      // keys and in between from the previous key's by the one-position rotation
      // R(1) = R(u + 1) R(u)^-1 (fp32 rounding of 15 steps, ~1e-6).
      if (kr0 < it.nvalid) {
        const float2* tab = it.local ? a.gtab : g.ptab;
        const int64_t u0 = (int64_t)it.t * KT + kr0;
        const int nv = it.nvalid - kr0;          // keys of this warp's half inside the tile (> 0)
        float* box0 = reinterpret_cast<float*>(stg) + kr0 * 32;
        float2 sa[4], sb[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int64_t u = u0 + min(16 * k, nv - 1);
          sa[k] = __ldg(tab + u * (DH / 2) + lane);
          sb[k] = __ldg(tab + u * (DH / 2) + 32 + lane);
        }
        float2 ra = make_float2(1.f, 0.f), rb = make_float2(1.f, 0.f);
        if (nv > 1) {
          const float2 a1 = __ldg(tab + (u0 + 1) * (DH / 2) + lane), b1 = __ldg(tab + (u0 + 1) * (DH / 2) + 32 + lane);
          ra = make_float2(a1.x * sa[0].x + a1.y * sa[0].y, a1.y * sa[0].x - a1.x * sa[0].y);
          rb = make_float2(b1.x * sb[0].x + b1.y * sb[0].y, b1.y * sb[0].x - b1.x * sb[0].y);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (16 * k >= nv) break;
          float2 ca = sa[k], cb = sb[k];
#pragma unroll
          for (int h8 = 0; h8 < 2; ++h8) {
            // 8 keys at a time: all loads, then the turns, then all stores (r % 8 == e, kr0 a multiple of 8);
            // dim l of row r: box 0, dim l + 32: box 1, their partners + 64: boxes 2 and 3
            const int rb8 = 16 * k + 8 * h8;
            float v[8][4];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float* x = box0 + (rb8 + e) * 32 + swz[e];
              const bool in = rb8 + e < nv;
#pragma unroll
              for (int c = 0; c < 4; ++c) v[e][c] = in ? x[c * KT * 32] : 0.f;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float a0 = v[e][0], a1 = v[e][1], b0 = v[e][2], b1 = v[e][3];
              v[e][0] = a0 * ca.x + b0 * ca.y;
              v[e][2] = b0 * ca.x - a0 * ca.y;
              v[e][1] = a1 * cb.x + b1 * cb.y;
              v[e][3] = b1 * cb.x - a1 * cb.y;
              ca = make_float2(ca.x * ra.x - ca.y * ra.y, ca.y * ra.x + ca.x * ra.y);
              cb = make_float2(cb.x * rb.x - cb.y * rb.y, cb.y * rb.x + cb.x * rb.y);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float* x = box0 + (rb8 + e) * 32 + swz[e];
              if (rb8 + e < nv) {
#pragma unroll
                for (int c = 0; c < 4; ++c) x[c * KT * 32] = v[e][c];
              }
            }
          }
        }
      }
      fence_proxy_async();
      __syncwarp();
      if (!lead) {
        if (lane == 0) mbar_arrive(rope_done);
      } else {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(rope_done, n_it & 1, a.err))) { ok = false; break; }
        if (lane == 0) {
#pragma unroll
          for (int c = 0; c < 4; ++c) tma_reduce_add_2d(mdk, stg + c * (KT * 128), 32 * c, it.kv_row);
          bulk_commit();
          bulk_wait_read0();
          mbar_arrive(&kv_empty[kvs]);             // the producer may refill the slot
        }
        __syncwarp();
      }
      ++n_it;
    }
    if (lead && lane == 0) bulk_wait0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Per KV head h (one CTA each), over the documents some problem of head h
// selected (ascending): the problems that selected each document, ascending and
// contiguous in idx_prob[h], and one record per 128-key tile of those documents,
//   {first row of the tile in the K/V maps, t | keys << 16, place of the
//    document's problems in idx_prob[h], number of problems},
// in idx_items[h][0 .. idx_nitems[h]). cnt is [Hkv][n_docs] scratch.
constexpr int IDX_THREADS = 1024;

__global__ void __launch_bounds__(IDX_THREADS)
    bwd_index_kernel(const int32_t* sel, const int32_t* doc_len, const int64_t* doc_row, int64_t kv_rows, int* cnt,
                     int* idx_nitems, int4* idx_items, int* idx_prob, int n_docs, int n_kv_heads, int ph, int top_k,
                     int item_cap, int cap, int* err) {
  __shared__ int warp_a[IDX_THREADS / 32], warp_b[IDX_THREADS / 32];
  const int h = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  int* c = cnt + (int64_t)h * n_docs;
  for (int i = tid; i < n_docs; i += IDX_THREADS) c[i] = 0;
  __syncthreads();
  const int E = ph * top_k;
  for (int e = tid; e < E; e += IDX_THREADS) {
    const int j = sel[((int64_t)(e / top_k) * n_kv_heads + h) * top_k + e % top_k];
    if (j >= 0 && j < n_docs) atomicAdd(c + j, 1);
    else atomicCAS(err, 0, kErrInvalidArg);
  }
  __syncthreads();
  // block-wide exclusive scan of (tiles, selections) over contiguous document ranges
  const int per = (n_docs + IDX_THREADS - 1) / IDX_THREADS;
  const int d0 = min(n_docs, tid * per), d1 = min(n_docs, d0 + per);
  int nt = 0, sum = 0;
  for (int i = d0; i < d1; ++i) {
    const int v = c[i];
    if (v > 0) nt += (doc_len[i] + KT - 1) / KT;
    sum += v;
  }
  int xa = nt, xb = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, xa, o), b = __shfl_up_sync(0xffffffffu, xb, o);
    if (lane >= o) { xa += a; xb += b; }
  }
  if (lane == 31) { warp_a[wid] = xa; warp_b[wid] = xb; }
  __syncthreads();
  if (wid == 0) {
    int a = warp_a[lane], b = warp_b[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, a, o), y = __shfl_up_sync(0xffffffffu, b, o);
      if (lane >= o) { a += x; b += y; }
    }
    warp_a[lane] = a;    // inclusive over warps
    warp_b[lane] = b;
  }
  __syncthreads();
  int it = xa - nt + (wid > 0 ? warp_a[wid - 1] : 0);
  int off = xb - sum + (wid > 0 ? warp_b[wid - 1] : 0);
  for (int i = d0; i < d1; ++i) {
    const int v = c[i];
    if (v > 0) {
      const int len = doc_len[i];
      const int64_t row0 = (int64_t)h * kv_rows + doc_row[i];
      for (int t = 0; t * KT < len; ++t, ++it)
        if (it < item_cap)
          idx_items[(int64_t)h * item_cap + it] = make_int4((int)(row0 + (int64_t)t * KT), t | (min(KT, len - t * KT) << 16),
                                                            off, v);
    }
    c[i] = off;           // from here on: the next free place of document i in idx_prob
    off += v;
  }
  if (tid == IDX_THREADS - 1) idx_nitems[h] = min(it, item_cap);
  __syncthreads();
  // problems in ascending order, one per round (a problem's documents are distinct
  // unless the caller repeated one; repeats take separate places either way)
  for (int q = 0; q < ph; ++q) {
    if (tid < top_k) {
      const int j = sel[((int64_t)q * n_kv_heads + h) * top_k + tid];
      if (j >= 0 && j < n_docs) {
        const int pos = atomicAdd(c + j, 1);
        if (pos < cap) idx_prob[(int64_t)h * cap + pos] = q * n_kv_heads + h;
      }
    }
    __syncthreads();
  }
}

__global__ void to_bf16_kernel(const float4* __restrict__ in, uint2* __restrict__ out, int64_t n4) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = in[i];
    out[i] = make_uint2(pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
  }
}

}  // namespace

bool attend_bwd_tc_supported(int head_dim, int route_block, int top_k) {
  return head_dim == DH && route_block % RC == 0 && top_k >= 1;
}

int attend_bwd_tc_tile_rows() { return KT; }
int attend_bwd_tc_chunk_rows() { return RC; }

cudaError_t launch_attend_bwd_index(const int32_t* sel, const int32_t* doc_len, const int64_t* doc_row,
                                    int64_t kv_rows, int* cnt, int* idx_nitems, int4* idx_items, int* idx_prob,
                                    int n_docs, int n_kv_heads, int problems_per_head, int top_k, int item_cap,
                                    int cap, int* err, cudaStream_t s) {
  bwd_index_kernel<<<n_kv_heads, IDX_THREADS, 0, s>>>(sel, doc_len, doc_row, kv_rows, cnt, idx_nitems, idx_items,
                                                      idx_prob, n_docs, n_kv_heads, problems_per_head, top_k,
                                                      item_cap, cap, err);
  return cudaGetLastError();
}

cudaError_t launch_to_bf16(const float* in, uint16_t* out, int64_t n, int sms, cudaStream_t s) {
  const int64_t n4 = n / 4;
  const int64_t want = (n4 + 255) / 256;
  const int blocks = (int)std::min<int64_t>(want, (int64_t)sms * 8);
  to_bf16_kernel<<<blocks < 1 ? 1 : blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(in),
                                                         reinterpret_cast<uint2*>(out), n4);
  return cudaGetLastError();
}

cudaError_t launch_attend_bwd_dkdv_tc(const AttendBwdArgs& g, const AttendMaps& m, const CUtensorMap& q_map,
                                      const CUtensorMap& do_map, const AttendGradMaps& gm, int sms, cudaStream_t s) {
  auto kern = bwd_dkdv_tc_kernel;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_TOTAL);
  if (e != cudaSuccess) return e;
  const AttendArgs& a = g.a;
  if (a.n_kv_heads > MAX_HKV) return cudaErrorInvalidValue;
  const int LT = (a.local_len + KT - 1) / KT;
  const int64_t bound = (int64_t)a.batch * a.n_kv_heads * LT + (int64_t)a.n_kv_heads * g.idx_item_cap;
  if (bound >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  const int grid = (int)std::min<int64_t>(bound, sms);
  kern<<<grid, THREADS, SMEM_TOTAL, s>>>(q_map, do_map, m.bank_k, m.bank_v, m.loc_k, m.loc_v, gm.dk_bank, gm.dv_bank,
                                         gm.dk_loc, gm.dv_loc, g);
  return cudaGetLastError();
}

}  // namespace msa
