// Internal launch interfaces of libmsa (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/msa.h"

namespace msa {

// Chunk-mean pooling of routing keys and in-place Parallel RoPE of bank keys
// for a contiguous run of chunks (documents [doc_begin, doc_end)).
struct BankBuildArgs {
  const uint16_t* r;        // bf16 routing keys, row 0 = first token of the slice
  int64_t r_head_stride;    // elements between heads
  uint16_t* k;              // bf16 keys (same row numbering) or nullptr
  int64_t k_head_stride;
  const int64_t* chunk_tok; // [n_chunks] first token of each chunk inside the bank
  int64_t tok_base;         // bank token that is row 0 of the slices
  const int32_t* chunk_len; // [n_chunks] tokens in the chunk (1..256)
  const int32_t* chunk_pos; // [n_chunks] position of its first token inside its document
  const float2* rope_tab;   // [max_doc_len][d/2] (cos, sin) of Parallel RoPE
  float* k_r;               // [Hkv][nch_total][d_r] (pointer at chunk 0 of the bank)
  float* k_r_inv;           // [Hkv][nch_total]
  uint16_t* k_hat_hi;       // [Hkv][nch_total][d_r] bf16 of K_r / |K_r|
  uint16_t* k_hat_lo;       // [Hkv][nch_total][d_r] bf16 of the remainder (hi + lo = K_r / |K_r|)
  int64_t nch_total;
  int64_t chunk0;           // global index of the slice's first chunk
  int32_t n_chunks;         // chunks in the slice
  int32_t n_kv_heads;
  int32_t head_dim;
  // fp32 banks: r32 / k32 take the place of r / k (same row numbering and strides)
  const float* r32;
  float* k32;
};
cudaError_t launch_bank_build(const BankBuildArgs& a, cudaStream_t s);

// q_r = mean of each routing block's routing queries, plus 1/||q_r||.
struct QrArgs {
  const uint16_t* qr;  // [B, Hkv, Tq, d_r] bf16 (or nullptr when qr32 is given)
  float* q_r;          // [B*nblk, Hkv, d_r]
  float* q_r_inv;      // [B*nblk, Hkv]
  int32_t batch, n_kv_heads, q_tokens, route_block, route_dim;
  const float* qr32;   // [B, Hkv, Tq, d_r] fp32 routing queries (fp32 banks), or nullptr
};
cudaError_t launch_qr_prep(const QrArgs& a, cudaStream_t s);

// Cosine of every (query row, chunk) and per-document max, on tensor cores:
// K_r / |K_r| is stored as bf16 hi + lo (tensor maps over [Hkv * nch, d_r]),
// q_r / |q_r| is split the same way, and the three products hi*hi + hi*lo +
// lo*hi carry the dot product to ~1e-5 relative.
struct RouteArgs {
  const int32_t* chunk_off;// [n_docs+1]
  const float* q_r;        // [rows][Hkv][d_r]   (used when qr == nullptr)
  const float* q_r_inv;    // [rows][Hkv]
  float* doc_scores;       // [rows][Hkv][n_docs]
  int64_t nch;
  int32_t rows, n_kv_heads, n_docs, route_dim;
  // Optional: compute q_r in the router from the bf16 routing queries
  // [B, Hkv, Tq, d_r] (rows = B * Tq / route_block); then q_r/q_r_inv are unused.
  const uint16_t* qr;
  int32_t q_tokens, route_block;
  int* err;                // device error flag for expired waits, or nullptr
  int32_t kr_bf16;         // 1: read only the bf16 high part of the normalised K_r (half the bytes)
  int32_t max_ctas_per_sm; // 0: as many as shared memory allows (3); fewer leaves room beside the router
};
// Largest routing block for which the router computes q_r itself.
constexpr int kRouteFuseMaxBlock = 4;
struct RouteMaps {
  CUtensorMap k_hat_hi, k_hat_lo;        // boxes of route_tile_rows() chunks x 64 dims
  CUtensorMap k_hat_hi128, k_hat_lo128;  // boxes of route_tc_tile_rows() chunks x 64 dims
};
cudaError_t launch_route(const RouteArgs& a, const RouteMaps& m, cudaStream_t s);
int route_tile_rows();
// tcgen05 router for more than 16 routing rows at d_r = 128 (q_r and 1/|q_r|
// precomputed by launch_qr_prep); same results up to summation order.
bool route_tc_supported(int route_dim, int rows);
int route_tc_tile_rows();
cudaError_t launch_route_tc(const RouteArgs& a, const RouteMaps& m, int sms, cudaStream_t s);

// Top-k per row of doc_scores, ordered (score desc, index asc).
struct TopkArgs {
  const float* scores;  // [rows][n]
  int32_t* idx;         // [rows][out_ld] (out_ld 0: k): idx_base + the document's index in the score
                        // row, written to columns [out_col, out_col + k)
  float* top_scores;    // [rows][k] or nullptr
  int32_t rows, n, k;
  int32_t idx_base;     // global index of the row's first document (a shard of a larger bank), else 0
  int32_t out_ld, out_col;
  int32_t pdl;          // launch as a programmatic dependent of the previous kernel on the stream
};
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s);
// path 0: the library's choice (the warp kernel for n <= 2048 and k <= 20); 1: one
// 512-thread block per row (radix select, any n, k <= 64); 2: one warp per row
// (n <= 2048, k <= 32). Same order, same output.
cudaError_t launch_topk_path(const TopkArgs& a, int path, cudaStream_t s);

// Split-KV routed attention for problems with at most 16 query rows.
struct AttendArgs {
  const uint16_t* q;        // [B, Hq, Tq, d]
  const int32_t* sel;       // [B*nblk*Hkv][top_k]
  const int64_t* doc_row;   // [n_docs] first row of the document inside each head's K/V
  const int64_t* sel_base;  // [P][top_k] or nullptr: row of each selected (document, head) slab in the
                            // K/V tensor maps (host tier: the device staging pool)
  const int32_t* doc_len;   // [n_docs]
  const float2* gtab;       // [Lc][d/2] Global RoPE (cos, sin) at k_off + u
  const float2* gstep;      // [d/2] (cos, sin) of the rotation by 512 / d positions
  float* part_o;            // [P][S][rows][d]   rows = G * route_block
  float* part_ml;           // [P][S][rows][2]   (running max in log2 units, sum)
  float* out;               // [B, Hq, Tq, d] fp32
  float* lse_out;           // [B, Hq, Tq] or nullptr: each row's log-sum-exp (natural log) of its
                            // logits q_rot . k / sqrt(d) over the row's key set
  int* counters;            // [P] split-completion counters, zero between calls
  int* err;
  int64_t kv_rows;          // rows per head in the bank tensor map
  int32_t batch, n_q_heads, n_kv_heads, q_tokens, local_len, route_block, top_k, n_docs;
  int32_t n_splits;
  float scale_log2;         // log2(e) / sqrt(d)
  // Memory Parallel (a bank that is one contiguous shard of a larger one): sel holds
  // global document indices; those in [doc_lo, doc_lo + n_docs) are this bank's
  // documents j - doc_lo, other indices in [0, n_docs_index) are skipped (another
  // shard's), anything else raises the error flag. with_local = 0 leaves the local
  // context out (another shard attends it). A whole bank: 0, n_docs, 1.
  int32_t doc_lo, n_docs_index, with_local;
  // Decode kernel: 0 cuts each problem's whole tile list (documents, then the local
  // context) into n_splits ranges of equal cost. n > 0 gives the local context splits
  // of its own: splits [0, n) cut the local tiles, splits [n, n_splits) the document
  // tiles. Those CTAs never read the selection, so with a programmatic dependent
  // launch (pdl), which puts them first, they run while the selection is still being
  // made; the document CTAs wait for it.
  int32_t n_local_splits;
  int32_t pdl;              // launch as a programmatic dependent of the previous kernel on the stream
};
struct AttendMaps {
  CUtensorMap bank_k, bank_v, loc_k, loc_v;
};
cudaError_t launch_attend_decode(const AttendArgs& a, const AttendMaps& m, int head_dim,
                                 cudaStream_t s);
// Many-row problems (G * route_block > 16); loc_k must map the RoPE'd local keys.
cudaError_t launch_attend_prefill(const AttendArgs& a, const AttendMaps& m, int head_dim, cudaStream_t s);
int attend_prefill_tile_rows();
// out[row] = Global RoPE of in[row] at local index offset + row % period (gtab row).
cudaError_t launch_rope_rows(const uint16_t* in, uint16_t* out, const float2* gtab, int64_t rows, int period,
                             int offset, int head_dim, cudaStream_t s);
// tcgen05/TMEM prefill for head_dim 128, routing blocks of 64 or 128 tokens and
// G * route_block a multiple of 128; loc_k must map the RoPE'd local keys and
// q_map the RoPE'd queries [B * Hq * Tq, 128] in boxes of 64 x 64.
bool attend_prefill_tc_supported(int head_dim, int group, int route_block);
int attend_prefill_tc_tile_rows();
cudaError_t launch_attend_prefill_tc(const AttendArgs& a, const AttendMaps& m, const CUtensorMap& q_map,
                                     cudaStream_t s);

// Host-side helpers.
int attend_tile_rows();               // keys per TMA tile of the decode attention kernel
int attend_max_splits();              // upper bound on n_splits
int attend_ctas_per_sm(int head_dim); // resident CTAs per SM (shared-memory bound)
size_t attend_smem_bytes(int head_dim);

// One CTA whose bounded wait on a never-completed mbarrier phase expires and
// raises kErrTimeout in *err.
cudaError_t launch_wait_timeout(int* err, cudaStream_t s);

// Backward of the routed attention (selection fixed). Row statistics and dQ by
// one kernel (it re-runs the forward for the log-sum-exp and dO . O), dK and
// dV by a second one (accumulated into the outputs with atomics).
struct AttendBwdArgs {
  AttendArgs a;              // as for the forward; maps: the bank K/V and the RoPE'd local K / local V
  const float* dout;         // [B, Hq, Tq, d]
  float* dq;                 // [B, Hq, Tq, d] written: gradient of the un-rotated queries
  float* lse2;               // [P][rows] log2-domain log-sum-exp of each row's scaled logits
  float* drow;               // [P][rows] dO . O of each row
  const uint16_t* q_rot;     // [B, Hq, Tq, d] queries with Global RoPE
  const float2* ptab;        // [max_doc_len][d/2] Parallel RoPE (cos, sin)
  float* dk_bank;            // [Hkv, kv_rows, d] += gradient of the bank keys before Parallel RoPE
  float* dv_bank;            // [Hkv, kv_rows, d] += gradient of the bank values
  float* dk_loc;             // [B, Hkv, Lc, d] += gradient of the local keys before Global RoPE
  float* dv_loc;             // [B, Hkv, Lc, d] += gradient of the local values
  // key-tile (tcgen05) dK/dV kernel only
  const int* idx_nitems;     // [Hkv] bank key tiles of the head's selected documents
  const int4* idx_items;     // [Hkv][idx_item_cap] {first K/V row, t | keys << 16, place in idx_prob, problems}
  const int* idx_prob;       // [Hkv][idx_cap] the problems that selected each document, ascending
  int idx_item_cap;          // bound on the key tiles of one head
  int idx_cap;               // selections per head (problems per head x top_k)
};
// fp32 gradient tensors [rows, 128] in boxes of 32 columns x 128 rows, 128-byte swizzle
struct AttendGradMaps {
  CUtensorMap dk_bank, dv_bank, dk_loc, dv_loc;
};
cudaError_t launch_attend_bwd_dq(const AttendBwdArgs& g, const AttendMaps& m, int head_dim, cudaStream_t s);
cudaError_t launch_attend_bwd_dkdv(const AttendBwdArgs& g, const AttendMaps& m, int head_dim, int max_tiles,
                                   cudaStream_t s);
int attend_bwd_tile_rows();  // keys per TMA box of both backward kernels
// tcgen05 dK/dV for head_dim 128 and routing blocks a multiple of 64 tokens: the
// maps take boxes of attend_bwd_tc_tile_rows() keys, q_map / do_map (RoPE'd
// queries, dO in bf16) boxes of attend_bwd_tc_chunk_rows() rows. The gradient
// outputs are added to (the local ones must be zeroed first); rows of a key tile
// past its document or context receive +0.
bool attend_bwd_tc_supported(int head_dim, int route_block, int top_k);
int attend_bwd_tc_tile_rows();
int attend_bwd_tc_chunk_rows();
cudaError_t launch_attend_bwd_index(const int32_t* sel, const int32_t* doc_len, const int64_t* doc_row,
                                    int64_t kv_rows, int* cnt, int* idx_nitems, int4* idx_items, int* idx_prob,
                                    int n_docs, int n_kv_heads, int problems_per_head, int top_k, int item_cap,
                                    int cap, int* err, cudaStream_t s);
cudaError_t launch_to_bf16(const float* in, uint16_t* out, int64_t n, int sms, cudaStream_t s);
// tcgen05 dQ for the shapes of attend_prefill_tc_supported (top_k <= 64), given
// lse2 and drow; maps as for launch_attend_prefill_tc, do_map like q_map over dO (bf16).
cudaError_t launch_attend_bwd_dq_tc(const AttendBwdArgs& g, const AttendMaps& m, const CUtensorMap& q_map,
                                    const CUtensorMap& do_map, cudaStream_t s);
// dO (fp32) -> bf16, drow[p][r] = dO . O and lse2[p][r] = lse[b, hq, t] * log2(e) of every
// query row (head_dim 128; lse is the forward's natural-log log-sum-exp).
cudaError_t launch_attend_bwd_prep(const float* dout, const float* out, const float* lse, uint16_t* dout_bf,
                                   float* drow, float* lse2, int batch, int n_q_heads, int n_kv_heads, int q_tokens,
                                   int route_block, int sms, cudaStream_t s);
cudaError_t launch_attend_bwd_dkdv_tc(const AttendBwdArgs& g, const AttendMaps& m, const CUtensorMap& q_map,
                                      const CUtensorMap& do_map, const AttendGradMaps& gm, int sms, cudaStream_t s);

// fp32 routed attention (banks of MSA_DTYPE_F32): the key set, masks and output of the
// bf16 kernels, with every operand and product in fp32 on the CUDA cores. One CTA per
// attend_f32_rows() query rows of a problem streams the problem's whole key list.
struct AttendF32Args {
  const float* q;           // [B, Hq, Tq, d], no RoPE
  const float* local_k;     // [B, Hkv, Lc, d], no RoPE
  const float* local_v;     // [B, Hkv, Lc, d]
  const float* bank_k;      // [Hkv, kv_rows, d], Parallel RoPE applied
  const float* bank_v;      // [Hkv, kv_rows, d]
  const int32_t* sel;       // [P][top_k]
  const int64_t* doc_row;   // [n_docs]
  const int32_t* doc_len;   // [n_docs]
  const float2* gtab;       // [Lc][d/2] Global RoPE (cos, sin) at k_off + u
  float* out;               // [B, Hq, Tq, d]
  float* lse_out;           // [B, Hq, Tq] or nullptr
  int* err;
  int64_t kv_rows;
  int32_t batch, n_q_heads, n_kv_heads, q_tokens, local_len, route_block, top_k, n_docs;
  float scale_log2;         // log2(e) / sqrt(d)
  int32_t doc_lo, n_docs_index, with_local;  // as AttendArgs
};
int attend_f32_rows();
cudaError_t launch_attend_f32(const AttendF32Args& a, int head_dim, cudaStream_t s);

// Memory Parallel merges. Candidates: n_parts lists of k (score, global index) per row,
// each ordered (score desc, index asc) and with indices disjoint between parts ->
// the first k of their union in the same order. Partials: softmax outputs and
// log-sum-exps over disjoint key sets -> the softmax over their union.
cudaError_t launch_merge_topk(int n_parts, int rows, int k, const float* cand_scores, const int32_t* cand_idx,
                              int32_t* idx, float* scores, cudaStream_t s);
cudaError_t launch_merge_partials(int n_parts, int64_t rows, int head_dim, const float* part_out,
                                  const float* part_lse, float* out, float* lse, cudaStream_t s);

// Memory Interleave. Context: the documents already in the context (ctx [rows_h][n_ctx],
// global indices) are copied to columns [0, n_ctx) of ctx_out [rows_h][ld_out] and their
// scores ([rows_h][n_docs], this bank's documents) set to -inf.
cudaError_t launch_interleave_context(const int32_t* ctx, int n_ctx, int64_t rows_h, int n_docs, int doc_lo,
                                      int n_docs_index, float* scores, int32_t* ctx_out, int ld_out, int* err,
                                      cudaStream_t s);
// Next routing query of a hop: q_r_out[b, h, blk] = q/|q| + (1/k) sum_j kbar_j/|kbar_j|
// over the hop's k documents (columns [sel_col, sel_col + k) of sel [rows][Hkv][sel_ld]),
// kbar_j = sum over document j's chunks of len_c * K_r[h, c].
struct InterleaveUpdateArgs {
  const float* q_r;         // [rows][Hkv][d_r] the hop's routing queries
  const float* q_r_inv;     // [rows][Hkv]
  const int32_t* sel;
  int32_t sel_ld, sel_col, k;
  const float* k_r;         // [Hkv][nch][d_r]
  const int32_t* chunk_off; // [n_docs + 1]
  const int32_t* chunk_len; // [nch]
  int64_t nch;
  int32_t rows, n_kv_heads, nblk, n_docs, doc_lo;
  float* q_r_out;           // [B][Hkv][nblk][d_r]
};
cudaError_t launch_interleave_update(const InterleaveUpdateArgs& a, int route_dim, cudaStream_t s);

// Pinned-host tier: one run of host-contiguous K/V rows and the staging rows it goes
// to; jobs ascend in piece0, the index of their first piece (host_gather_piece_rows
// rows of K and of V each) among all pieces of a launch.
struct HostGatherJob {
  int64_t src_row;  // first row in the host K / V ([Hkv * kv_rows, d])
  int64_t dst_row;  // first row in the staging pool
  int64_t rows;
  int64_t piece0;
};
int64_t host_gather_piece_rows(int head_dim);
// hk / hv: device mappings of the page-locked host K / V; dk / dv: the staging pool.
cudaError_t launch_host_gather(const HostGatherJob* jobs, int njobs, int64_t npieces, const void* hk, const void* hv,
                               void* dk, void* dv, int head_dim, int ctas, cudaStream_t s);

}  // namespace msa

// msa_route with its scratch supplied by the caller instead of the bank's workspace:
// `scratch` (256-byte aligned, `scratch_bytes` long) receives q_r [rows][Hkv][d_r],
// 1/|q_r| [rows][Hkv] and, when doc_scores is NULL, the document scores
// [rows][Hkv][n_docs], each part rounded up to 256 bytes (rows = B * Tq / Bq).
// The same checks, router choice and kernels as msa_route; MSA_ERR_UNSUPPORTED
// before any launch when the parts do not fit.
msa_status msa_route_with_scratch(msa_bank* bank, const msa_query* q, int32_t top_k, float* doc_scores,
                                  int32_t* topk_idx, float* topk_scores, void* scratch, size_t scratch_bytes,
                                  cudaStream_t st);
