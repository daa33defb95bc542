// Internal launch interfaces of libmsa (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

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
  int64_t nch_total;
  int64_t chunk0;           // global index of the slice's first chunk
  int32_t n_chunks;         // chunks in the slice
  int32_t n_kv_heads;
  int32_t head_dim;
};
cudaError_t launch_bank_build(const BankBuildArgs& a, cudaStream_t s);

// q_r = mean of each routing block's routing queries, plus 1/||q_r||.
struct QrArgs {
  const uint16_t* qr;  // [B, Hkv, Tq, d_r]
  float* q_r;          // [B*nblk, Hkv, d_r]
  float* q_r_inv;      // [B*nblk, Hkv]
  int32_t batch, n_kv_heads, q_tokens, route_block, route_dim;
};
cudaError_t launch_qr_prep(const QrArgs& a, cudaStream_t s);

// Cosine of every (query row, chunk) and per-document max.
struct RouteArgs {
  const float* k_r;        // [Hkv][nch][d_r]
  const float* k_r_inv;    // [Hkv][nch]
  const int32_t* chunk_off;// [n_docs+1]
  const float* q_r;        // [rows][Hkv][d_r]
  const float* q_r_inv;    // [rows][Hkv]
  float* doc_scores;       // [rows][Hkv][n_docs]
  int64_t nch;
  int32_t rows, n_kv_heads, n_docs, route_dim;
};
cudaError_t launch_route(const RouteArgs& a, cudaStream_t s);

// Top-k per row of doc_scores, ordered (score desc, index asc).
struct TopkArgs {
  const float* scores;  // [rows][n]
  int32_t* idx;         // [rows][k]
  float* top_scores;    // [rows][k] or nullptr
  int32_t rows, n, k;
};
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s);

// Split-KV routed attention for problems with at most 16 query rows.
struct AttendArgs {
  const uint16_t* q;        // [B, Hq, Tq, d]
  const int32_t* sel;       // [B*nblk*Hkv][top_k]
  const int64_t* doc_row;   // [n_docs] first row of the document inside each head's K/V
  const int32_t* doc_len;   // [n_docs]
  const float2* gtab;       // [Lc][d/2] Global RoPE (cos, sin) at k_off + u
  float* part_o;            // [P][S][rows][d]   rows = G * route_block
  float* part_ml;           // [P][S][rows][2]   (running max in log2 units, sum)
  int* err;
  int64_t kv_rows;          // rows per head in the bank tensor map
  int32_t batch, n_q_heads, n_kv_heads, q_tokens, local_len, route_block, top_k, n_docs;
  int32_t n_splits;
  float scale_log2;         // log2(e) / sqrt(d)
};
struct AttendMaps {
  CUtensorMap bank_k, bank_v, loc_k, loc_v;
};
cudaError_t launch_attend_decode(const AttendArgs& a, const AttendMaps& m, int head_dim,
                                 cudaStream_t s);

struct MergeArgs {
  const float* part_o;
  const float* part_ml;
  float* out;               // [B, Hq, Tq, d]
  int32_t batch, n_q_heads, n_kv_heads, q_tokens, route_block, n_splits, head_dim;
};
cudaError_t launch_attend_merge(const MergeArgs& a, cudaStream_t s);

// Device pointers and sizes of a bank that the routing kernels read.
struct BankRouteView {
  const float* k_r;
  const float* k_r_inv;
  const int32_t* chunk_off;
  int64_t nch;
  int32_t n_docs, n_kv_heads, route_dim;
};

// Host-side helpers.
int attend_rows_per_problem(int group, int route_block);
int attend_tile_rows();  // keys per TMA tile of the decode attention kernel
size_t attend_smem_bytes(int head_dim);

}  // namespace msa

struct msa_bank;
// Fills `v` from a bank handle (no allocation, no CUDA call).
void msa_bank_route_view(const msa_bank* bank, msa::BankRouteView* v);
