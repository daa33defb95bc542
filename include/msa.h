/*
 * msa.h — C ABI of the routed sparse-attention step of Memory Sparse Attention
 * (MSA) on NVIDIA B200 (sm_100a).
 *
 * The step, as the pages state it:
 *   - a memory bank of documents; each document's per-token routing keys are
 *     compressed by chunk-mean pooling over 256-token chunks into K_r
 *     ("MSA架构：突破大模型记忆瓶颈的稀疏注意力技术", §2.1 item 2, §3.1);
 *   - the bank keys carry document-wise (Parallel) RoPE, positions restarting at
 *     0 in every document ("MSA (Memory Sparse Attention)", robocikowo.com,
 *     Komponenty: Document-wise RoPE; "MSA架构…", §2.2);
 *   - a router scores the query's routing vector against K_r by cosine
 *     similarity and keeps the top-k documents ("MSA架构…", §2.1 item 1;
 *     robocikowo.com, Komponenty: Router (Routing Projector); Hiperparametry:
 *     Top-k documents);
 *   - attention runs over the selected documents' K/V appended to the local
 *     context, whose queries and keys carry Global RoPE with a k-offset
 *     (robocikowo.com, Komponenty: Memory Sparse Attention Layer; Pułapki
 *     implementacyjne: RoPE consistency; Paradygmat wykonania).
 *
 * Readings this library takes where the pages are silent: a document's score
 * is the max of its chunks' cosines; a ragged last chunk is the mean of its
 * actual tokens; q_r of a routing block is the mean of its tokens' routing
 * queries; equal scores go to the lower document index; the Global-RoPE offset
 * is k_off = top_k * (longest document in the bank); local token u sits at
 * position k_off + u; the Tq queries are the last Tq local tokens; local key u
 * is visible to local query i iff u <= i; every selected document token is
 * visible to every query; softmax scale 1/sqrt(d); RoPE is rotate-half with
 * theta_i = base^(-2i/d); query head hq reads KV head hq / (Hq/Hkv).
 *
 * Conventions for every entry point:
 *   - All tensors are caller-owned, row-major, densely packed, of the bank's
 *     element type (msa_bank_config.dtype: bf16 unless stated) where no type is
 *     named, and live in device memory unless the argument says "host".
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are
 *     asynchronous on it; host arrays are read before the call returns.
 *   - Every call returns an msa_status and never throws. Argument errors are
 *     detected on the host before any launch. CUDA errors map to MSA_ERR_CUDA.
 *     Device-side bounded waits that expire set a flag read by
 *     msa_get_device_error() (MSA_ERR_TIMEOUT).
 *   - There is no CPU fallback: without a usable sm_100 device the calls that
 *     launch work return MSA_ERR_CUDA or MSA_ERR_UNSUPPORTED.
 *   - A bank belongs to the CUDA device that was current at msa_bank_create;
 *     make that device current for every call on it. Every call that launches
 *     work, waits or allocates returns MSA_ERR_INVALID_ARG, before touching any
 *     device, when another device is current (msa_bank_destroy switches to the
 *     bank's device itself and back). A bank is not safe for
 *     concurrent use: calls on one bank must not overlap in time (several banks
 *     may be used from several threads). The bank's workspace is shared by its
 *     calls, which are ordered on their streams; calls on one bank issued to two
 *     unordered streams may race on it.
 *   - Supported shapes: head_dim = route_dim in {64, 128}; n_q_heads a
 *     multiple of n_kv_heads; 1 <= top_k <= min(n_docs, 64); q_tokens a
 *     multiple of route_block; batch * (q_tokens / route_block) * n_kv_heads
 *     <= 65535. With G = n_q_heads / n_kv_heads, a routing block holds
 *     G * route_block query rows per KV head: up to 16 rows run the split-KV
 *     decode kernel, more rows the prefill kernels (tensor-memory tcgen05
 *     kernel when head_dim = 128, route_block is 64 or 128 and G * route_block
 *     is a multiple of 128; an mma.sync kernel otherwise).
 *   - Bank K/V may live in pinned host memory (MSA_KV_PINNED_HOST): msa_attend
 *     and msa_forward then read the step's selection back to the host, move
 *     every distinct selected (document, KV head) slab into a device staging
 *     pool (by default with one gather kernel that reads the page-locked K/V
 *     through its device mapping; else cudaMemcpyAsync on side streams, see
 *     msa_set_host_fetch), and attend from there. The whole K and V ranges must
 *     be page-locked (cudaHostAlloc, or cudaHostRegister'd). Those two calls
 *     synchronise the stream once per call and cannot be captured into a CUDA
 *     graph; msa_route never touches host K/V.
 */
#ifndef MSA_H_
#define MSA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1, /* a null pointer, an out-of-range size or index */
  MSA_ERR_UNSUPPORTED = 2, /* a valid shape this build does not implement */
  MSA_ERR_OOM = 3,         /* device or pinned allocation failed */
  MSA_ERR_CUDA = 4,        /* a CUDA runtime or driver call failed */
  MSA_ERR_TIMEOUT = 5,     /* a bounded device-side wait expired */
  MSA_ERR_HOST_TIER = 6    /* the pinned-host K/V tier could not serve a fetch */
} msa_status;

typedef enum {
  MSA_KV_DEVICE = 0,      /* bank K/V in device memory */
  MSA_KV_PINNED_HOST = 1  /* bank K/V in pinned (page-locked) host memory */
} msa_kv_location;

/* Precision of the routing keys the router reads (msa_set_router_precision). */
typedef enum {
  MSA_KR_F32 = 0,         /* normalised K_r as a bf16 high part + bf16 remainder (~16 significant bits) */
  MSA_KR_BF16 = 1         /* the bf16 high part only: half the router's bytes */
} msa_kr_precision;

/* How a pinned-host bank moves its selected slabs to the device (msa_set_host_fetch). */
typedef enum {
  MSA_FETCH_COPY_ENGINE = 0, /* cudaMemcpyAsync per run of host-contiguous slabs, on side streams */
  MSA_FETCH_SM_GATHER = 1    /* one kernel per stretch reads the mapped host K/V (the default) */
} msa_host_fetch;

/* Element type of a bank's tensors and of its steps' inputs (msa_bank_config.dtype). */
typedef enum {
  MSA_DTYPE_BF16 = 0,     /* bf16 storage, tensor-core arithmetic with fp32 accumulation (the default) */
  MSA_DTYPE_F32 = 1       /* fp32 storage and fp32 arithmetic throughout (CUDA cores; device-tier banks) */
} msa_dtype;

/* Opaque bank handle. Owns: K_r (fp32) and its inverse norms, document and
 * chunk offsets, RoPE tables, workspace, and (host tier) the device staging
 * pool, side stream and events. */
typedef struct msa_bank msa_bank;

typedef struct {
  int32_t n_docs;          /* number of documents, >= 1 */
  int32_t n_kv_heads;      /* Hkv, >= 1 */
  int32_t head_dim;        /* d: 64 or 128 */
  int32_t route_dim;       /* d_r: equal to head_dim */
  const int64_t* doc_lens; /* host [n_docs], each >= 1 token */
  float rope_base;         /* RoPE base, > 1 (10000 in the workloads) */
  int32_t kv_location;     /* msa_kv_location */
  const void* k;           /* bank keys   [Hkv, kv_rows, d]; Parallel RoPE already applied
                              (msa_build_bank applies it in place) */
  const void* v;           /* bank values [Hkv, kv_rows, d] */
  int64_t kv_rows;         /* rows per head in k/v; 0 means Ntok = sum(doc_lens) */
  const int64_t* doc_rows; /* host [n_docs] or NULL: first row of document j inside
                              each head's k/v; NULL means the prefix sums of doc_lens.
                              Several documents may share rows (an aliased pool). */
  int32_t dtype;           /* msa_dtype of k, v, the routing keys msa_build_bank pools and
                              every msa_query tensor (q, qr, local_k, local_v). 0 = bf16.
                              MSA_DTYPE_F32 keeps every value in fp32 end to end: Parallel
                              RoPE is stored in fp32 and attention runs in fp32 on the CUDA
                              cores (no bf16 rounding of the rotated query, keys or P);
                              device-tier banks and the forward calls only (pinned-host
                              banks and the backward return MSA_ERR_UNSUPPORTED). */
} msa_bank_config;

/* Creates a bank: validates the layout, computes document/chunk offsets and
 * the Parallel-RoPE table (angles in fp64), allocates K_r. Launches nothing
 * that reads k/v; the handle keeps the k/v pointers (caller-owned; they must
 * outlive the handle). On error *out is set to NULL. */
msa_status msa_bank_create(const msa_bank_config* cfg, msa_bank** out);

/* Frees everything the handle owns (synchronises the device first). NULL is a no-op. */
msa_status msa_bank_destroy(msa_bank* bank);

/* Offline bank build for documents [doc_begin, doc_end):
 *  - pools K_r[h, c] = mean of the per-token routing keys of chunk c over its
 *    actual tokens (fp32 accumulate, fp32 store) and 1/||K_r[h, c]||;
 *  - if k_slice != NULL, applies Parallel RoPE in place to k_slice (position of
 *    a token = its index inside its document), rounding to bf16.
 * r_slice: [Hkv][T][d_r] routing keys of those documents, where T = their total
 *   length and row 0 is the first token of doc_begin; head h starts at
 *   r_slice + h * r_head_stride elements (r_head_stride >= T).
 * k_slice: same layout for the keys, head stride k_head_stride (>= T); for a
 *   device bank, pass the bank's own k + doc_rows[doc_begin] * d with stride
 *   kv_rows. For a pinned-host bank, pass a device copy and copy it back.
 * Building in slices lets routing keys that do not fit in HBM stream through.
 * (robocikowo.com, Pułapki implementacyjne: encode offline, chunked mean pooling.) */
msa_status msa_build_bank(msa_bank* bank, int32_t doc_begin, int32_t doc_end,
                          const void* r_slice, int64_t r_head_stride,
                          void* k_slice, int64_t k_head_stride, void* stream);

/* Sizes and device pointers owned by the bank: K_r fp32 [Hkv, n_chunks, d_r],
 * inverse norms fp32 [Hkv, n_chunks] -- the compressed routing keys that stay in
 * GPU memory while the full K/V may live elsewhere ("MSA (Memory Sparse
 * Attention)", robocikowo.com, Komponenty: Router K_r in VRAM; "MSA架构…",
 * §2.1 item 2: one pooled key per 256-token chunk). n_chunks = sum over
 * documents of ceil(L_j / 256). Any output pointer may be NULL; the device
 * pointers stay valid until msa_bank_destroy. Host-only: MSA_ERR_INVALID_ARG for
 * a NULL bank, nothing else. */
msa_status msa_bank_info(const msa_bank* bank, int64_t* n_tokens, int64_t* n_chunks,
                         int64_t* max_doc_len, const float** k_r, const float** k_r_inv_norm);

/* One step's queries. */
typedef struct {
  int32_t batch;        /* B */
  int32_t n_q_heads;    /* Hq, a multiple of Hkv */
  int32_t q_tokens;     /* Tq: the last Tq local tokens are the queries */
  int32_t local_len;    /* Lc >= Tq */
  int32_t route_block;  /* Bq: query tokens per routing block; Tq % Bq == 0 */
  const void* q;        /* [B, Hq, Tq, d]   queries, no RoPE applied */
  const void* qr;       /* [B, Hkv, Tq, d_r] per-token routing queries */
  const void* local_k;  /* [B, Hkv, Lc, d]  local keys, no RoPE applied */
  const void* local_v;  /* [B, Hkv, Lc, d]  local values */
} msa_query;

/* Pre-allocates the workspace and Global-RoPE table for steps up to the given
 * sizes, so that later calls allocate nothing (required before capturing
 * calls into a CUDA graph). The pages describe no such call: it serves the
 * per-step routing + attention of "MSA (Memory Sparse Attention)",
 * robocikowo.com, Paradygmat wykonania, run back to back. `shape` carries the
 * step's sizes; its q / local_k / local_v may be NULL (routing only: the
 * attention workspace is not reserved). Same argument checks as msa_route /
 * msa_attend; MSA_ERR_OOM when the device memory cannot be allocated.
 * Synchronises the device when it has to grow the workspace. */
msa_status msa_reserve(msa_bank* bank, const msa_query* shape, int32_t top_k);

/* Router ("MSA架构…", §2.1 item 1: cosine top-k over the pooled routing keys;
 * robocikowo.com, Komponenty: Router / Routing Projector, and Hiperparametry:
 * top-k documents): q_r per (sequence, routing block, KV head) = mean of the
 * block's routing queries; score of chunk c = cos(q_r, K_r[h, c]); document
 * score = max over its chunks; selection = top_k documents, ordered by (score
 * desc, index asc). Scores are computed in fp32 with the normalised K_r read
 * as a bf16 high part plus remainder (msa_set_router_precision). q, local_k and
 * local_v of `q` are not read and may be NULL; qr must be 16-byte aligned.
 * MSA_ERR_INVALID_ARG for a NULL bank, q, qr or topk_idx, a shape outside the
 * supported set, or 1 <= top_k <= n_docs violated; MSA_ERR_UNSUPPORTED for
 * top_k > 64. Grows the bank's workspace on first use of a larger shape.
 * doc_scores:  [B, nblk, Hkv, n_docs] fp32, or NULL.
 * topk_idx:    [B, nblk, Hkv, top_k] int32 (required).
 * topk_scores: [B, nblk, Hkv, top_k] fp32, or NULL.  (nblk = Tq / Bq) */
msa_status msa_route(msa_bank* bank, const msa_query* q, int32_t top_k, float* doc_scores,
                     int32_t* topk_idx, float* topk_scores, void* stream);

/* Routed attention ("MSA (Memory Sparse Attention)", robocikowo.com,
 * Komponenty: Memory Sparse Attention Layer -- the selected documents' K/V are
 * appended to the local context and one softmax runs over both; Pułapki
 * implementacyjne: Global RoPE with a k-offset for the active context;
 * Paradygmat wykonania: only the k selected documents take part):
 * for query head hq at local index i = Lc - Tq + t,
 * out[b, hq, t] = softmax over { all tokens of the documents in
 * topk_idx[b, t / Bq, hq / G] (bank keys, Parallel RoPE) } and { local keys
 * u <= i with Global RoPE at k_off + u }, query with Global RoPE at k_off + i,
 * scale 1/sqrt(d), applied to the matching values. k_off = top_k * max_doc_len.
 * topk_idx: [B, nblk, Hkv, top_k] int32 in [0, n_docs) (checked on the device;
 *   an out-of-range index sets MSA_ERR_INVALID_ARG in the device error flag and
 *   that document is skipped).
 * out: [B, Hq, Tq, d] fp32. */
msa_status msa_attend(msa_bank* bank, const msa_query* q, int32_t top_k,
                      const int32_t* topk_idx, float* out, void* stream);

/* msa_attend that also writes each row's log-sum-exp, the state a training step
 * keeps for msa_attend_backward_saved (the layer trains end to end:
 * robocikowo.com, Komponenty):
 *   lse [B, Hq, Tq] fp32: log sum_j exp(s_j), natural log, over the row's key
 *   set, s_j = q_rot . k_j / sqrt(d) (so out = sum_j exp(s_j - lse) v_j).
 * out is bit for bit what msa_attend writes. Same shapes, errors and device-side
 * checks as msa_attend; MSA_ERR_INVALID_ARG for a NULL lse. */
msa_status msa_attend_lse(msa_bank* bank, const msa_query* q, int32_t top_k,
                          const int32_t* topk_idx, float* out, float* lse, void* stream);

/* Backward of msa_attend for the selection in topk_idx (the top-k routing is not
 * differentiated: the layer trains end to end on each step's selection,
 * "MSA (Memory Sparse Attention)", robocikowo.com, Komponenty). Gradients of
 * sum(d_out * out), with out = msa_attend(q, top_k, topk_idx):
 *   dq        [B, Hq, Tq, d]   fp32, written: the queries as msa_query takes them
 *                              (before Global RoPE);
 *   dlocal_k  [B, Hkv, Lc, d]  fp32, written: the local keys (before Global RoPE);
 *   dlocal_v  [B, Hkv, Lc, d]  fp32, written: the local values;
 *   dbank_k   [Hkv, kv_rows, d] fp32, ADDED TO: the bank keys before Parallel RoPE
 *                              (as msa_build_bank takes them); rows that several
 *                              documents share receive the sum;
 *   dbank_v   [Hkv, kv_rows, d] fp32, added to: the bank values.
 * d_out: [B, Hq, Tq, d] fp32. The call recomputes each row's softmax statistics
 * (it does not need the forward's output) and uses workspace for the RoPE'd
 * queries and local keys. Device-tier banks only (MSA_ERR_UNSUPPORTED for a
 * pinned-host bank). Pointers must be 16-byte aligned. */
msa_status msa_attend_backward(msa_bank* bank, const msa_query* q, int32_t top_k, const int32_t* topk_idx,
                               const float* d_out, float* dq, float* dlocal_k, float* dlocal_v,
                               float* dbank_k, float* dbank_v, void* stream);

/* msa_attend_backward given the forward's state: out and lse as msa_attend_lse
 * wrote them for the same q, top_k and topk_idx (both read, not written). Where
 * the backward runs on the tcgen05 tensor cores (head_dim 128, routing blocks of
 * 64 or 128 tokens, Hq / Hkv * route_block a multiple of 128, top_k <= 64) they
 * replace the forward recompute that msa_attend_backward performs; other shapes
 * recompute as msa_attend_backward does. Same outputs, layouts, errors and
 * accumulation; MSA_ERR_INVALID_ARG for a NULL or unaligned out or a NULL lse. */
msa_status msa_attend_backward_saved(msa_bank* bank, const msa_query* q, int32_t top_k, const int32_t* topk_idx,
                                     const float* out, const float* lse, const float* d_out, float* dq,
                                     float* dlocal_k, float* dlocal_v, float* dbank_k, float* dbank_v,
                                     void* stream);

/* One routed step as the pages run it per decoding step -- score the bank,
 * select top-k, fetch and attend ("MSA (Memory Sparse Attention)",
 * robocikowo.com, Paradygmat wykonania; Równoległość: selection then K/V fetch
 * in sequence within a step): msa_route followed by msa_attend on one stream;
 * topk_idx [B, nblk, Hkv, top_k] receives the selection, out [B, Hq, Tq, d]
 * fp32 the attention. On a pinned-host bank the fetch overlaps the routing of
 * the next micro-batch of sequences. For decode-sized problems (at most 16 query
 * rows per problem) on a device bf16 bank, the top-k and the attention start as
 * programmatic dependents of the kernel before them, so the attention's CTAs
 * for the local context run while the selection is made; the outputs are
 * identical, bit for bit, to msa_route followed by msa_attend. Errors as
 * msa_route and msa_attend. */
msa_status msa_forward(msa_bank* bank, const msa_query* q, int32_t top_k, int32_t* topk_idx,
                       float* out, void* stream);

/* msa_route without any allocation, for callers that must not allocate device
 * memory while they run: a process held to a fixed device-memory budget or
 * pool it may not grow, or a host that cannot accept the implicit device
 * synchronisation a cudaMalloc can bring. The pages describe no such entry
 * point; it exists for those callers only. Same arguments, checks, kernels,
 * device error flag and results as msa_route (the one routing path of the
 * library, given this scratch instead of the bank's workspace).
 * Scratch: q_r, 1/|q_r| and (when doc_scores is NULL) the document scores live
 * in one 4 MiB device array that libmsa defines at file scope; every GPU that
 * loads the library holds it until the process exits. A step needing more than
 * 4 MiB (rows * Hkv * (4*d_r + 4 + 4*n_docs) bytes, each part rounded up to 256)
 * returns MSA_ERR_UNSUPPORTED before any launch; pass doc_scores to keep the
 * scores out of the scratch. Nothing in the scratch needs to start at zero:
 * every word the kernels read was written earlier in the same call.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and caches it; make that first call before any stream
 * capture. All calls share the one array, so calls whose work overlaps on the
 * GPU (e.g. on two streams without ordering) race and corrupt each other. */
msa_status msa_route_noalloc(msa_bank* bank, const msa_query* q, int32_t top_k, float* doc_scores,
                             int32_t* topk_idx, float* topk_scores, void* stream);

/* ---- Memory Parallel: the bank's documents split into contiguous shards, one per
 * device ("MSA架构：突破大模型记忆瓶颈的稀疏注意力技术", §2.1 item 3: distributed
 * memory retrieval across GPUs through an AllGather; "MSA (Memory Sparse
 * Attention)", robocikowo.com, Równoległość: router scoring spread over devices,
 * then top-k and the K/V fetch in sequence). A step on S shards:
 *   1. each shard: msa_route -> its own top_k candidates (scores + GLOBAL indices);
 *   2. all-gather the candidates (NCCL, or plain copies when the shards share a GPU);
 *   3. every shard: msa_merge_topk -> the global top_k, identical on all shards and
 *      equal to what one bank holding every document would select;
 *   4. each shard: msa_attend_partial over the selected documents it holds, the
 *      sequence's owner shard with with_local = 1 -> (out_s, lse_s);
 *   5. gather the partials at the owner: msa_merge_partials -> the step's output.
 * The library moves no data between devices; the caller's collectives do. */

/* Marks `bank` as the shard holding documents [doc_base, doc_base + n_docs) of a
 * bank of n_docs_total documents whose longest document has max_doc_len_total
 * tokens. Afterwards: msa_route returns global indices (doc_base + local index);
 * attention calls read global indices, attend the ones in this shard and skip the
 * other shards' (MSA_ERR_INVALID_ARG in the device error flag only outside
 * [0, n_docs_total)); top_k may reach n_docs_total for attention (routing still
 * needs top_k <= this shard's n_docs); the Global-RoPE offset is
 * top_k * max_doc_len_total, the whole bank's. Every attention kernel takes
 * shard selections; the backward returns MSA_ERR_UNSUPPORTED on a shard.
 * MSA_ERR_INVALID_ARG for a NULL bank, doc_base < 0, a range past n_docs_total,
 * or max_doc_len_total below this shard's longest document. Call it before the
 * steps that use it (it is not ordered with work in flight). */
msa_status msa_bank_set_shard(msa_bank* bank, int32_t doc_base, int32_t n_docs_total, int64_t max_doc_len_total);

/* This shard's part of the routed attention for the selection topk_idx
 * [B, nblk, Hkv, top_k] (global indices; the merged selection): for every query
 * row, the softmax over the selected documents this bank holds -- and, when
 * with_local = 1, the causal local context -- applied to their values (out
 * [B, Hq, Tq, d] fp32), and that softmax's log-sum-exp (lse [B, Hq, Tq] fp32,
 * natural log of sum_j exp(q_rot . k_j / sqrt(d))). A row with no key here gets
 * out = 0 and lse = -inf. On a whole bank with with_local = 1 it equals
 * msa_attend_lse. MSA_ERR_INVALID_ARG for a NULL pointer or with_local not 0/1;
 * other errors as msa_attend. */
msa_status msa_attend_partial(msa_bank* bank, const msa_query* q, int32_t top_k, const int32_t* topk_idx,
                              int32_t with_local, float* out, float* lse, void* stream);

/* Merges n_parts candidate lists into the global top_k: cand_scores / cand_idx
 * [n_parts][rows][top_k] fp32 / int32 (the shards' msa_route outputs stacked part
 * after part, as an all-gather leaves them), each list ordered (score desc, index
 * asc) and no index in two lists -> topk_idx [rows][top_k] (and topk_scores, or
 * NULL): the first top_k of the union in the same order. rows = B * nblk * Hkv.
 * Device pointers, asynchronous on `stream`; no bank. MSA_ERR_INVALID_ARG for a
 * NULL pointer or a size < 1; MSA_ERR_UNSUPPORTED for n_parts > 64, top_k > 64 or
 * rows > 65535. The pages describe the gather, not this layout. */
msa_status msa_merge_topk(int32_t n_parts, int32_t rows, int32_t top_k, const float* cand_scores,
                          const int32_t* cand_idx, int32_t* topk_idx, float* topk_scores, void* stream);

/* Merges n_parts partial attentions over disjoint key sets into one softmax over
 * their union: part_out [n_parts][rows][head_dim] and part_lse [n_parts][rows]
 * fp32 (msa_attend_partial outputs stacked part after part) -> out [rows][head_dim]
 * = sum_s exp(part_lse[s] - L) part_out[s], L = log sum_s exp(part_lse[s]), and lse
 * [rows] = L (or NULL). Parts with lse = -inf weigh nothing; a row empty in every
 * part gets 0 and -inf. rows = B * Hq * Tq. Device pointers, asynchronous on
 * `stream`; no bank. MSA_ERR_INVALID_ARG for a NULL pointer or a size < 1. */
msa_status msa_merge_partials(int32_t n_parts, int64_t rows, int32_t head_dim, const float* part_out,
                              const float* part_lse, float* out, float* lse, void* stream);

/* One hop of Memory Interleave ("MSA (Memory Sparse Attention)", robocikowo.com,
 * Komponenty: generation of document identifiers and context expansion alternate,
 * so retrieval proceeds in several steps; "MSA架构…", §3.2: retrieval in rounds).
 * There is no generating model in this library, so the next hop's routing query
 * is a stated update in routing space (below). Per (sequence, routing block, KV
 * head):
 *   - the hop routes with q_r_in [B, Hkv, nblk, d_r] fp32 (NULL on the first hop:
 *     the block means of q->qr, as msa_route forms them);
 *   - it ranks only documents outside the context: context_idx
 *     [B, nblk, Hkv, n_ctx] int32 (NULL when n_ctx = 0), the documents earlier
 *     hops took;
 *   - ctx_out [B, nblk, Hkv, n_ctx + top_k] receives the expanded context: the
 *     n_ctx documents, then the hop's top_k new ones in (score desc, index asc)
 *     order (topk_scores [B, nblk, Hkv, top_k] fp32 their scores, or NULL);
 *   - q_r_out [B, Hkv, nblk, d_r] fp32 (or NULL) receives the next hop's query
 *     q/|q| + (1/top_k) sum_j kbar_j/|kbar_j| over the hop's documents, kbar_j the
 *     mean of document j's routing keys (its chunks' K_r weighted by their lengths).
 * Attention over the expanded context is msa_attend with top_k = n_ctx + top_k and
 * ctx_out as the selection (its Global-RoPE offset grows with the context). q->qr
 * must be given on every hop (q, local_k, local_v are not read). Whole banks only
 * (MSA_ERR_UNSUPPORTED on a shard). MSA_ERR_INVALID_ARG for a NULL ctx_out,
 * n_ctx < 0, n_ctx + top_k > n_docs or an unaligned q_r_in; a context index
 * outside [0, n_docs) raises MSA_ERR_INVALID_ARG in the device error flag. */
msa_status msa_interleave_route(msa_bank* bank, const msa_query* q, int32_t top_k, const float* q_r_in,
                                const int32_t* context_idx, int32_t n_ctx, int32_t* ctx_out, float* topk_scores,
                                float* q_r_out, void* stream);

/* Device-resident cache of selected K/V slabs for a pinned-host bank: the hot tier
 * of a hot/cold split ("MSA (Memory Sparse Attention)", robocikowo.com, Komponenty:
 * K_r in GPU memory, K/V in CPU RAM; "MSA：大模型高效推理的新突破，仅需2张A800显卡驱动1亿Token",
 * yicaiai.com: a hierarchical KV cache pool). `bytes` is the device memory budget
 * for K and V together; it is split into slots of max_doc_len rows (one (document,
 * KV head) slab each). With the cache on, msa_attend and msa_forward copy over PCIe
 * only the selected slabs that are not resident; a slab is replaced least recently
 * used first, never while the current step uses it. A step that selects more
 * distinct slabs than there are slots returns MSA_ERR_UNSUPPORTED. bytes = 0 turns
 * the cache off (the default: every step copies its selection). Synchronises the
 * device. MSA_ERR_INVALID_ARG for a NULL or device-tier bank or bytes < 0, MSA_ERR_OOM
 * if the slots cannot be allocated. */
msa_status msa_set_kv_cache(msa_bank* bank, int64_t bytes);

/* Host-tier statistics of the most recent msa_attend / msa_forward on a
 * pinned-host bank (any pointer may be NULL): distinct (document, KV head) slabs
 * the step selected, how many of them were already resident in the cache, and
 * the bytes copied over PCIe. */
msa_status msa_kv_cache_stats(const msa_bank* bank, int64_t* slabs, int64_t* hits, int64_t* bytes_copied);

/* Transport of a pinned-host bank's slab fetch ("MSA (Memory Sparse Attention)",
 * robocikowo.com, Pułapki implementacyjne: pinned memory and asynchronous
 * prefetch). MSA_FETCH_SM_GATHER (the default when msa_bank_create finds the
 * whole K and V ranges page-locked and mapped into the device's address space):
 * per planned stretch of slabs, one kernel on a side stream reads the host rows
 * with 16-byte loads through that mapping and writes the staging pool, so a step
 * of many small slabs pays no per-transfer cost (the bank keeps a job list of 32
 * bytes per selection entry, pinned and on the device). MSA_FETCH_COPY_ENGINE: one
 * cudaMemcpyAsync of K and one of V per run of host-contiguous slabs, round-robin
 * over the side streams. Both move the same bytes to the same staging rows, so
 * outputs are identical. Applies to later msa_attend / msa_forward calls;
 * synchronises the device. Returns MSA_ERR_INVALID_ARG for a NULL or device-tier
 * bank or another value, MSA_ERR_UNSUPPORTED for MSA_FETCH_SM_GATHER when the host
 * K/V is not mapped. msa_get_host_fetch reports the current transport. */
msa_status msa_set_host_fetch(msa_bank* bank, msa_host_fetch mode);
msa_status msa_get_host_fetch(const msa_bank* bank, msa_host_fetch* mode);

/* Precision of the routing keys the router reads (a 16-bit memory bank: the
 * nxmr.cn article "MSA技术解析为什么它能引爆AI社区", §2.2). MSA_KR_F32 (the
 * default): the normalised K_r is read as a bf16 high part plus a bf16
 * remainder, about 16 significant bits, so scores are the fp32 cosine to ~1e-5.
 * MSA_KR_BF16: only the bf16 high part, half the router's bytes; a score then
 * differs from the exact cosine by at most 2^-8 sum_i |q^_i k^_i| (the query
 * keeps full precision). Applies to every later msa_route / msa_forward /
 * msa_route_noalloc call on the bank. Returns MSA_ERR_INVALID_ARG for a NULL
 * bank or another value. */
msa_status msa_set_router_precision(msa_bank* bank, msa_kr_precision precision);

/* Failure-detection check of the device-side bounded waits (the pages describe
 * no such call): launches one small kernel on `stream` whose thread waits on an
 * mbarrier phase that nothing ever completes, with the same limit every kernel
 * of this library uses (mbarrier.try_wait polls that suspend up to 1 us each,
 * about 1.1 s in all). The wait gives
 * up, raises the bank's device error flag and the kernel returns normally: no
 * fault, and the context stays usable. A following msa_get_device_error()
 * returns MSA_ERR_TIMEOUT (and clears the flag). Returns MSA_ERR_INVALID_ARG for
 * a NULL bank, MSA_ERR_CUDA if the launch fails. */
msa_status msa_check_wait_timeout(msa_bank* bank, void* stream);

/* Synchronises `stream`, then returns and clears the device-side error flag
 * (MSA_OK, MSA_ERR_TIMEOUT or MSA_ERR_INVALID_ARG). */
msa_status msa_get_device_error(msa_bank* bank, void* stream);

/* Static description of a status code. */
const char* msa_status_string(msa_status status);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */
