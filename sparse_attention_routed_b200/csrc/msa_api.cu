// Host side of libmsa: argument validation, the bank handle, RoPE tables,
// TMA descriptors, workspace, and the C entry points declared in msa.h.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <list>
#include <mutex>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/msa.h"
#include "common.cuh"
#include "internal.h"

using namespace msa;

namespace {

constexpr int kChunk = 256;  // routing chunk ("MSA架构…" §2.1 item 2: 256-token chunks)
constexpr int kMaxTopK = 64;
constexpr int kMaxRows = 16;
constexpr size_t kCounterBytes = 65536 * sizeof(int);  // one split counter per problem (P <= 65535)

msa_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return MSA_OK;
  if (e == cudaErrorMemoryAllocation) return MSA_ERR_OOM;
  return MSA_ERR_CUDA;
}

#define MSA_CUDA(call)                                \
  do {                                                \
    cudaError_t e_ = (call);                          \
    if (e_ != cudaSuccess) return from_cuda(e_);      \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor [rows][d], boxes of box_rows rows x 64 elements (128 bytes), 128-byte swizzle.
msa_status make_map(CUtensorMap* map, const void* base, int64_t rows, int d, int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return MSA_ERR_CUDA;
  if (!aligned16(base) || rows <= 0 || rows >= (int64_t(1) << 31)) return MSA_ERR_INVALID_ARG;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MSA_OK : MSA_ERR_CUDA;
}

// fp32 [rows, d] in boxes of 32 columns x box_rows rows, 128-byte swizzle (TMA reduce-add targets)
msa_status make_map_f32(CUtensorMap* map, void* base, int64_t rows, int d, int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return MSA_ERR_CUDA;
  if (!aligned16(base) || rows <= 0 || rows >= (int64_t(1) << 31)) return MSA_ERR_INVALID_ARG;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 4};
  cuuint32_t box[2] = {32, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MSA_OK : MSA_ERR_CUDA;
}

// (cos, sin) of pos * base^(-2i/d) for positions p0 .. p0+n-1, angles in fp64
// reduced mod 2*pi before the fp32 rounding.
std::vector<float2> rope_table(int64_t p0, int64_t n, int d, double base) {
  std::vector<float2> t((size_t)n * (d / 2));
  const double two_pi = 6.283185307179586476925286766559;
  std::vector<double> inv(d / 2);
  for (int i = 0; i < d / 2; ++i) inv[i] = std::pow(base, -2.0 * i / d);
  for (int64_t p = 0; p < n; ++p)
    for (int i = 0; i < d / 2; ++i) {
      const double ang = std::fmod((double)(p0 + p) * inv[i], two_pi);
      t[(size_t)p * (d / 2) + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
    }
  return t;
}

template <typename T>
msa_status upload(T** dst, const std::vector<T>& src) {
  *dst = nullptr;
  if (src.empty()) return MSA_OK;
  MSA_CUDA(cudaMalloc(dst, src.size() * sizeof(T)));
  MSA_CUDA(cudaMemcpy(*dst, src.data(), src.size() * sizeof(T), cudaMemcpyHostToDevice));
  return MSA_OK;
}

// Device address of page-locked host memory [p, p + bytes), mapped as one range, or
// nullptr.
const void* mapped_host(const void* p, size_t bytes) {
  int dev = 0, can = 0;
  cudaGetDevice(&dev);
  if (cudaDeviceGetAttribute(&can, cudaDevAttrCanMapHostMemory, dev) != cudaSuccess || !can) return nullptr;
  cudaPointerAttributes a{}, z{};
  const char* last = static_cast<const char*>(p) + bytes - 1;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess || cudaPointerGetAttributes(&z, last) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost || z.type != cudaMemoryTypeHost || !a.devicePointer ||
      static_cast<const char*>(z.devicePointer) != static_cast<const char*>(a.devicePointer) + bytes - 1)
    return nullptr;
  return a.devicePointer;
}

}  // namespace

struct msa_bank {
  // configuration
  int n_docs = 0, hkv = 0, d = 0, dr = 0, kv_loc = 0;
  bool f32 = false;  // MSA_DTYPE_F32: fp32 tensors and fp32 arithmetic (attend_f32_kernel)
  // Memory Parallel: this bank holds documents [doc_lo, doc_lo + n_docs) of a bank of
  // n_docs_total documents whose longest is koff_len tokens (a whole bank: 0, n_docs, max_len)
  int doc_lo = 0, n_docs_total = 0;
  int64_t koff_len = 0;
  double base = 10000.0;
  const void* k = nullptr;
  const void* v = nullptr;
  int64_t kv_rows = 0, ntok = 0, nch = 0, max_len = 0;
  std::vector<int64_t> doc_lens, doc_off, doc_rows;
  std::vector<int32_t> chunk_off;
  int sms = 148;
  int device = 0;  // the CUDA device current at msa_bank_create; every launch happens there
  // device, owned
  int64_t* d_doc_row = nullptr;
  int32_t* d_doc_len = nullptr;
  int32_t* d_chunk_off = nullptr;
  int64_t* d_chunk_tok = nullptr;  // relative to the bank's first token
  int32_t* d_chunk_len = nullptr;
  int32_t* d_chunk_pos = nullptr;
  float2* d_ptab = nullptr;
  float* d_kr = nullptr;
  float* d_kr_inv = nullptr;
  uint16_t* d_khi = nullptr;  // bf16 K_r/|K_r| (hi), router operand
  uint16_t* d_klo = nullptr;  // bf16 remainder (lo)
  int* d_err = nullptr;
  // Global RoPE table cache
  float2* d_gtab = nullptr;
  int64_t gtab_koff = -1;
  int gtab_lc = 0;
  size_t gtab_cap = 0;
  // workspace
  uint8_t* ws = nullptr;
  size_t ws_cap = 0;
  // TMA descriptors of the bank K/V (device tier) and of the router operands
  CUtensorMap map_k{}, map_v{};      // boxes of the decode kernel's tile
  CUtensorMap map_k64{}, map_v64{};  // boxes of the mma.sync prefill kernel's tile
  CUtensorMap map_k128{}, map_v128{};  // boxes of the tcgen05 prefill kernel's tile
  RouteMaps route_maps{};
  // pinned-host K/V tier: selected slabs are copied into a device staging pool
#ifndef MSA_HOST_SIDE
#define MSA_HOST_SIDE 4
#endif
  static constexpr int kSide = MSA_HOST_SIDE;  // copies round-robin over several streams (copy engines)
#ifndef MSA_HOST_MICRO
#define MSA_HOST_MICRO 2
#endif
  static constexpr int kMicro = MSA_HOST_MICRO;  // micro-batches of msa_forward's fetch / attention pipeline
  cudaStream_t side[kSide] = {};
  cudaEvent_t ev_fetch[kSide] = {};
  cudaStream_t att = nullptr;        // attention stream of the pipelined forward
  cudaStream_t rb = nullptr;         // selection read-back, kept apart from the copy queues
  cudaEvent_t ev_route[kMicro] = {};
  cudaEvent_t ev_att = nullptr;
  int32_t* h_idx = nullptr;   // pinned copy of the selection
  int64_t* h_base = nullptr;  // pinned staging row of every selection entry
  int64_t* d_base = nullptr;  // device copy of h_base
  size_t sel_cap = 0;         // entries of h_idx / h_base / d_base
  // slabs move by an SM gather through the device mapping of the page-locked K/V
  // (MSA_FETCH_SM_GATHER) or by copy-engine transfers (MSA_FETCH_COPY_ENGINE)
#ifndef MSA_HOST_FETCH_DEFAULT
#define MSA_HOST_FETCH_DEFAULT MSA_FETCH_SM_GATHER
#endif
  const void* k_map = nullptr;  // device addresses of the host K / V, or nullptr: not mapped
  const void* v_map = nullptr;
  bool gather = false;
  msa::HostGatherJob* h_jobs = nullptr;  // pinned, sel_cap entries: the jobs of selection entries [e0, e1) start at e0
  msa::HostGatherJob* d_jobs = nullptr;
  std::vector<msa::HostGatherJob> jobs;  // the stretch being planned
  uint16_t* stage_k = nullptr;
  uint16_t* stage_v = nullptr;
  int64_t stage_cap = 0;      // rows of stage_k / stage_v
  int64_t last_fetch_bytes = 0;
  // device-resident slab cache (msa_set_kv_cache): stage_k / stage_v become slots of
  // max_len rows that keep their slab across steps
  bool cache_on = false;
  int64_t cache_slots = 0;
  std::unordered_map<int64_t, int64_t> cache_map;  // doc * Hkv + head -> slot
  std::vector<int64_t> slot_key;                   // -1: free
  std::vector<int64_t> slot_use;                   // step that last used the slot
  std::list<int64_t> lru;                          // slots, least recently used first
  std::vector<std::list<int64_t>::iterator> slot_it;
  int64_t step_no = 0;
  bool kr_bf16 = false;     // router reads only the bf16 high part of the normalised K_r
  int64_t st_slabs = 0, st_hits = 0;  // the last step's distinct slabs and cache hits
};

namespace {

void free_bank(msa_bank* b) {
  if (!b) return;
  cudaDeviceSynchronize();
  for (int i = 0; i < msa_bank::kSide; ++i) {
    if (b->side[i]) cudaStreamDestroy(b->side[i]);
    if (b->ev_fetch[i]) cudaEventDestroy(b->ev_fetch[i]);
  }
  for (int i = 0; i < msa_bank::kMicro; ++i)
    if (b->ev_route[i]) cudaEventDestroy(b->ev_route[i]);
  if (b->att) cudaStreamDestroy(b->att);
  if (b->rb) cudaStreamDestroy(b->rb);
  if (b->ev_att) cudaEventDestroy(b->ev_att);
  if (b->h_idx) cudaFreeHost(b->h_idx);
  if (b->h_base) cudaFreeHost(b->h_base);
  if (b->d_base) cudaFree(b->d_base);
  if (b->h_jobs) cudaFreeHost(b->h_jobs);
  if (b->d_jobs) cudaFree(b->d_jobs);
  if (b->stage_k) cudaFree(b->stage_k);
  if (b->stage_v) cudaFree(b->stage_v);
  void* ptrs[] = {b->d_doc_row, b->d_doc_len, b->d_chunk_off, b->d_chunk_tok, b->d_chunk_len,
                  b->d_chunk_pos, b->d_ptab, b->d_kr, b->d_kr_inv, b->d_khi, b->d_klo, b->d_err, b->d_gtab, b->ws};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  delete b;
}

struct StepShape {
  int B, Hq, Tq, Lc, Bq, G, nblk, rows, P, k;
};

// A bank's kernels, tensor maps and workspace belong to the device that was current
// when it was created: a call made with another device current is refused before
// anything is launched or allocated.
bool on_bank_device(const msa_bank* bank) {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess && dev == bank->device;
}

msa_status check_query(const msa_bank* bank, const msa_query* q, int top_k, StepShape* s, bool need_attn) {
  if (!bank || !q) return MSA_ERR_INVALID_ARG;
  if (!on_bank_device(bank)) return MSA_ERR_INVALID_ARG;
  if (q->batch < 1 || q->n_q_heads < 1 || q->q_tokens < 1 || q->local_len < 1 || q->route_block < 1)
    return MSA_ERR_INVALID_ARG;
  if (q->n_q_heads % bank->hkv) return MSA_ERR_INVALID_ARG;
  if (q->q_tokens > q->local_len || q->q_tokens % q->route_block) return MSA_ERR_INVALID_ARG;
  // routing ranks the bank's own documents; attention takes the selection of the whole
  // (possibly sharded) bank
  if (top_k < 1 || top_k > (need_attn ? bank->n_docs_total : bank->n_docs)) return MSA_ERR_INVALID_ARG;
  if (top_k > kMaxTopK) return MSA_ERR_UNSUPPORTED;
  if (!q->qr || !aligned16(q->qr)) return MSA_ERR_INVALID_ARG;
  s->B = q->batch;
  s->Hq = q->n_q_heads;
  s->Tq = q->q_tokens;
  s->Lc = q->local_len;
  s->Bq = q->route_block;
  s->G = q->n_q_heads / bank->hkv;
  s->nblk = q->q_tokens / q->route_block;
  s->rows = s->G * s->Bq;
  s->P = s->B * s->nblk * bank->hkv;
  s->k = top_k;
  if (need_attn) {
    if (!q->q || !q->local_k || !q->local_v) return MSA_ERR_INVALID_ARG;
    if (!aligned16(q->q) || !aligned16(q->local_k) || !aligned16(q->local_v)) return MSA_ERR_INVALID_ARG;
    if ((int64_t)s->B * bank->hkv * s->Lc >= (int64_t(1) << 31)) return MSA_ERR_UNSUPPORTED;
  }
  if ((int64_t)s->B * s->nblk > 65535 || s->P > 65535) return MSA_ERR_UNSUPPORTED;
  return MSA_OK;
}

// Splits per problem. Every split of a problem carries the same work, so the
// grid should fill whole waves of resident CTAs: among split counts that leave
// every warp at least ~4 tiles, take the one whose last wave is fullest
// (ties to fewer CTAs, which means fewer partials to merge).
int choose_splits(const msa_bank* bank, const StepShape& s) {
  const double avg_len = (double)bank->ntok / bank->n_docs;
  const int tile = attend_tile_rows();
  const int64_t tiles = (int64_t)s.k * (int64_t)std::ceil(avg_len / tile) + (s.Lc + tile - 1) / tile;
  const int64_t resident = (int64_t)bank->sms * attend_ctas_per_sm(bank->d);
  const int64_t s_max = std::max<int64_t>(1, std::min<int64_t>(attend_max_splits(), tiles / 16));
  int best = 1;
  double best_eff = -1.0;
  for (int64_t S = 1; S <= s_max; ++S) {
    const double waves = (double)(s.P * S) / resident;
    if (waves < 1.0 && S < s_max) continue;  // fill the machine at least once when possible
    const double eff = waves / std::ceil(waves);
    if (eff > best_eff + 0.01) {
      best_eff = eff;
      best = (int)S;
    }
  }
  return best;
}

struct Workspace {
  int* counters;
  float* q_r;
  float* q_r_inv;
  float* scores;
  int32_t* idx;
  float* part_o;
  float* part_ml;
  uint16_t* local_rot;  // prefill: local keys with Global RoPE applied
  uint16_t* q_rot;      // tcgen05 prefill: queries with Global RoPE applied
  size_t bytes;
};

size_t align_up(size_t x) { return (x + 255) & ~size_t(255); }

Workspace layout(const msa_bank* bank, const StepShape& s, int splits, uint8_t* base) {
  Workspace w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? base + off : nullptr;
    off += align_up(bytes);
    return p;
  };
  const size_t rows_route = (size_t)s.B * s.nblk;
  w.counters = (int*)take(kCounterBytes);  // always first: a fixed place that stays zero between calls
  w.q_r = (float*)take(rows_route * bank->hkv * bank->dr * 4);
  w.q_r_inv = (float*)take(rows_route * bank->hkv * 4);
  w.scores = (float*)take(rows_route * bank->hkv * bank->n_docs * 4);
  w.idx = (int32_t*)take((size_t)s.P * s.k * 4);
  const bool prefill = s.rows > kMaxRows && !bank->f32;
  const bool decode = s.rows <= kMaxRows && !bank->f32;
  w.part_o = (float*)take(decode ? (size_t)s.P * splits * s.rows * bank->d * 4 : 0);
  w.part_ml = (float*)take(decode ? (size_t)s.P * splits * s.rows * 2 * 4 : 0);
  w.local_rot = (uint16_t*)take(prefill ? (size_t)s.B * bank->hkv * s.Lc * bank->d * 2 : 0);
  const bool tc = prefill && attend_prefill_tc_supported(bank->d, s.G, s.Bq);
  w.q_rot = (uint16_t*)take(tc ? (size_t)s.B * s.Hq * s.Tq * bank->d * 2 : 0);
  w.bytes = off;
  return w;
}

bool capturing(cudaStream_t s) {
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  return cudaStreamIsCapturing(s, &st) == cudaSuccess && st != cudaStreamCaptureStatusNone;
}

// Grows the workspace; refuses while `s` is being captured (call msa_reserve first).
msa_status ensure_workspace(msa_bank* bank, size_t bytes, cudaStream_t s) {
  if (bytes <= bank->ws_cap) return MSA_OK;
  if (capturing(s)) return MSA_ERR_INVALID_ARG;
  if (bank->ws) {
    MSA_CUDA(cudaDeviceSynchronize());
    cudaFree(bank->ws);
    bank->ws = nullptr;
    bank->ws_cap = 0;
  }
  MSA_CUDA(cudaMalloc(&bank->ws, bytes));
  MSA_CUDA(cudaMemset(bank->ws, 0, bytes));
  bank->ws_cap = bytes;
  return MSA_OK;
}

msa_status ensure_gtab(msa_bank* bank, int64_t koff, int lc, cudaStream_t s) {
  if (bank->gtab_koff == koff && bank->gtab_lc >= lc) return MSA_OK;
  if (capturing(s)) return MSA_ERR_INVALID_ARG;
  std::vector<float2> t = rope_table(koff, lc, bank->d, bank->base);
  // one more row: the rotation by 512 / d positions, the distance between the keys of a
  // local tile that one lane of the decode kernel rotates (it steps the angles by it)
  const std::vector<float2> step = rope_table(512 / bank->d, 1, bank->d, bank->base);
  t.insert(t.end(), step.begin(), step.end());
  const size_t bytes = t.size() * sizeof(float2);
  if (bytes > bank->gtab_cap) {
    MSA_CUDA(cudaDeviceSynchronize());
    if (bank->d_gtab) cudaFree(bank->d_gtab);
    bank->d_gtab = nullptr;
    bank->gtab_cap = 0;
    MSA_CUDA(cudaMalloc(&bank->d_gtab, bytes));
    bank->gtab_cap = bytes;
  } else {
    MSA_CUDA(cudaDeviceSynchronize());  // an in-flight step may still read the old table
  }
  MSA_CUDA(cudaMemcpy(bank->d_gtab, t.data(), bytes, cudaMemcpyHostToDevice));
  bank->gtab_koff = koff;
  bank->gtab_lc = lc;
  return MSA_OK;
}

// Cosine of every routing row against every chunk and the per-document max into
// `scores` [rows][Hkv][n_docs]: from q_r / q_r_inv ([rows][Hkv][d_r], [rows][Hkv]),
// or, when `fuse`, with q_r formed inside the router from q->qr.
msa_status run_router(msa_bank* bank, const msa_query* q, const StepShape& s, const float* q_r,
                      const float* q_r_inv, float* scores, bool fuse, cudaStream_t st, int max_ctas_per_sm = 0) {
  RouteArgs ra{};
  ra.max_ctas_per_sm = max_ctas_per_sm;
  if (fuse) {
    ra.qr = (const uint16_t*)q->qr;
    ra.q_tokens = s.Tq;
    ra.route_block = s.Bq;
  }
  ra.chunk_off = bank->d_chunk_off;
  ra.q_r = q_r;
  ra.q_r_inv = q_r_inv;
  ra.doc_scores = scores;
  ra.nch = bank->nch;
  ra.rows = s.B * s.nblk;
  ra.n_kv_heads = bank->hkv;
  ra.n_docs = bank->n_docs;
  ra.route_dim = bank->dr;
  ra.err = bank->d_err;
  ra.kr_bf16 = bank->kr_bf16 ? 1 : 0;
  if (route_tc_supported(bank->dr, s.B * s.nblk)) {
    MSA_CUDA(launch_route_tc(ra, bank->route_maps, bank->sms, st));
  } else {
    MSA_CUDA(launch_route(ra, bank->route_maps, st));
  }
  return MSA_OK;
}

// The routing step. q_r / q_r_inv ([rows][Hkv][d_r], [rows][Hkv]) and score_scratch
// ([rows][Hkv][n_docs], used when doc_scores is NULL) are the caller's scratch.
// `overlap` (the decode router, with the decode attention queued right behind it on
// `st`): the top-k is a programmatic dependent of the router, and the router keeps to 2
// CTAs per SM, so that the attention (a programmatic dependent of the top-k) streams the
// local context with one CTA per SM beside the router.
msa_status route_into(msa_bank* bank, const msa_query* q, const StepShape& s, float* q_r, float* q_r_inv,
                      float* score_scratch, float* doc_scores, int32_t* idx, float* top_scores, cudaStream_t st,
                      bool overlap = false) {
  const bool tc = route_tc_supported(bank->dr, s.B * s.nblk);
  const bool fuse = !tc && !bank->f32 && s.Bq <= kRouteFuseMaxBlock;  // the router forms q_r itself
  overlap = overlap && fuse;
  if (!fuse) {
    QrArgs qa{bank->f32 ? nullptr : (const uint16_t*)q->qr, q_r, q_r_inv, s.B, bank->hkv, s.Tq, s.Bq, bank->dr,
              bank->f32 ? (const float*)q->qr : nullptr};
    MSA_CUDA(launch_qr_prep(qa, st));
  }
  float* scores = doc_scores ? doc_scores : score_scratch;
  msa_status rc = run_router(bank, q, s, q_r, q_r_inv, scores, fuse, st, overlap ? 2 : 0);
  if (rc != MSA_OK) return rc;
  TopkArgs ta{scores, idx, top_scores, s.P, bank->n_docs, s.k, bank->doc_lo};
  ta.pdl = overlap ? 1 : 0;
  MSA_CUDA(launch_topk(ta, st));
  return MSA_OK;
}

msa_status route_impl(msa_bank* bank, const msa_query* q, const StepShape& s, const Workspace& w,
                      float* doc_scores, int32_t* idx, float* top_scores, cudaStream_t st, bool overlap = false) {
  return route_into(bank, q, s, w.q_r, w.q_r_inv, w.scores, doc_scores, idx, top_scores, st, overlap);
}

// Pinned-host tier ("MSA (Memory Sparse Attention)", robocikowo.com, Komponenty:
// K_r in GPU memory, full K/V in CPU RAM; Pułapki implementacyjne: pinned memory
// and asynchronous prefetch). A step's selection is read back, every distinct
// (document, KV head) slab it names is moved from pinned host memory into the
// device staging pool on the bank's side streams -- by host_gather_kernel reading
// the mapped host K/V, or by cudaMemcpyAsync -- and the attention kernels read the
// pool. Slabs that are neighbours in host memory (the same head, one document
// right after the other) get neighbouring staging rows and travel as one run.
// Host-synchronising: not capturable.

// Side streams, events, the attention stream and the pinned selection buffers.
msa_status ensure_host_tier(msa_bank* bank, size_t entries) {
  if (!bank->side[0]) {
    for (int i = 0; i < msa_bank::kSide; ++i) {
      MSA_CUDA(cudaStreamCreateWithFlags(&bank->side[i], cudaStreamNonBlocking));
      MSA_CUDA(cudaEventCreateWithFlags(&bank->ev_fetch[i], cudaEventDisableTiming));
    }
    for (int i = 0; i < msa_bank::kMicro; ++i)
      MSA_CUDA(cudaEventCreateWithFlags(&bank->ev_route[i], cudaEventDisableTiming));
    MSA_CUDA(cudaStreamCreateWithFlags(&bank->att, cudaStreamNonBlocking));
    MSA_CUDA(cudaStreamCreateWithFlags(&bank->rb, cudaStreamNonBlocking));
    MSA_CUDA(cudaEventCreateWithFlags(&bank->ev_att, cudaEventDisableTiming));
  }
  if (entries > bank->sel_cap) {
    MSA_CUDA(cudaDeviceSynchronize());
    if (bank->h_idx) cudaFreeHost(bank->h_idx);
    if (bank->h_base) cudaFreeHost(bank->h_base);
    if (bank->d_base) cudaFree(bank->d_base);
    if (bank->h_jobs) cudaFreeHost(bank->h_jobs);
    if (bank->d_jobs) cudaFree(bank->d_jobs);
    bank->h_idx = nullptr;
    bank->h_base = nullptr;
    bank->d_base = nullptr;
    bank->h_jobs = bank->d_jobs = nullptr;
    bank->sel_cap = 0;
    if (cudaHostAlloc(&bank->h_idx, entries * 4, cudaHostAllocDefault) != cudaSuccess) return MSA_ERR_HOST_TIER;
    if (cudaHostAlloc(&bank->h_base, entries * 8, cudaHostAllocDefault) != cudaSuccess) return MSA_ERR_HOST_TIER;
    MSA_CUDA(cudaMalloc(&bank->d_base, entries * 8));
    if (bank->k_map) {
      const size_t jb = entries * sizeof(msa::HostGatherJob);
      if (cudaHostAlloc(&bank->h_jobs, jb, cudaHostAllocDefault) != cudaSuccess) return MSA_ERR_HOST_TIER;
      MSA_CUDA(cudaMalloc(&bank->d_jobs, jb));
    }
    bank->sel_cap = entries;
  }
  return MSA_OK;
}

// Staging pool of at least `rows` rows for K and for V (grows only; the caller
// has made sure no kernel still reads the old pool).
msa_status ensure_stage(msa_bank* bank, int64_t rows, cudaStream_t st) {
  if (rows >= (int64_t(1) << 31)) return MSA_ERR_UNSUPPORTED;
  if (rows <= bank->stage_cap) return MSA_OK;
  if (capturing(st)) return MSA_ERR_INVALID_ARG;
  MSA_CUDA(cudaDeviceSynchronize());
  if (bank->stage_k) cudaFree(bank->stage_k);
  if (bank->stage_v) cudaFree(bank->stage_v);
  bank->stage_k = bank->stage_v = nullptr;
  bank->stage_cap = 0;
  const size_t bytes = (size_t)rows * bank->d * 2;
  if (cudaMalloc(&bank->stage_k, bytes) != cudaSuccess || cudaMalloc(&bank->stage_v, bytes) != cudaSuccess)
    return MSA_ERR_OOM;
  bank->stage_cap = rows;
  return MSA_OK;
}

// One run of `rows` host-contiguous K/V rows, host row `src` to staging row `dst`:
// a job of the stretch's gather launch, or a copy-engine transfer each of K and V.
msa_status issue_rows(msa_bank* bank, int64_t src, int64_t dst, int64_t rows, int& stream_rr) {
  const size_t bytes = (size_t)rows * bank->d * 2;
  bank->last_fetch_bytes += 2 * (int64_t)bytes;
  if (bank->gather) {
    bank->jobs.push_back({src, dst, rows, 0});
    return MSA_OK;
  }
  const uint16_t* hk = static_cast<const uint16_t*>(bank->k);
  const uint16_t* hv = static_cast<const uint16_t*>(bank->v);
  if (cudaMemcpyAsync(bank->stage_k + dst * bank->d, hk + src * bank->d, bytes, cudaMemcpyHostToDevice,
                      bank->side[stream_rr++ % msa_bank::kSide]) != cudaSuccess ||
      cudaMemcpyAsync(bank->stage_v + dst * bank->d, hv + src * bank->d, bytes, cudaMemcpyHostToDevice,
                      bank->side[stream_rr++ % msa_bank::kSide]) != cudaSuccess)
    return MSA_ERR_HOST_TIER;
  return MSA_OK;
}

// Launches the gather of the jobs just planned for the stretch of selection entries
// that starts at e0, on side stream 0. The stretch has at least as many entries as
// jobs, so its jobs go to the job buffers' entries from e0 on, which no other stretch
// of the step uses; the previous step's launches are over before any plan is made.
msa_status flush_jobs(msa_bank* bank, size_t e0) {
  if (!bank->gather || bank->jobs.empty()) {
    bank->jobs.clear();
    return MSA_OK;
  }
  const int64_t pr = host_gather_piece_rows(bank->d);
  const int nj = (int)bank->jobs.size();
  msa::HostGatherJob* hj = bank->h_jobs + e0;
  int64_t pieces = 0;
  for (int i = 0; i < nj; ++i) {
    hj[i] = bank->jobs[i];
    hj[i].piece0 = pieces;
    pieces += (hj[i].rows + pr - 1) / pr;
  }
  bank->jobs.clear();
  MSA_CUDA(cudaMemcpyAsync(bank->d_jobs + e0, hj, nj * sizeof(msa::HostGatherJob), cudaMemcpyHostToDevice,
                           bank->side[0]));
  MSA_CUDA(launch_host_gather(bank->d_jobs + e0, nj, pieces, bank->k_map, bank->v_map, bank->stage_k, bank->stage_v,
                              bank->d, bank->sms, bank->side[0]));
  return MSA_OK;
}

// Staging plan of one stretch of selection entries [e0, e1) (bank->h_idx holds
// them): slabs not staged earlier in the step get rows in host-address order,
// runs of host-contiguous slabs are copied as one, and h_base[e] receives each
// entry's first staging row. `slot` and `rows` carry the step's earlier plans.
msa_status stage_entries(msa_bank* bank, int k, size_t e0, size_t e1, std::unordered_map<int64_t, int64_t>& slot,
                         int64_t& rows, int& stream_rr) {
  std::vector<std::pair<int64_t, int64_t>> fresh;  // (host row of the slab's first token, doc * Hkv + head)
  for (size_t e = e0; e < e1; ++e) {
    const int h = (int)((e / k) % bank->hkv);
    const int jg = bank->h_idx[e];
    const int j = jg - bank->doc_lo;  // a global index on a shard bank
    if (jg < 0 || jg >= bank->n_docs_total) return MSA_ERR_INVALID_ARG;
    if (j < 0 || j >= bank->n_docs) continue;  // another shard's document: nothing to stage
    const int64_t key = (int64_t)j * bank->hkv + h;
    if (slot.emplace(key, -1).second) fresh.emplace_back((int64_t)h * bank->kv_rows + bank->doc_rows[j], key);
  }
  bank->st_slabs += (int64_t)fresh.size();
  std::sort(fresh.begin(), fresh.end());
  size_t i = 0;
  while (i < fresh.size()) {
    // a run: each next slab starts where the previous one ends, inside the same head
    const int64_t src0 = fresh[i].first, dst0 = rows;
    int64_t len = 0;
    size_t r = i;
    for (; r < fresh.size(); ++r) {
      const int64_t key = fresh[r].second;
      const int j = (int)(key / bank->hkv), h = (int)(key % bank->hkv);
      if (r > i && (fresh[r].first != src0 + len || (src0 / bank->kv_rows) != h)) break;
      slot[key] = dst0 + len;
      len += bank->doc_lens[j];
    }
    if (rows + len > bank->stage_cap) return MSA_ERR_HOST_TIER;
    const msa_status rc = issue_rows(bank, src0, dst0, len, stream_rr);
    if (rc != MSA_OK) return rc;
    rows += len;
    i = r;
  }
  for (size_t e = e0; e < e1; ++e) {
    const int h = (int)((e / k) % bank->hkv);
    const int j = bank->h_idx[e] - bank->doc_lo;
    bank->h_base[e] = (j >= 0 && j < bank->n_docs) ? slot[(int64_t)j * bank->hkv + h] : 0;
  }
  return MSA_OK;
}

// Cache-mode plan of selection entries [e0, e1): a slab resident in a slot is a
// hit; a missing one takes the least recently used slot that the current step has
// not used and is copied into it. `step` maps the slabs already placed in this step.
msa_status stage_entries_cached(msa_bank* bank, int k, size_t e0, size_t e1,
                                std::unordered_map<int64_t, int64_t>& step, int& stream_rr) {
  for (size_t e = e0; e < e1; ++e) {
    const int h = (int)((e / k) % bank->hkv);
    const int jg = bank->h_idx[e];
    const int j = jg - bank->doc_lo;  // a global index on a shard bank
    if (jg < 0 || jg >= bank->n_docs_total) return MSA_ERR_INVALID_ARG;
    if (j < 0 || j >= bank->n_docs) {  // another shard's document
      bank->h_base[e] = 0;
      continue;
    }
    const int64_t key = (int64_t)j * bank->hkv + h;
    auto placed = step.find(key);
    if (placed != step.end()) {
      bank->h_base[e] = placed->second;
      continue;
    }
    ++bank->st_slabs;
    int64_t slot;
    auto c = bank->cache_map.find(key);
    if (c != bank->cache_map.end()) {
      slot = c->second;
      ++bank->st_hits;
    } else {
      slot = bank->lru.front();
      if (bank->slot_use[slot] == bank->step_no) return MSA_ERR_UNSUPPORTED;  // more slabs than slots
      if (bank->slot_key[slot] >= 0) bank->cache_map.erase(bank->slot_key[slot]);
      bank->cache_map[key] = slot;
      bank->slot_key[slot] = key;
      const int64_t src = (int64_t)h * bank->kv_rows + bank->doc_rows[j];
      const msa_status rc = issue_rows(bank, src, slot * bank->max_len, bank->doc_lens[j], stream_rr);
      if (rc != MSA_OK) return rc;
    }
    bank->slot_use[slot] = bank->step_no;
    bank->lru.splice(bank->lru.end(), bank->lru, bank->slot_it[slot]);
    const int64_t base = slot * bank->max_len;
    step[key] = base;
    bank->h_base[e] = base;
  }
  return MSA_OK;
}

// A new host-tier step: statistics restart, and the cache's "used by this step" marks.
void begin_host_step(msa_bank* bank) {
  ++bank->step_no;
  bank->st_slabs = bank->st_hits = 0;
  bank->last_fetch_bytes = 0;
}

// Upper bound of the staging rows a step can need (every entry a different slab).
int64_t stage_bound(const msa_bank* bank, const StepShape& s) { return (int64_t)s.P * s.k * bank->max_len; }

// `to` waits for everything issued so far on the side streams.
msa_status join_side(msa_bank* bank, cudaStream_t to) {
  for (int i = 0; i < msa_bank::kSide; ++i) {
    MSA_CUDA(cudaEventRecord(bank->ev_fetch[i], bank->side[i]));
    MSA_CUDA(cudaStreamWaitEvent(to, bank->ev_fetch[i], 0));
  }
  return MSA_OK;
}

// Whole-step fetch for msa_attend: returns the staging row of every selection
// entry in bank->d_base; `st` waits for the copies.
msa_status host_fetch(msa_bank* bank, const StepShape& s, const int32_t* idx_dev, cudaStream_t st) {
  const size_t n = (size_t)s.P * s.k;
  msa_status rc = ensure_host_tier(bank, n);
  if (rc != MSA_OK) return rc;
  MSA_CUDA(cudaMemcpyAsync(bank->h_idx, idx_dev, n * 4, cudaMemcpyDeviceToHost, st));
  MSA_CUDA(cudaStreamSynchronize(st));  // also retires every earlier step that read the staging pool
  if (!bank->cache_on && (rc = ensure_stage(bank, stage_bound(bank, s), st)) != MSA_OK) return rc;
  std::unordered_map<int64_t, int64_t> slot;
  slot.reserve(n * 2);
  int64_t rows = 0;
  int rr = 0;
  begin_host_step(bank);
  bank->jobs.clear();
  rc = bank->cache_on ? stage_entries_cached(bank, s.k, 0, n, slot, rr) : stage_entries(bank, s.k, 0, n, slot, rows, rr);
  // what was planned is moved even when the plan stops early: the cache already lists it
  const msa_status rg = flush_jobs(bank, 0);
  if (rc == MSA_OK) rc = rg;
  if (rc != MSA_OK) return rc;
  MSA_CUDA(cudaMemcpyAsync(bank->d_base, bank->h_base, n * 8, cudaMemcpyHostToDevice, bank->side[0]));
  return join_side(bank, st);
}

// `staged`: for a pinned-host bank whose selection the caller has already staged,
// the device table of staging rows (one per selection entry); NULL fetches here.
bool is_shard(const msa_bank* bank) { return bank->doc_lo != 0 || bank->n_docs_total != bank->n_docs; }

msa_status attend_impl(msa_bank* bank, const msa_query* q, const StepShape& s, int splits, const Workspace& w,
                       const int32_t* idx, float* out, cudaStream_t st, const int64_t* staged = nullptr,
                       float* lse_out = nullptr, int with_local = 1, bool overlap = false) {
  if (bank->f32) {
    AttendF32Args f{};
    f.q = (const float*)q->q;
    f.local_k = (const float*)q->local_k;
    f.local_v = (const float*)q->local_v;
    f.bank_k = (const float*)bank->k;
    f.bank_v = (const float*)bank->v;
    f.sel = idx;
    f.doc_row = bank->d_doc_row;
    f.doc_len = bank->d_doc_len;
    f.gtab = bank->d_gtab;
    f.out = out;
    f.lse_out = lse_out;
    f.err = bank->d_err;
    f.kv_rows = bank->kv_rows;
    f.batch = s.B;
    f.n_q_heads = s.Hq;
    f.n_kv_heads = bank->hkv;
    f.q_tokens = s.Tq;
    f.local_len = s.Lc;
    f.route_block = s.Bq;
    f.top_k = s.k;
    f.n_docs = bank->n_docs;
    f.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)bank->d));
    f.doc_lo = bank->doc_lo;
    f.n_docs_index = bank->n_docs_total;
    f.with_local = with_local;
    MSA_CUDA(launch_attend_f32(f, bank->d, st));
    return MSA_OK;
  }
  const bool prefill = s.rows > kMaxRows;
  const bool tc = prefill && attend_prefill_tc_supported(bank->d, s.G, s.Bq);
  const int box = tc ? attend_prefill_tc_tile_rows() : prefill ? attend_prefill_tile_rows() : attend_tile_rows();
  const int64_t lrows = (int64_t)s.B * bank->hkv * s.Lc;
  AttendMaps maps;
  const int64_t* sel_base = nullptr;
  if (bank->kv_loc == MSA_KV_PINNED_HOST) {
    msa_status rf = MSA_OK;
    if (!staged) {
      if ((rf = host_fetch(bank, s, idx, st)) != MSA_OK) return rf;
      staged = bank->d_base;
    }
    if ((rf = make_map(&maps.bank_k, bank->stage_k, bank->stage_cap, bank->d, box)) != MSA_OK) return rf;
    if ((rf = make_map(&maps.bank_v, bank->stage_v, bank->stage_cap, bank->d, box)) != MSA_OK) return rf;
    sel_base = staged;
  } else {
    maps.bank_k = tc ? bank->map_k128 : prefill ? bank->map_k64 : bank->map_k;
    maps.bank_v = tc ? bank->map_v128 : prefill ? bank->map_v64 : bank->map_v;
  }
  if (prefill)
    MSA_CUDA(launch_rope_rows((const uint16_t*)q->local_k, w.local_rot, bank->d_gtab, lrows, s.Lc, 0, bank->d, st));
  CUtensorMap q_map{};
  if (tc) {
    const int64_t qrows = (int64_t)s.B * s.Hq * s.Tq;
    MSA_CUDA(launch_rope_rows((const uint16_t*)q->q, w.q_rot, bank->d_gtab, qrows, s.Tq, s.Lc - s.Tq, bank->d, st));
    msa_status r0 = make_map(&q_map, w.q_rot, qrows, bank->d, 64);
    if (r0 != MSA_OK) return r0;
  }
  msa_status rc = make_map(&maps.loc_k, prefill ? (const void*)w.local_rot : q->local_k, lrows, bank->d, box);
  if (rc != MSA_OK) return rc;
  rc = make_map(&maps.loc_v, q->local_v, lrows, bank->d, box);
  if (rc != MSA_OK) return rc;
  AttendArgs a{};
  a.q = (const uint16_t*)q->q;
  a.sel = idx;
  a.doc_row = bank->d_doc_row;
  a.sel_base = sel_base;
  a.doc_len = bank->d_doc_len;
  a.gtab = bank->d_gtab;
  a.gstep = bank->d_gtab + (size_t)bank->gtab_lc * (bank->d / 2);
  a.part_o = w.part_o;
  a.part_ml = w.part_ml;
  a.out = out;
  a.counters = w.counters;
  a.err = bank->d_err;
  a.kv_rows = bank->kv_rows;
  a.batch = s.B;
  a.n_q_heads = s.Hq;
  a.n_kv_heads = bank->hkv;
  a.q_tokens = s.Tq;
  a.local_len = s.Lc;
  a.route_block = s.Bq;
  a.top_k = s.k;
  a.n_docs = bank->n_docs;
  a.n_splits = splits;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)bank->d));
  a.lse_out = lse_out;
  a.doc_lo = bank->doc_lo;
  a.n_docs_index = bank->n_docs_total;
  a.with_local = with_local;
  if (!prefill && with_local && splits >= 2) {
    // the local context's own splits, in proportion to its cost (a local tile costs
    // about two bank tiles: Global RoPE in shared memory), at least one on each side
    const int tile = attend_tile_rows();
    const double doc_tiles = (double)s.k * std::ceil((double)bank->ntok / bank->n_docs / tile);
    const double loc_cost = 2.0 * (double)((s.Lc + tile - 1) / tile);
    const int nls = (int)std::lround(splits * loc_cost / (loc_cost + doc_tiles));
    a.n_local_splits = std::max(1, std::min(splits - 1, nls));
    a.pdl = overlap ? 1 : 0;
  }
  if (tc) {
    MSA_CUDA(launch_attend_prefill_tc(a, maps, q_map, st));
  } else if (prefill) {
    MSA_CUDA(launch_attend_prefill(a, maps, bank->d, st));
  } else {
    MSA_CUDA(launch_attend_decode(a, maps, bank->d, st));
  }
  return MSA_OK;
}

}  // namespace

static size_t route_scratch_bytes(const msa_bank* bank, const StepShape& s, bool with_scores) {
  const size_t rows = (size_t)s.B * s.nblk;
  return align_up(rows * bank->hkv * bank->dr * sizeof(float)) + align_up(rows * bank->hkv * sizeof(float)) +
         (with_scores ? align_up(rows * bank->hkv * (size_t)bank->n_docs * sizeof(float)) : 0);
}

msa_status msa_route_with_scratch(msa_bank* bank, const msa_query* q, int32_t top_k, float* doc_scores,
                                  int32_t* topk_idx, float* topk_scores, void* scratch, size_t scratch_bytes,
                                  cudaStream_t st) {
  StepShape s;
  msa_status rc = check_query(bank, q, top_k, &s, false);
  if (rc != MSA_OK) return rc;
  if (!topk_idx) return MSA_ERR_INVALID_ARG;
  if (route_scratch_bytes(bank, s, !doc_scores) > scratch_bytes) return MSA_ERR_UNSUPPORTED;
  if (!scratch || (reinterpret_cast<uintptr_t>(scratch) & 255u)) return MSA_ERR_INVALID_ARG;
  const size_t rows = (size_t)s.B * s.nblk;
  uint8_t* p = static_cast<uint8_t*>(scratch);
  float* q_r = reinterpret_cast<float*>(p);
  float* q_inv = reinterpret_cast<float*>(p + align_up(rows * bank->hkv * bank->dr * sizeof(float)));
  float* scores = reinterpret_cast<float*>(p + align_up(rows * bank->hkv * bank->dr * sizeof(float)) +
                                           align_up(rows * bank->hkv * sizeof(float)));
  return route_into(bank, q, s, q_r, q_inv, scores, doc_scores, topk_idx, topk_scores, st);
}

// msa_forward on a pinned-host bank: the batch runs as up to kMicro
// micro-batches of sequences, so that the PCIe fetch overlaps the GPU work
// ("MSA (Memory Sparse Attention)", robocikowo.com, Pułapki implementacyjne:
// pinned memory and asynchronous prefetch). Every micro-batch's routing is
// queued on `st` at once; the host then takes the micro-batches in order: it
// reads one's selection back as soon as its routing is done (the next
// micro-batch's routing runs meanwhile), stages its slabs on the side streams,
// and queues its attention on the attention stream behind those copies, so that
// attention of micro-batch i runs while micro-batch i+1 is being copied. A slab
// selected by several micro-batches is copied once. `st` waits for the last
// attention.
msa_status forward_host(msa_bank* bank, const msa_query* q, const StepShape& s, int32_t* topk_idx, float* out,
                        cudaStream_t st) {
  const int M = std::min(s.B, msa_bank::kMicro);
  const int nb = (s.B + M - 1) / M;  // sequences per micro-batch (the last may hold fewer)
  StepShape sm = s;
  sm.B = nb;
  sm.P = nb * s.nblk * bank->hkv;
  const int splits = choose_splits(bank, sm);
  Workspace w = layout(bank, sm, splits, nullptr);
  msa_status rc = ensure_workspace(bank, w.bytes, st);
  if (rc != MSA_OK) return rc;
  if ((rc = ensure_gtab(bank, (int64_t)s.k * bank->koff_len, s.Lc, st)) != MSA_OK) return rc;
  w = layout(bank, sm, splits, bank->ws);
  const size_t n = (size_t)s.P * s.k;
  if ((rc = ensure_host_tier(bank, n)) != MSA_OK) return rc;
  if (!bank->cache_on && (rc = ensure_stage(bank, stage_bound(bank, s), st)) != MSA_OK) return rc;
  if (capturing(st)) return MSA_ERR_INVALID_ARG;

  const size_t d = bank->d;
  auto sub = [&](int b0, int bn, msa_query* qm, StepShape* sh) {
    *qm = *q;
    qm->batch = bn;
    qm->q = static_cast<const uint16_t*>(q->q) + (size_t)b0 * s.Hq * s.Tq * d;
    qm->qr = static_cast<const uint16_t*>(q->qr) + (size_t)b0 * bank->hkv * s.Tq * bank->dr;
    qm->local_k = static_cast<const uint16_t*>(q->local_k) + (size_t)b0 * bank->hkv * s.Lc * d;
    qm->local_v = static_cast<const uint16_t*>(q->local_v) + (size_t)b0 * bank->hkv * s.Lc * d;
    *sh = s;
    sh->B = bn;
    sh->P = bn * s.nblk * bank->hkv;
  };
  const size_t per_seq = (size_t)s.nblk * bank->hkv * s.k;  // selection entries per sequence
  for (int m = 0; m < M; ++m) {
    const int b0 = m * nb, bn = std::min(nb, s.B - b0);
    if (bn <= 0) break;
    msa_query qm;
    StepShape sh;
    sub(b0, bn, &qm, &sh);
    if ((rc = route_impl(bank, &qm, sh, w, nullptr, topk_idx + b0 * per_seq, nullptr, st)) != MSA_OK) return rc;
    MSA_CUDA(cudaEventRecord(bank->ev_route[m], st));
  }
  std::unordered_map<int64_t, int64_t> slot;
  slot.reserve(n * 2);
  int64_t rows = 0;
  int rr = 0;
  begin_host_step(bank);
  for (int m = 0; m < M; ++m) {
    const int b0 = m * nb, bn = std::min(nb, s.B - b0);
    if (bn <= 0) break;
    msa_query qm;
    StepShape sh;
    sub(b0, bn, &qm, &sh);
    const size_t e0 = (size_t)b0 * per_seq, e1 = e0 + (size_t)bn * per_seq;
    // the selection of micro-batch m (its routing is the last thing ev_route[m] waits for;
    // for m = 0 it also follows every earlier step's attention, which read the pool)
    MSA_CUDA(cudaStreamWaitEvent(bank->rb, bank->ev_route[m], 0));
    MSA_CUDA(cudaMemcpyAsync(bank->h_idx + e0, topk_idx + e0, (e1 - e0) * 4, cudaMemcpyDeviceToHost, bank->rb));
    MSA_CUDA(cudaStreamSynchronize(bank->rb));
    bank->jobs.clear();
    rc = bank->cache_on ? stage_entries_cached(bank, s.k, e0, e1, slot, rr)
                        : stage_entries(bank, s.k, e0, e1, slot, rows, rr);
    const msa_status rg = flush_jobs(bank, e0);
    if (rc == MSA_OK) rc = rg;
    if (rc != MSA_OK) return rc;
    MSA_CUDA(cudaMemcpyAsync(bank->d_base + e0, bank->h_base + e0, (e1 - e0) * 8, cudaMemcpyHostToDevice,
                             bank->side[0]));
    if ((rc = join_side(bank, bank->att)) != MSA_OK) return rc;
    MSA_CUDA(cudaStreamWaitEvent(bank->att, bank->ev_route[m], 0));
    if ((rc = attend_impl(bank, &qm, sh, splits, w, topk_idx + e0, out + (size_t)b0 * s.Hq * s.Tq * d, bank->att,
                          bank->d_base + e0)) != MSA_OK)
      return rc;
  }
  MSA_CUDA(cudaEventRecord(bank->ev_att, bank->att));
  MSA_CUDA(cudaStreamWaitEvent(st, bank->ev_att, 0));
  return MSA_OK;
}

extern "C" {

const char* msa_status_string(msa_status s) {
  switch (s) {
    case MSA_OK: return "ok";
    case MSA_ERR_INVALID_ARG: return "invalid argument";
    case MSA_ERR_UNSUPPORTED: return "unsupported shape or configuration";
    case MSA_ERR_OOM: return "out of memory";
    case MSA_ERR_CUDA: return "CUDA error";
    case MSA_ERR_TIMEOUT: return "device-side wait timed out";
    case MSA_ERR_HOST_TIER: return "host K/V tier error";
  }
  return "unknown status";
}

msa_status msa_bank_create(const msa_bank_config* cfg, msa_bank** out) {
  if (!out) return MSA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cfg || cfg->n_docs < 1 || cfg->n_kv_heads < 1 || !cfg->doc_lens) return MSA_ERR_INVALID_ARG;
  if ((cfg->head_dim != 64 && cfg->head_dim != 128) || cfg->route_dim != cfg->head_dim)
    return MSA_ERR_INVALID_ARG;
  if (!(cfg->rope_base > 1.0f)) return MSA_ERR_INVALID_ARG;
  if (cfg->kv_location != MSA_KV_DEVICE && cfg->kv_location != MSA_KV_PINNED_HOST) return MSA_ERR_INVALID_ARG;
  if (!cfg->k || !cfg->v || !aligned16(cfg->k) || !aligned16(cfg->v)) return MSA_ERR_INVALID_ARG;
  if (cfg->dtype != MSA_DTYPE_BF16 && cfg->dtype != MSA_DTYPE_F32) return MSA_ERR_INVALID_ARG;
  if (cfg->dtype == MSA_DTYPE_F32 && cfg->kv_location != MSA_KV_DEVICE) return MSA_ERR_UNSUPPORTED;

  msa_bank* b = new (std::nothrow) msa_bank();
  if (!b) return MSA_ERR_OOM;
  b->n_docs = cfg->n_docs;
  b->hkv = cfg->n_kv_heads;
  b->d = cfg->head_dim;
  b->dr = cfg->route_dim;
  b->base = cfg->rope_base;
  b->kv_loc = cfg->kv_location;
  b->f32 = cfg->dtype == MSA_DTYPE_F32;
  b->k = cfg->k;
  b->v = cfg->v;
  b->doc_lens.assign(cfg->doc_lens, cfg->doc_lens + cfg->n_docs);
  b->doc_off.assign(b->n_docs + 1, 0);
  b->chunk_off.assign(b->n_docs + 1, 0);
  for (int j = 0; j < b->n_docs; ++j) {
    const int64_t L = b->doc_lens[j];
    if (L < 1 || L >= (int64_t(1) << 30)) {
      delete b;
      return MSA_ERR_INVALID_ARG;
    }
    b->doc_off[j + 1] = b->doc_off[j] + L;
    const int64_t nc = b->chunk_off[j] + (L + kChunk - 1) / kChunk;
    if (nc >= (int64_t(1) << 31)) {
      delete b;
      return MSA_ERR_UNSUPPORTED;
    }
    b->chunk_off[j + 1] = (int32_t)nc;
    b->max_len = std::max(b->max_len, L);
  }
  b->ntok = b->doc_off[b->n_docs];
  b->nch = b->chunk_off[b->n_docs];
  b->n_docs_total = b->n_docs;
  b->koff_len = b->max_len;
  b->kv_rows = cfg->kv_rows > 0 ? cfg->kv_rows : b->ntok;
  b->doc_rows.resize(b->n_docs);
  for (int j = 0; j < b->n_docs; ++j) {
    b->doc_rows[j] = cfg->doc_rows ? cfg->doc_rows[j] : b->doc_off[j];
    if (b->doc_rows[j] < 0 || b->doc_rows[j] + b->doc_lens[j] > b->kv_rows) {
      delete b;
      return MSA_ERR_INVALID_ARG;
    }
  }
  if ((int64_t)b->hkv * b->kv_rows >= (int64_t(1) << 31)) {
    delete b;
    return MSA_ERR_UNSUPPORTED;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    delete b;
    return MSA_ERR_CUDA;
  }
  b->device = dev;
  cudaDeviceGetAttribute(&b->sms, cudaDevAttrMultiProcessorCount, dev);
  if (b->kv_loc == MSA_KV_PINNED_HOST) {
    const size_t kv_bytes = (size_t)b->hkv * b->kv_rows * b->d * 2;
    b->k_map = mapped_host(b->k, kv_bytes);
    b->v_map = b->k_map ? mapped_host(b->v, kv_bytes) : nullptr;
    if (!b->v_map) b->k_map = nullptr;
    b->gather = MSA_HOST_FETCH_DEFAULT == MSA_FETCH_SM_GATHER && b->k_map;
  }

  // chunk table
  std::vector<int64_t> ctok(b->nch);
  std::vector<int32_t> clen(b->nch), cpos(b->nch), dlen(b->n_docs);
  for (int j = 0; j < b->n_docs; ++j) {
    dlen[j] = (int32_t)b->doc_lens[j];
    for (int c = b->chunk_off[j]; c < b->chunk_off[j + 1]; ++c) {
      const int64_t s = (int64_t)(c - b->chunk_off[j]) * kChunk;
      ctok[c] = b->doc_off[j] + s;
      clen[c] = (int32_t)std::min<int64_t>(kChunk, b->doc_lens[j] - s);
      cpos[c] = (int32_t)s;
    }
  }
  msa_status rc = MSA_OK;
  auto fail = [&](msa_status r) {
    free_bank(b);
    return r;
  };
  if ((rc = upload(&b->d_doc_row, b->doc_rows)) != MSA_OK) return fail(rc);
  if ((rc = upload(&b->d_doc_len, dlen)) != MSA_OK) return fail(rc);
  if ((rc = upload(&b->d_chunk_off, b->chunk_off)) != MSA_OK) return fail(rc);
  if ((rc = upload(&b->d_chunk_tok, ctok)) != MSA_OK) return fail(rc);
  if ((rc = upload(&b->d_chunk_len, clen)) != MSA_OK) return fail(rc);
  if ((rc = upload(&b->d_chunk_pos, cpos)) != MSA_OK) return fail(rc);
  if ((rc = upload(&b->d_ptab, rope_table(0, b->max_len, b->d, b->base))) != MSA_OK) return fail(rc);
  if (cudaMalloc(&b->d_kr, (size_t)b->hkv * b->nch * b->dr * 4) != cudaSuccess) return fail(MSA_ERR_OOM);
  if (cudaMalloc(&b->d_kr_inv, (size_t)b->hkv * b->nch * 4) != cudaSuccess) return fail(MSA_ERR_OOM);
  if (cudaMalloc(&b->d_khi, (size_t)b->hkv * b->nch * b->dr * 2) != cudaSuccess) return fail(MSA_ERR_OOM);
  if (cudaMalloc(&b->d_klo, (size_t)b->hkv * b->nch * b->dr * 2) != cudaSuccess) return fail(MSA_ERR_OOM);
  if ((rc = make_map(&b->route_maps.k_hat_hi, b->d_khi, (int64_t)b->hkv * b->nch, b->dr, route_tile_rows())) != MSA_OK)
    return fail(rc);
  if ((rc = make_map(&b->route_maps.k_hat_lo, b->d_klo, (int64_t)b->hkv * b->nch, b->dr, route_tile_rows())) != MSA_OK)
    return fail(rc);
  if ((rc = make_map(&b->route_maps.k_hat_hi128, b->d_khi, (int64_t)b->hkv * b->nch, b->dr,
                     route_tc_tile_rows())) != MSA_OK)
    return fail(rc);
  if ((rc = make_map(&b->route_maps.k_hat_lo128, b->d_klo, (int64_t)b->hkv * b->nch, b->dr,
                     route_tc_tile_rows())) != MSA_OK)
    return fail(rc);
  if (cudaMalloc(&b->d_err, sizeof(int)) != cudaSuccess) return fail(MSA_ERR_OOM);
  if (cudaMemset(b->d_err, 0, sizeof(int)) != cudaSuccess) return fail(MSA_ERR_CUDA);
  if (b->kv_loc == MSA_KV_DEVICE && !b->f32) {  // bf16 tensor maps of the bank K/V
    if ((rc = make_map(&b->map_k, b->k, (int64_t)b->hkv * b->kv_rows, b->d, attend_tile_rows())) != MSA_OK) return fail(rc);
    if ((rc = make_map(&b->map_v, b->v, (int64_t)b->hkv * b->kv_rows, b->d, attend_tile_rows())) != MSA_OK) return fail(rc);
    if ((rc = make_map(&b->map_k64, b->k, (int64_t)b->hkv * b->kv_rows, b->d, attend_prefill_tile_rows())) != MSA_OK)
      return fail(rc);
    if ((rc = make_map(&b->map_v64, b->v, (int64_t)b->hkv * b->kv_rows, b->d, attend_prefill_tile_rows())) != MSA_OK)
      return fail(rc);
    if ((rc = make_map(&b->map_k128, b->k, (int64_t)b->hkv * b->kv_rows, b->d, attend_prefill_tc_tile_rows())) !=
        MSA_OK)
      return fail(rc);
    if ((rc = make_map(&b->map_v128, b->v, (int64_t)b->hkv * b->kv_rows, b->d, attend_prefill_tc_tile_rows())) !=
        MSA_OK)
      return fail(rc);
  }
  *out = b;
  return MSA_OK;
}

msa_status msa_bank_destroy(msa_bank* bank) {
  if (!bank) return MSA_OK;
  // free on the bank's own device, whichever device the caller has current
  int cur = -1;
  const bool other = cudaGetDevice(&cur) == cudaSuccess && cur != bank->device;
  if (other) cudaSetDevice(bank->device);
  free_bank(bank);
  if (other) cudaSetDevice(cur);
  return MSA_OK;
}

// Strides are in rows; a row is d * 2 >= 128 bytes, so every head of an aligned slice stays aligned.
msa_status msa_build_bank(msa_bank* bank, int32_t doc_begin, int32_t doc_end, const void* r_slice,
                          int64_t r_head_stride, void* k_slice, int64_t k_head_stride, void* stream) {
  if (!bank || (!r_slice && !k_slice)) return MSA_ERR_INVALID_ARG;
  if (!on_bank_device(bank)) return MSA_ERR_INVALID_ARG;
  if (doc_begin < 0 || doc_end > bank->n_docs || doc_begin >= doc_end) return MSA_ERR_INVALID_ARG;
  const int64_t T = bank->doc_off[doc_end] - bank->doc_off[doc_begin];
  if (r_slice && (r_head_stride < T || !aligned16(r_slice))) return MSA_ERR_INVALID_ARG;
  if (k_slice && (k_head_stride < T || !aligned16(k_slice))) return MSA_ERR_INVALID_ARG;
  const int64_t c0 = bank->chunk_off[doc_begin], c1 = bank->chunk_off[doc_end];
  if (c1 - c0 >= (int64_t(1) << 31) / bank->hkv) return MSA_ERR_UNSUPPORTED;
  BankBuildArgs a{};
  if (bank->f32) {
    a.r32 = (const float*)r_slice;
    a.k32 = (float*)k_slice;
  } else {
    a.r = (const uint16_t*)r_slice;
    a.k = (uint16_t*)k_slice;
  }
  a.r_head_stride = r_head_stride * bank->dr;
  a.tok_base = bank->doc_off[doc_begin];
  a.k_head_stride = k_head_stride * bank->d;
  a.chunk_tok = bank->d_chunk_tok + c0;
  a.chunk_len = bank->d_chunk_len + c0;
  a.chunk_pos = bank->d_chunk_pos + c0;
  a.rope_tab = bank->d_ptab;
  a.k_r = bank->d_kr;
  a.k_r_inv = bank->d_kr_inv;
  a.k_hat_hi = bank->d_khi;
  a.k_hat_lo = bank->d_klo;
  a.nch_total = bank->nch;
  a.chunk0 = c0;
  a.n_chunks = (int32_t)(c1 - c0);
  a.n_kv_heads = bank->hkv;
  a.head_dim = bank->d;
  return from_cuda(launch_bank_build(a, (cudaStream_t)stream));
}

msa_status msa_bank_info(const msa_bank* bank, int64_t* n_tokens, int64_t* n_chunks, int64_t* max_doc_len,
                         const float** k_r, const float** k_r_inv_norm) {
  if (!bank) return MSA_ERR_INVALID_ARG;
  if (n_tokens) *n_tokens = bank->ntok;
  if (n_chunks) *n_chunks = bank->nch;
  if (max_doc_len) *max_doc_len = bank->max_len;
  if (k_r) *k_r = bank->d_kr;
  if (k_r_inv_norm) *k_r_inv_norm = bank->d_kr_inv;
  return MSA_OK;
}

msa_status msa_reserve(msa_bank* bank, const msa_query* shape, int32_t top_k) {
  StepShape s;
  const bool attn = shape && shape->q && shape->local_k && shape->local_v;
  msa_status rc = check_query(bank, shape, top_k, &s, attn);
  if (rc != MSA_OK) return rc;
  const int splits = choose_splits(bank, s);
  if ((rc = ensure_workspace(bank, layout(bank, s, splits, nullptr).bytes, nullptr)) != MSA_OK) return rc;
  return ensure_gtab(bank, (int64_t)top_k * bank->koff_len, s.Lc, nullptr);
}

msa_status msa_route(msa_bank* bank, const msa_query* q, int32_t top_k, float* doc_scores, int32_t* topk_idx,
                     float* topk_scores, void* stream) {
  StepShape s;
  msa_status rc = check_query(bank, q, top_k, &s, false);
  if (rc != MSA_OK) return rc;
  if (!topk_idx) return MSA_ERR_INVALID_ARG;
  const int splits = 1;
  Workspace w = layout(bank, s, splits, nullptr);
  if ((rc = ensure_workspace(bank, w.bytes, (cudaStream_t)stream)) != MSA_OK) return rc;
  w = layout(bank, s, splits, bank->ws);
  return route_impl(bank, q, s, w, doc_scores, topk_idx, topk_scores, (cudaStream_t)stream);
}

msa_status msa_attend(msa_bank* bank, const msa_query* q, int32_t top_k, const int32_t* topk_idx, float* out,
                      void* stream) {
  StepShape s;
  msa_status rc = check_query(bank, q, top_k, &s, true);
  if (rc != MSA_OK) return rc;
  if (!topk_idx || !out) return MSA_ERR_INVALID_ARG;
  const int splits = choose_splits(bank, s);
  Workspace w = layout(bank, s, splits, nullptr);
  if ((rc = ensure_workspace(bank, w.bytes, (cudaStream_t)stream)) != MSA_OK) return rc;
  if ((rc = ensure_gtab(bank, (int64_t)top_k * bank->koff_len, s.Lc, (cudaStream_t)stream)) != MSA_OK) return rc;
  w = layout(bank, s, splits, bank->ws);
  return attend_impl(bank, q, s, splits, w, topk_idx, out, (cudaStream_t)stream);
}

msa_status msa_attend_lse(msa_bank* bank, const msa_query* q, int32_t top_k, const int32_t* topk_idx, float* out,
                          float* lse, void* stream) {
  StepShape s;
  msa_status rc = check_query(bank, q, top_k, &s, true);
  if (rc != MSA_OK) return rc;
  if (!topk_idx || !out || !lse) return MSA_ERR_INVALID_ARG;
  const int splits = choose_splits(bank, s);
  Workspace w = layout(bank, s, splits, nullptr);
  if ((rc = ensure_workspace(bank, w.bytes, (cudaStream_t)stream)) != MSA_OK) return rc;
  if ((rc = ensure_gtab(bank, (int64_t)top_k * bank->koff_len, s.Lc, (cudaStream_t)stream)) != MSA_OK) return rc;
  w = layout(bank, s, splits, bank->ws);
  return attend_impl(bank, q, s, splits, w, topk_idx, out, (cudaStream_t)stream, nullptr, lse);
}

msa_status msa_forward(msa_bank* bank, const msa_query* q, int32_t top_k, int32_t* topk_idx, float* out,
                       void* stream) {
  StepShape s;
  msa_status rc = check_query(bank, q, top_k, &s, true);
  if (rc != MSA_OK) return rc;
  if (!topk_idx || !out || top_k > bank->n_docs) return MSA_ERR_INVALID_ARG;
  const int splits = choose_splits(bank, s);
  Workspace w = layout(bank, s, splits, nullptr);
  if ((rc = ensure_workspace(bank, w.bytes, (cudaStream_t)stream)) != MSA_OK) return rc;
  if ((rc = ensure_gtab(bank, (int64_t)top_k * bank->koff_len, s.Lc, (cudaStream_t)stream)) != MSA_OK) return rc;
  w = layout(bank, s, splits, bank->ws);
  cudaStream_t st = (cudaStream_t)stream;
  if (bank->kv_loc == MSA_KV_PINNED_HOST) return forward_host(bank, q, s, topk_idx, out, st);
  // decode: the attention's local-context CTAs run beside the routing (programmatic
  // dependent launches); the steps and their results are those of msa_route + msa_attend
  const bool overlap = s.rows <= kMaxRows && !bank->f32;
  if ((rc = route_impl(bank, q, s, w, nullptr, topk_idx, nullptr, st, overlap)) != MSA_OK) return rc;
  return attend_impl(bank, q, s, splits, w, topk_idx, out, st, nullptr, nullptr, 1, overlap);
}

namespace {
// saved_out / saved_lse: the forward's output and log-sum-exp, or both NULL (recomputed)
msa_status backward_impl(msa_bank* bank, const msa_query* q, int32_t top_k, const int32_t* topk_idx,
                         const float* saved_out, const float* saved_lse, const float* d_out, float* dq,
                         float* dlocal_k, float* dlocal_v, float* dbank_k, float* dbank_v, void* stream) {
  StepShape s;
  msa_status rc = check_query(bank, q, top_k, &s, true);
  if (rc != MSA_OK) return rc;
  if (!topk_idx || !d_out || !dq || !dlocal_k || !dlocal_v || !dbank_k || !dbank_v) return MSA_ERR_INVALID_ARG;
  for (const void* p : {(const void*)d_out, (const void*)dq, (const void*)dlocal_k, (const void*)dlocal_v,
                        (const void*)dbank_k, (const void*)dbank_v})
    if (!aligned16(p)) return MSA_ERR_INVALID_ARG;
  if (bank->kv_loc != MSA_KV_DEVICE || bank->f32 || is_shard(bank)) return MSA_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  // workspace after the split counters: RoPE'd queries and local keys, row statistics
  const size_t qrot = align_up((size_t)s.B * s.Hq * s.Tq * bank->d * 2);
  const size_t lrot = align_up((size_t)s.B * bank->hkv * s.Lc * bank->d * 2);
  const size_t stats = align_up((size_t)s.P * s.rows * 4);
  // the key-tile (tcgen05) dK/dV path: dO in bf16 and the per-head index of who selected what
  const bool tc = attend_bwd_tc_supported(bank->d, s.Bq, s.k);
  // the whole step on the tensor cores: the tcgen05 forward gives O and each row's
  // log-sum-exp, then the tcgen05 dQ and dK/dV kernels
  const bool tc_all = tc && attend_prefill_tc_supported(bank->d, s.G, s.Bq) && s.k <= 64;
  const bool saved = saved_out && saved_lse;
  const size_t otmp = tc_all && !saved ? align_up((size_t)s.B * s.Hq * s.Tq * bank->d * 4) : 0;
  const size_t ltmp = tc_all && !saved ? align_up((size_t)s.B * s.Hq * s.Tq * 4) : 0;
  const int64_t ph = (int64_t)s.B * (s.Tq / s.Bq);           // problems per KV head
  const int64_t cap = ph * s.k;                              // selections per KV head
  const int64_t rb = std::min<int64_t>(bank->n_docs, cap);    // documents one head can have selected
  const int kt = attend_bwd_tc_tile_rows();
  const int64_t item_cap = rb * ((bank->max_len + kt - 1) / kt);  // their key tiles, at most
  const size_t dob = tc ? align_up((size_t)s.B * s.Hq * s.Tq * bank->d * 2) : 0;
  const size_t i_cnt = tc ? align_up((size_t)bank->hkv * bank->n_docs * 4) : 0;
  const size_t i_nit = tc ? align_up((size_t)bank->hkv * 4) : 0;
  const size_t i_items = tc ? align_up((size_t)bank->hkv * item_cap * 16) : 0;
  const size_t i_prob = tc ? align_up((size_t)bank->hkv * cap * 4) : 0;
  if (tc && (cap >= (int64_t(1) << 31) || item_cap >= (int64_t(1) << 31) || bank->hkv > 64))
    return MSA_ERR_UNSUPPORTED;
  const size_t base_ws = kCounterBytes + qrot + lrot + 2 * stats;
  if ((rc = ensure_workspace(bank, base_ws + dob + i_cnt + i_nit + i_items + i_prob + otmp + ltmp, st)) != MSA_OK)
    return rc;
  if ((rc = ensure_gtab(bank, (int64_t)top_k * bank->koff_len, s.Lc, st)) != MSA_OK) return rc;
  uint8_t* ws = bank->ws + kCounterBytes;
  uint16_t* q_rot = reinterpret_cast<uint16_t*>(ws);
  uint16_t* l_rot = reinterpret_cast<uint16_t*>(ws + qrot);
  float* lse2 = reinterpret_cast<float*>(ws + qrot + lrot);
  float* drow = reinterpret_cast<float*>(ws + qrot + lrot + stats);
  uint8_t* wtc = bank->ws + base_ws;
  uint16_t* do_bf = reinterpret_cast<uint16_t*>(wtc);
  int* idx_cnt = reinterpret_cast<int*>(wtc + dob);
  int* idx_nitems = reinterpret_cast<int*>(wtc + dob + i_cnt);
  int4* idx_items = reinterpret_cast<int4*>(wtc + dob + i_cnt + i_nit);
  int* idx_prob = reinterpret_cast<int*>(wtc + dob + i_cnt + i_nit + i_items);
  float* o_tmp = reinterpret_cast<float*>(wtc + dob + i_cnt + i_nit + i_items + i_prob);
  float* lse_tmp = reinterpret_cast<float*>(wtc + dob + i_cnt + i_nit + i_items + i_prob + otmp);
  const int64_t qrows = (int64_t)s.B * s.Hq * s.Tq, lrows = (int64_t)s.B * bank->hkv * s.Lc;
  MSA_CUDA(launch_rope_rows((const uint16_t*)q->q, q_rot, bank->d_gtab, qrows, s.Tq, s.Lc - s.Tq, bank->d, st));
  MSA_CUDA(launch_rope_rows((const uint16_t*)q->local_k, l_rot, bank->d_gtab, lrows, s.Lc, 0, bank->d, st));
  MSA_CUDA(cudaMemsetAsync(dlocal_k, 0, (size_t)lrows * bank->d * 4, st));
  MSA_CUDA(cudaMemsetAsync(dlocal_v, 0, (size_t)lrows * bank->d * 4, st));
  const int box = attend_bwd_tile_rows();
  AttendMaps maps;
  if ((rc = make_map(&maps.bank_k, bank->k, (int64_t)bank->hkv * bank->kv_rows, bank->d, box)) != MSA_OK) return rc;
  if ((rc = make_map(&maps.bank_v, bank->v, (int64_t)bank->hkv * bank->kv_rows, bank->d, box)) != MSA_OK) return rc;
  if ((rc = make_map(&maps.loc_k, l_rot, lrows, bank->d, box)) != MSA_OK) return rc;
  if ((rc = make_map(&maps.loc_v, q->local_v, lrows, bank->d, box)) != MSA_OK) return rc;
  AttendBwdArgs g{};
  AttendArgs& a = g.a;
  a.q = (const uint16_t*)q->q;
  a.sel = topk_idx;
  a.doc_row = bank->d_doc_row;
  a.doc_len = bank->d_doc_len;
  a.gtab = bank->d_gtab;
  a.err = bank->d_err;
  a.kv_rows = bank->kv_rows;
  a.batch = s.B;
  a.n_q_heads = s.Hq;
  a.n_kv_heads = bank->hkv;
  a.q_tokens = s.Tq;
  a.local_len = s.Lc;
  a.route_block = s.Bq;
  a.top_k = s.k;
  a.n_docs = bank->n_docs;
  a.n_docs_index = bank->n_docs;  // a whole bank (shards are refused above)
  a.with_local = 1;
  a.n_splits = 1;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)bank->d));
  g.dout = d_out;
  g.dq = dq;
  g.lse2 = lse2;
  g.drow = drow;
  g.q_rot = q_rot;
  g.ptab = bank->d_ptab;
  g.dk_bank = dbank_k;
  g.dv_bank = dbank_v;
  g.dk_loc = dlocal_k;
  g.dv_loc = dlocal_v;
  if (!tc_all) MSA_CUDA(launch_attend_bwd_dq(g, maps, bank->d, st));
  if (tc) {
    if (!tc_all) MSA_CUDA(launch_to_bf16(d_out, do_bf, qrows * bank->d, bank->sms, st));
    MSA_CUDA(launch_attend_bwd_index(topk_idx, bank->d_doc_len, bank->d_doc_row, bank->kv_rows, idx_cnt, idx_nitems,
                                     idx_items, idx_prob, bank->n_docs, bank->hkv, (int)ph, s.k, (int)item_cap,
                                     (int)cap, bank->d_err, st));
    const int rc_rows = attend_bwd_tc_chunk_rows();
    AttendMaps m2;
    m2.bank_k = bank->map_k128;
    m2.bank_v = bank->map_v128;
    if (kt != attend_prefill_tc_tile_rows()) return MSA_ERR_UNSUPPORTED;
    if ((rc = make_map(&m2.loc_k, l_rot, lrows, bank->d, kt)) != MSA_OK) return rc;
    if ((rc = make_map(&m2.loc_v, q->local_v, lrows, bank->d, kt)) != MSA_OK) return rc;
    CUtensorMap q_map{}, do_map{};
    if ((rc = make_map(&q_map, q_rot, qrows, bank->d, rc_rows)) != MSA_OK) return rc;
    if ((rc = make_map(&do_map, do_bf, qrows, bank->d, rc_rows)) != MSA_OK) return rc;
    if (tc_all) {
      // the forward's O and log-sum-exp (saved by the caller, else recomputed into the
      // workspace), dO . O, then dQ
      const float* o_use = saved_out;
      const float* lse_use = saved_lse;
      if (!saved) {
        AttendArgs fa = a;
        fa.out = o_tmp;
        fa.lse_out = lse_tmp;
        MSA_CUDA(launch_attend_prefill_tc(fa, m2, q_map, st));
        o_use = o_tmp;
        lse_use = lse_tmp;
      }
      MSA_CUDA(launch_attend_bwd_prep(d_out, o_use, lse_use, do_bf, drow, lse2, s.B, s.Hq, bank->hkv, s.Tq, s.Bq,
                                      bank->sms, st));
      MSA_CUDA(launch_attend_bwd_dq_tc(g, m2, q_map, do_map, st));
    }
    AttendGradMaps gm;
    if ((rc = make_map_f32(&gm.dk_bank, dbank_k, (int64_t)bank->hkv * bank->kv_rows, bank->d, kt)) != MSA_OK) return rc;
    if ((rc = make_map_f32(&gm.dv_bank, dbank_v, (int64_t)bank->hkv * bank->kv_rows, bank->d, kt)) != MSA_OK) return rc;
    if ((rc = make_map_f32(&gm.dk_loc, dlocal_k, lrows, bank->d, kt)) != MSA_OK) return rc;
    if ((rc = make_map_f32(&gm.dv_loc, dlocal_v, lrows, bank->d, kt)) != MSA_OK) return rc;
    g.idx_nitems = idx_nitems;
    g.idx_items = idx_items;
    g.idx_prob = idx_prob;
    g.idx_item_cap = (int)item_cap;
    g.idx_cap = (int)cap;
    MSA_CUDA(launch_attend_bwd_dkdv_tc(g, m2, q_map, do_map, gm, bank->sms, st));
    return MSA_OK;
  }
  const int max_tiles = s.k * (int)((bank->max_len + box - 1) / box) + (s.Lc + box - 1) / box;
  MSA_CUDA(launch_attend_bwd_dkdv(g, maps, bank->d, max_tiles, st));
  return MSA_OK;
}

}  // namespace

msa_status msa_attend_backward(msa_bank* bank, const msa_query* q, int32_t top_k, const int32_t* topk_idx,
                               const float* d_out, float* dq, float* dlocal_k, float* dlocal_v,
                               float* dbank_k, float* dbank_v, void* stream) {
  return backward_impl(bank, q, top_k, topk_idx, nullptr, nullptr, d_out, dq, dlocal_k, dlocal_v, dbank_k, dbank_v,
                       stream);
}

msa_status msa_attend_backward_saved(msa_bank* bank, const msa_query* q, int32_t top_k, const int32_t* topk_idx,
                                     const float* out, const float* lse, const float* d_out, float* dq,
                                     float* dlocal_k, float* dlocal_v, float* dbank_k, float* dbank_v,
                                     void* stream) {
  if (!out || !lse || !aligned16(out)) return MSA_ERR_INVALID_ARG;
  return backward_impl(bank, q, top_k, topk_idx, out, lse, d_out, dq, dlocal_k, dlocal_v, dbank_k, dbank_v, stream);
}

msa_status msa_set_kv_cache(msa_bank* bank, int64_t bytes) {
  if (!bank || bank->kv_loc != MSA_KV_PINNED_HOST || bytes < 0) return MSA_ERR_INVALID_ARG;
  if (!on_bank_device(bank)) return MSA_ERR_INVALID_ARG;
  MSA_CUDA(cudaDeviceSynchronize());
  if (bank->stage_k) cudaFree(bank->stage_k);
  if (bank->stage_v) cudaFree(bank->stage_v);
  bank->stage_k = bank->stage_v = nullptr;
  bank->stage_cap = 0;
  bank->cache_on = false;
  bank->cache_slots = 0;
  bank->cache_map.clear();
  bank->slot_key.clear();
  bank->slot_use.clear();
  bank->lru.clear();
  bank->slot_it.clear();
  if (bytes == 0) return MSA_OK;
  const int64_t slot_bytes = 2 * bank->max_len * bank->d * 2;
  const int64_t slots = bytes / slot_bytes;
  if (slots < 1) return MSA_ERR_INVALID_ARG;
  const int64_t rows = slots * bank->max_len;
  if (rows >= (int64_t(1) << 31)) return MSA_ERR_UNSUPPORTED;
  const size_t b = (size_t)rows * bank->d * 2;
  if (cudaMalloc(&bank->stage_k, b) != cudaSuccess || cudaMalloc(&bank->stage_v, b) != cudaSuccess) {
    if (bank->stage_k) cudaFree(bank->stage_k);
    bank->stage_k = nullptr;
    return MSA_ERR_OOM;
  }
  bank->stage_cap = rows;
  bank->cache_slots = slots;
  bank->slot_key.assign(slots, -1);
  bank->slot_use.assign(slots, -1);
  bank->slot_it.resize(slots);
  for (int64_t i = 0; i < slots; ++i) bank->slot_it[i] = bank->lru.insert(bank->lru.end(), i);
  bank->cache_map.reserve((size_t)slots * 2);
  bank->cache_on = true;
  return MSA_OK;
}

msa_status msa_kv_cache_stats(const msa_bank* bank, int64_t* slabs, int64_t* hits, int64_t* bytes_copied) {
  if (!bank) return MSA_ERR_INVALID_ARG;
  if (slabs) *slabs = bank->st_slabs;
  if (hits) *hits = bank->st_hits;
  if (bytes_copied) *bytes_copied = bank->last_fetch_bytes;
  return MSA_OK;
}

msa_status msa_set_host_fetch(msa_bank* bank, msa_host_fetch mode) {
  if (!bank || bank->kv_loc != MSA_KV_PINNED_HOST) return MSA_ERR_INVALID_ARG;
  if (mode != MSA_FETCH_COPY_ENGINE && mode != MSA_FETCH_SM_GATHER) return MSA_ERR_INVALID_ARG;
  if (mode == MSA_FETCH_SM_GATHER && !bank->k_map) return MSA_ERR_UNSUPPORTED;
  if (!on_bank_device(bank)) return MSA_ERR_INVALID_ARG;
  MSA_CUDA(cudaDeviceSynchronize());
  bank->gather = mode == MSA_FETCH_SM_GATHER;
  return MSA_OK;
}

msa_status msa_get_host_fetch(const msa_bank* bank, msa_host_fetch* mode) {
  if (!bank || !mode || bank->kv_loc != MSA_KV_PINNED_HOST) return MSA_ERR_INVALID_ARG;
  *mode = bank->gather ? MSA_FETCH_SM_GATHER : MSA_FETCH_COPY_ENGINE;
  return MSA_OK;
}

msa_status msa_set_router_precision(msa_bank* bank, msa_kr_precision precision) {
  if (!bank || (precision != MSA_KR_F32 && precision != MSA_KR_BF16)) return MSA_ERR_INVALID_ARG;
  bank->kr_bf16 = precision == MSA_KR_BF16;
  return MSA_OK;
}

msa_status msa_check_wait_timeout(msa_bank* bank, void* stream) {
  if (!bank || !on_bank_device(bank)) return MSA_ERR_INVALID_ARG;
  MSA_CUDA(launch_wait_timeout(bank->d_err, (cudaStream_t)stream));
  return MSA_OK;
}

msa_status msa_bank_set_shard(msa_bank* bank, int32_t doc_base, int32_t n_docs_total, int64_t max_doc_len_total) {
  if (!bank || !on_bank_device(bank)) return MSA_ERR_INVALID_ARG;
  if (doc_base < 0 || n_docs_total < 1 || (int64_t)doc_base + bank->n_docs > n_docs_total ||
      max_doc_len_total < bank->max_len || max_doc_len_total >= (int64_t(1) << 30))
    return MSA_ERR_INVALID_ARG;
  bank->doc_lo = doc_base;
  bank->n_docs_total = n_docs_total;
  bank->koff_len = max_doc_len_total;
  bank->gtab_koff = -1;  // the Global-RoPE offset follows the whole bank's longest document
  return MSA_OK;
}

msa_status msa_attend_partial(msa_bank* bank, const msa_query* q, int32_t top_k, const int32_t* topk_idx,
                              int32_t with_local, float* out, float* lse, void* stream) {
  StepShape s;
  msa_status rc = check_query(bank, q, top_k, &s, true);
  if (rc != MSA_OK) return rc;
  if (!topk_idx || !out || !lse || (with_local != 0 && with_local != 1)) return MSA_ERR_INVALID_ARG;
  const int splits = choose_splits(bank, s);
  Workspace w = layout(bank, s, splits, nullptr);
  if ((rc = ensure_workspace(bank, w.bytes, (cudaStream_t)stream)) != MSA_OK) return rc;
  if ((rc = ensure_gtab(bank, (int64_t)top_k * bank->koff_len, s.Lc, (cudaStream_t)stream)) != MSA_OK) return rc;
  w = layout(bank, s, splits, bank->ws);
  return attend_impl(bank, q, s, splits, w, topk_idx, out, (cudaStream_t)stream, nullptr, lse, with_local);
}

msa_status msa_merge_topk(int32_t n_parts, int32_t rows, int32_t top_k, const float* cand_scores,
                          const int32_t* cand_idx, int32_t* topk_idx, float* topk_scores, void* stream) {
  if (!cand_scores || !cand_idx || !topk_idx || n_parts < 1 || rows < 1 || top_k < 1) return MSA_ERR_INVALID_ARG;
  if (n_parts > 64 || top_k > kMaxTopK || rows > 65535) return MSA_ERR_UNSUPPORTED;
  return from_cuda(launch_merge_topk(n_parts, rows, top_k, cand_scores, cand_idx, topk_idx, topk_scores,
                                     (cudaStream_t)stream));
}

msa_status msa_merge_partials(int32_t n_parts, int64_t rows, int32_t head_dim, const float* part_out,
                              const float* part_lse, float* out, float* lse, void* stream) {
  if (!part_out || !part_lse || !out || n_parts < 1 || rows < 1 || head_dim < 1) return MSA_ERR_INVALID_ARG;
  if ((rows + 7) / 8 > 0x7fffffff) return MSA_ERR_UNSUPPORTED;
  return from_cuda(launch_merge_partials(n_parts, rows, head_dim, part_out, part_lse, out, lse,
                                         (cudaStream_t)stream));
}

msa_status msa_interleave_route(msa_bank* bank, const msa_query* q, int32_t top_k, const float* q_r_in,
                                const int32_t* context_idx, int32_t n_ctx, int32_t* ctx_out, float* topk_scores,
                                float* q_r_out, void* stream) {
  StepShape s;
  msa_status rc = check_query(bank, q, top_k, &s, false);
  if (rc != MSA_OK) return rc;
  if (is_shard(bank)) return MSA_ERR_UNSUPPORTED;
  if (!ctx_out || n_ctx < 0 || (n_ctx > 0 && !context_idx) || (int64_t)n_ctx + top_k > bank->n_docs)
    return MSA_ERR_INVALID_ARG;
  if (q_r_in && !aligned16(q_r_in)) return MSA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  Workspace w = layout(bank, s, 1, nullptr);
  if ((rc = ensure_workspace(bank, w.bytes, st)) != MSA_OK) return rc;
  w = layout(bank, s, 1, bank->ws);
  // the hop's routing query: the given one ([B, Hkv, nblk, d_r]: one "token" per block),
  // or the block means of the routing queries on the first hop
  QrArgs qa = q_r_in ? QrArgs{nullptr, w.q_r, w.q_r_inv, s.B, bank->hkv, s.nblk, 1, bank->dr, q_r_in}
                     : QrArgs{bank->f32 ? nullptr : (const uint16_t*)q->qr, w.q_r, w.q_r_inv, s.B, bank->hkv,
                              s.Tq, s.Bq, bank->dr, bank->f32 ? (const float*)q->qr : nullptr};
  MSA_CUDA(launch_qr_prep(qa, st));
  if ((rc = run_router(bank, q, s, w.q_r, w.q_r_inv, w.scores, false, st)) != MSA_OK) return rc;
  const int ld = n_ctx + top_k;
  MSA_CUDA(launch_interleave_context(context_idx, n_ctx, s.P, bank->n_docs, bank->doc_lo, bank->n_docs_total, w.scores,
                                     ctx_out, ld, bank->d_err, st));
  TopkArgs ta{w.scores, ctx_out, topk_scores, s.P, bank->n_docs, top_k, bank->doc_lo, ld, n_ctx};
  MSA_CUDA(launch_topk(ta, st));
  if (q_r_out) {
    InterleaveUpdateArgs u{w.q_r, w.q_r_inv, ctx_out, ld, n_ctx, top_k, bank->d_kr, bank->d_chunk_off,
                           bank->d_chunk_len, bank->nch, s.B * s.nblk, bank->hkv, s.nblk, bank->n_docs,
                           bank->doc_lo, q_r_out};
    MSA_CUDA(launch_interleave_update(u, bank->dr, st));
  }
  return MSA_OK;
}

msa_status msa_get_device_error(msa_bank* bank, void* stream) {
  if (!bank || !on_bank_device(bank)) return MSA_ERR_INVALID_ARG;
  MSA_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
  int v = 0;
  MSA_CUDA(cudaMemcpy(&v, bank->d_err, sizeof(int), cudaMemcpyDeviceToHost));
  MSA_CUDA(cudaMemset(bank->d_err, 0, sizeof(int)));
  // A step cut short may leave split counters mid-count: reset them.
  if (v != 0 && bank->ws) MSA_CUDA(cudaMemset(bank->ws, 0, kCounterBytes));
  return (msa_status)v;
}

}  // extern "C"
