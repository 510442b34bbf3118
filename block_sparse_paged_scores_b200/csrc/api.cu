// api.cu — the C ABI of libmsa.so (declared in include/msa.h): argument validation, route
// selection, split-K sizing, workspace layout, tensor-map encoding and kernel launches.
//
// Mojo module "msa": both ops take the same arguments for every step and pick the kernel at
// run time from the largest number of new query tokens in the batch (1: decode, 2..8:
// speculative decode, more: prefill); decode splits the selected blocks over SM-filling
// split-K partitions.  The library owns no device memory: every buffer, the workspace
// included, comes from the caller, and every call only enqueues work on the caller's stream.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "internal.h"

namespace msa {

namespace {

// ---- tensor maps: the runtime hands out the driver's encoder, no link against libcuda
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A paged cache [tiles = num_pages * heads][128 tokens][128 dims] as a 3-D tensor map whose
// box is one (page, head) tile: 128 tokens x 64 bf16 (two loads per tile) or 128 x 128 e4m3,
// written to shared memory with the 128-byte swizzle.
// `rows` < 128 views a tile of 1-byte elements as `rows` rows of 128 bytes (the fp4 index-K
// tile: 64 rows, two tokens' code pairs each).
bool page_tensor_map(CUtensorMap *map, const void *base, long long tiles, bool fp8,
                     int rows = kBlock) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t esz = fp8 ? 1 : 2;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(tiles)};
  const cuuint64_t strides[2] = {kHeadDim * esz, kHeadDim * rows * esz};
  const cuuint32_t box[3] = {fp8 ? 128u : 64u, static_cast<cuuint32_t>(rows), 1u};
  const cuuint32_t estr[3] = {1, 1, 1};
  memset(map, 0, sizeof(*map));
  const CUresult r = fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        3, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return 0;
  return d;
}

int num_sms_of_current_device() {
  static int cache[64] = {0};
  const int d = current_device();
  if (d < 0 || d >= 64) return 148;
  if (!cache[d]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0)
      n = 148;
    cache[d] = n;
  }
  return cache[d];
}

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool ragged_ok(const msa_ragged_paged_t *rp) {
  return rp && rp->input_row_offsets && rp->cache_lengths && rp->kv_lookup_table &&
         rp->batch >= 1 && rp->total_q >= 0 && rp->max_q_len >= 1 &&
         rp->max_pages_per_seq >= 1 && rp->num_pages >= 1;
}

// ---- attention route: tiles, row groups, partitions and the workspace layout
struct Route {
  bool plan;      // speculative / prefill: per-tile union in the workspace
  bool stream;    // decode / speculative: the persistent split-K kernel + combine
  bool tc;        // prefill on tcgen05 (BF16 KV): 128-row tiles
  int qt, tiles;  // query tokens per tile, tiles per sequence
  int rg;         // 16-row groups per CTA
  int cap;        // work-list slots per item
  int items;
  int grid;       // persistent kernel: CTAs (= split-K partitions)
  long long R;    // slots per CTA
  int P;          // most CTAs one item spans
  int splits;     // partial split indices (= P)
  size_t off_o, off_lse, off_list, off_masks, off_counts, bytes;
};

constexpr int kMaxRows = 64;  // rows (tokens x group heads) per attention CTA
constexpr int kMaxSplits = 4096;
constexpr int kMinSlotsPerCta = 8;

int stream_grid(long long total, int num_splits, int num_sms) {
  long long grid = num_splits > 0 ? num_splits
                                  : std::min<long long>(num_sms,
                                                        (total + kMinSlotsPerCta - 1) /
                                                            kMinSlotsPerCta);
  if (grid > total) grid = total;
  if (grid < 1) grid = 1;
  return static_cast<int>(grid);
}

bool make_route(const msa_ragged_paged_t *rp, int S, int H_q, int H_kv, int max_blocks,
                int num_splits, int num_sms, bool fp8, Route *r) {
  const int G = H_q / H_kv;
  r->plan = rp->max_q_len > 1;
  r->stream = rp->max_q_len <= MSA_MAX_SPEC_DRAFT;
  r->tc = !r->stream && G <= 128 && attention_tc_supported(G, std::max(1, 128 / G));
  if (!r->plan) {
    r->qt = 1;
  } else {
    int qt = (r->tc ? 128 : kMaxRows) / G;
    if (qt > 32) qt = 32;  // token masks are 32-bit
    if (qt > rp->max_q_len) qt = rp->max_q_len;
    r->qt = qt < 1 ? 1 : qt;
  }
  r->tiles = (rp->max_q_len + r->qt - 1) / r->qt;
  r->rg = (r->qt * G + 15) / 16;
  if (r->rg < 1 || (r->rg > 4 && !r->tc)) return false;
  const long long cap = r->plan ? std::min<long long>(static_cast<long long>(r->qt) * S, max_blocks)
                                : S;
  r->cap = static_cast<int>(cap);
  const long long items = static_cast<long long>(rp->batch) * r->tiles * H_kv;
  if (items > 0x7fffffffLL) return false;
  r->items = static_cast<int>(items);
  r->grid = 1;
  r->R = 0;
  r->P = 0;
  r->splits = 0;
  if (r->stream) {
    const long long total = items * cap;
    r->grid = stream_grid(total, num_splits, num_sms);
    r->R = (total + r->grid - 1) / r->grid;
    r->grid = static_cast<int>((total + r->R - 1) / r->R);
    int P = 1;
    for (long long it = 0; it < items; ++it) {
      const long long first = it * cap / r->R, last = (it * cap + cap - 1) / r->R;
      P = std::max<int>(P, static_cast<int>(last - first + 1));
    }
    r->P = P;
    r->splits = P;
  }
  const size_t rows = static_cast<size_t>(rp->total_q) * H_q;
  size_t off = 0;
  r->off_o = off;
  if (r->stream) off = round_up(off + rows * kHeadDim * sizeof(float) * r->splits, 256);
  r->off_lse = off;
  if (r->stream) off = round_up(off + rows * sizeof(float) * r->splits, 256);
  r->off_list = off;
  if (r->plan) off = round_up(off + static_cast<size_t>(items) * r->cap * sizeof(int32_t), 256);
  r->off_masks = off;
  if (r->plan) off = round_up(off + static_cast<size_t>(items) * r->cap * sizeof(uint32_t), 256);
  r->off_counts = off;
  if (r->plan) off = round_up(off + static_cast<size_t>(items) * sizeof(int32_t), 256);
  r->bytes = off;
  return true;
}

}  // namespace

// One cudaFuncSetAttribute per (kernel, device) for the dynamic shared-memory opt-in.
cudaError_t ensure_smem_limit(const void *func, int bytes) {
  struct Entry {
    const void *func;
    int device;
    int bytes;
  };
  static Entry table[256];
  static int n = 0;
  static std::mutex mu;
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n; ++i)
    if (table[i].func == func && table[i].device == dev && table[i].bytes >= bytes)
      return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (n < 256) table[n++] = Entry{func, dev, bytes};
  return cudaSuccess;
}

}  // namespace msa

using namespace msa;

extern "C" {

const char *msa_status_string(msa_status_t status) {
  switch (status) {
    case MSA_OK: return "MSA_OK";
    case MSA_ERR_INVALID_ARG: return "MSA_ERR_INVALID_ARG";
    case MSA_ERR_UNSUPPORTED: return "MSA_ERR_UNSUPPORTED";
    case MSA_ERR_CUDA: return "MSA_ERR_CUDA";
  }
  return "MSA_ERR_UNKNOWN";
}

int32_t msa_default_num_splits(int32_t batch, int32_t max_q_len, int32_t num_kv_heads, int32_t S,
                               int32_t num_sms) {
  if (batch < 1 || max_q_len < 1 || num_kv_heads < 1 || S < 1 || num_sms < 1 ||
      max_q_len > MSA_MAX_SPEC_DRAFT)
    return 1;
  const long long total = static_cast<long long>(batch) * num_kv_heads * S * max_q_len;
  return stream_grid(total, 0, num_sms);
}

size_t msa_attn_workspace_bytes(const msa_ragged_paged_t *rp, int32_t S, int32_t num_q_heads,
                                int32_t num_kv_heads, int32_t max_blocks, int32_t num_splits) {
  if (!rp || rp->batch < 1 || rp->max_q_len < 1 || S < 1 || num_kv_heads < 1 ||
      num_q_heads < num_kv_heads || num_q_heads % num_kv_heads || max_blocks < 1 ||
      num_splits < 0)
    return 0;
  // the size covers either KV dtype (the prefill routes tile differently)
  Route r, r8;
  const int sms = num_splits > 0 ? 1 : num_sms_of_current_device();
  if (!make_route(rp, S, num_q_heads, num_kv_heads, max_blocks, num_splits, sms, false, &r) ||
      !make_route(rp, S, num_q_heads, num_kv_heads, max_blocks, num_splits, sms, true, &r8))
    return 0;
  return std::max(r.bytes, r8.bytes);
}

int32_t msa_attn_partials(const msa_ragged_paged_t *rp, int32_t S, int32_t num_q_heads,
                          int32_t num_kv_heads, int32_t max_blocks, int32_t num_splits,
                          size_t *partial_o_offset, size_t *partial_lse_offset) {
  if (!rp || rp->batch < 1 || rp->max_q_len < 1 || S < 1 || num_kv_heads < 1 ||
      num_q_heads < num_kv_heads || num_q_heads % num_kv_heads || max_blocks < 1 ||
      num_splits < 0)
    return 0;
  Route r;
  const int sms = num_splits > 0 ? 1 : num_sms_of_current_device();
  if (!make_route(rp, S, num_q_heads, num_kv_heads, max_blocks, num_splits, sms, false, &r) ||
      !r.stream)
    return 0;
  if (partial_o_offset) *partial_o_offset = r.off_o;
  if (partial_lse_offset) *partial_lse_offset = r.off_lse;
  return r.splits;
}

namespace {

// The selection to fuse into the decode indexer (nullptr: scores only).  With publish set
// instead (the one-call decode step), the indexer selects nothing: the last CTA of every unit
// publishes publish[unit] = *epoch + 1.
struct FusedSelect {
  int32_t *counters, *block_ids, *num_selected;
  int top_k, init_blocks, local_blocks, S;
  int32_t *publish = nullptr;
  const int32_t *epoch = nullptr;
};

// The prefill route scores BF16 index-K on tcgen05 (query rows as M); the speculative route
// too when its units hold more than 16 rows, with a page's positions as M and the rows as 32
// columns (the per-token top-k; the top-k shared across drafts scores one token and stays on
// the warp-MMA kernel, which selects in the same launch); the scaled formats take the warp-MMA
// kernel on every route.
bool index_uses_tc(const msa_ragged_paged_t *rp, int Hg, int idx_fmt) {
  return idx_fmt == kIdxBf16 && rp->max_q_len > MSA_MAX_SPEC_DRAFT && Hg <= 128;
}
bool index_uses_tc_pos(const msa_ragged_paged_t *rp, int Hg, int idx_fmt, uint32_t flags) {
  if (idx_fmt != kIdxBf16 || rp->max_q_len < 2 || rp->max_q_len > MSA_MAX_SPEC_DRAFT ||
      (flags & MSA_SHARE_ACROSS_DRAFTS) || Hg < 1 || Hg > 32)
    return false;
  const int qt = rp->max_q_len * Hg <= 32 ? rp->max_q_len : 32 / Hg;  // as index_scores_impl
  return qt * Hg > 16;
}

bool index_k_ok(const msa_index_k_t *k, int32_t num_kv_heads) {
  if (!k || !k->codes || !aligned(k->codes, 16) ||
      !(k->num_heads == 1 || k->num_heads == num_kv_heads))
    return false;
  if (k->dtype == MSA_IDX_BF16) return true;
  if (k->dtype == MSA_IDX_FP8_E4M3 || k->dtype == MSA_IDX_FP4_E2M1)
    return k->scales && aligned(k->scales, 16);
  return false;
}

// The flags msa_index_scores_k / msa_index_select_k accept for this batch.
bool index_flags_ok(const msa_ragged_paged_t *rp, uint32_t flags) {
  if (flags & ~static_cast<uint32_t>(MSA_SHARE_ACROSS_DRAFTS)) return false;
  return !(flags & MSA_SHARE_ACROSS_DRAFTS) || rp->max_q_len <= MSA_MAX_SPEC_DRAFT;
}

msa_status_t index_scores_impl(const msa_ragged_paged_t *rp, const void *q_idx,
                               const msa_index_k_t *kidx, int32_t num_kv_heads,
                               int32_t max_blocks, uint32_t flags, float *scores,
                               int32_t *dev_err, cudaStream_t stream, const FusedSelect *fs) {
  if (!ragged_ok(rp) || !q_idx || !scores || num_kv_heads < 1 || !index_k_ok(kidx, num_kv_heads) ||
      max_blocks < 1 || max_blocks > rp->max_pages_per_seq || !aligned(q_idx, 16) ||
      !index_flags_ok(rp, flags))
    return MSA_ERR_INVALID_ARG;
  const bool share = (flags & MSA_SHARE_ACROSS_DRAFTS) != 0;
  const void *k_idx_cache = kidx->codes;
  const int32_t num_idx_k_heads = kidx->num_heads;
  const int idx_fmt = static_cast<int>(kidx->dtype);
  const int Hg = num_kv_heads / num_idx_k_heads;
  if (Hg > 32) return MSA_ERR_UNSUPPORTED;
  if (static_cast<long long>(rp->num_pages) * num_idx_k_heads >= (1LL << 31))
    return MSA_ERR_UNSUPPORTED;

  IndexerArgs a{};
  a.row_off = rp->input_row_offsets;
  a.cache_len = rp->cache_lengths;
  a.table = rp->kv_lookup_table;
  a.q_idx = static_cast<const uint16_t *>(q_idx);
  a.scores = scores;
  a.dev_err = dev_err;
  a.batch = rp->batch;
  a.max_q_len = rp->max_q_len;
  a.max_pages = rp->max_pages_per_seq;
  a.num_pages = rp->num_pages;
  a.H_kv = num_kv_heads;
  a.H_idxk = num_idx_k_heads;
  a.max_blocks = max_blocks;
  a.counters = nullptr;
  a.idx_fmt = idx_fmt;
  a.k_idx_scale = kidx->scales;
  // prefill: the dense tile x page contraction runs on tcgen05 (128-row tiles)
  if (index_uses_tc(rp, Hg, idx_fmt)) {
    if (fs) return MSA_ERR_UNSUPPORTED;  // the caller selects with a separate launch
    a.qt = std::min(rp->max_q_len, std::max(1, 128 / Hg));
    a.tiles = (rp->max_q_len + a.qt - 1) / a.qt;
    a.chunk = max_blocks;
    if (static_cast<long long>(rp->batch) * a.tiles > 0x7fffffffLL) return MSA_ERR_UNSUPPORTED;
    CUtensorMap kmap;
    if (!page_tensor_map(&kmap, k_idx_cache,
                         static_cast<long long>(rp->num_pages) * num_idx_k_heads, false))
      return MSA_ERR_CUDA;
    return launch_index_scores_tc(kmap, a, stream) == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
  }
  a.qt = rp->max_q_len * Hg <= 32 ? rp->max_q_len : (32 / Hg > 0 ? 32 / Hg : 1);
  a.tiles = (rp->max_q_len + a.qt - 1) / a.qt;
  if (share) {  // only each sequence's first new token is scored
    a.qt = 1;
    a.tiles = 1;
    a.share = 1;
  }
  const int mt = a.qt * Hg <= 16 ? 1 : 2;
  // pages per CTA: about eight CTAs per SM over the launch, at least 4 pages each
  const long long units = static_cast<long long>(rp->batch) * a.tiles * num_idx_k_heads;
  if (units > 0x7fffffffLL) return MSA_ERR_UNSUPPORTED;
  const long long want = (8LL * num_sms_of_current_device() + units - 1) / units;
  long long chunk = (max_blocks + want - 1) / want;
  if (chunk < 4) chunk = 4;
  long long chunks = (max_blocks + chunk - 1) / chunk;
  a.chunk = static_cast<int>(chunk);
  a.chunks = static_cast<int>(chunks);
  if (units * chunks > 0x7fffffffLL) return MSA_ERR_UNSUPPORTED;
  const bool tc_pos = index_uses_tc_pos(rp, Hg, idx_fmt, flags);
  if (tc_pos && fs) return MSA_ERR_UNSUPPORTED;  // the caller selects with a separate launch
  if (fs) {
    a.publish = fs->publish;
    a.epoch = fs->epoch;
    a.counters = fs->counters;
    a.block_ids = fs->block_ids;
    a.num_selected = fs->num_selected;
    a.top_k = fs->top_k;
    a.init_blocks = fs->init_blocks;
    a.local_blocks = fs->local_blocks;
    a.S = fs->S;
  }

  CUtensorMap kmap;
  const long long ktiles = static_cast<long long>(rp->num_pages) * num_idx_k_heads;
  const bool ok_map = idx_fmt == kIdxBf16 ? page_tensor_map(&kmap, k_idx_cache, ktiles, false)
                      : idx_fmt == kIdxFp8
                          ? page_tensor_map(&kmap, k_idx_cache, ktiles, true)
                          : page_tensor_map(&kmap, k_idx_cache, ktiles, true, kBlock / 2);
  if (!ok_map) return MSA_ERR_CUDA;
  if (tc_pos)
    return launch_index_scores_tc_pos(kmap, a, static_cast<int>(chunks), stream) == cudaSuccess
               ? MSA_OK
               : MSA_ERR_CUDA;
  return launch_index_scores(kmap, a, mt, static_cast<int>(chunks), stream) == cudaSuccess
             ? MSA_OK
             : MSA_ERR_CUDA;
}

msa_index_k_t bf16_index_k(const void *k_idx_cache, int32_t num_idx_k_heads) {
  msa_index_k_t k;
  k.dtype = MSA_IDX_BF16;
  k.codes = k_idx_cache;
  k.scales = nullptr;
  k.num_heads = num_idx_k_heads;
  return k;
}

}  // namespace

msa_status_t msa_index_scores_k(const msa_ragged_paged_t *rp, const void *q_idx,
                                const msa_index_k_t *k_idx, int32_t num_kv_heads,
                                int32_t max_blocks, uint32_t flags, float *scores,
                                int32_t *dev_err, struct CUstream_st *stream) {
  if (ragged_ok(rp) && rp->total_q == 0 && index_flags_ok(rp, flags)) return MSA_OK;
  return index_scores_impl(rp, q_idx, k_idx, num_kv_heads, max_blocks, flags, scores, dev_err,
                           reinterpret_cast<cudaStream_t>(stream), nullptr);
}

msa_status_t msa_index_scores(const msa_ragged_paged_t *rp, const void *q_idx,
                              const void *k_idx_cache, int32_t num_kv_heads,
                              int32_t num_idx_k_heads, int32_t max_blocks, float *scores,
                              int32_t *dev_err, struct CUstream_st *stream) {
  const msa_index_k_t k = bf16_index_k(k_idx_cache, num_idx_k_heads);
  return msa_index_scores_k(rp, q_idx, &k, num_kv_heads, max_blocks, 0u, scores, dev_err,
                            stream);
}

size_t msa_index_select_counters(const msa_ragged_paged_t *rp, int32_t num_idx_k_heads) {
  if (!ragged_ok(rp) || num_idx_k_heads < 1) return 0;
  return static_cast<size_t>(rp->batch) * rp->max_q_len * num_idx_k_heads;
}

msa_status_t msa_index_select_k(const msa_ragged_paged_t *rp, const void *q_idx,
                                const msa_index_k_t *k_idx, int32_t num_kv_heads,
                                int32_t max_blocks, int32_t top_k, int32_t init_blocks,
                                int32_t local_blocks, uint32_t flags, float *scores,
                                int32_t *block_ids, int32_t *num_selected, int32_t *counters,
                                int32_t *dev_err, struct CUstream_st *stream) {
  const long long S = static_cast<long long>(top_k) + init_blocks + local_blocks;
  if (!ragged_ok(rp) || num_kv_heads < 1 || !k_idx || k_idx->num_heads < 1 || max_blocks < 1 ||
      top_k < 0 || init_blocks < 0 || local_blocks < 0 || S < 1 || S > (1 << 20) ||
      !index_flags_ok(rp, flags))
    return MSA_ERR_INVALID_ARG;
  if (rp->total_q == 0) return MSA_OK;
  if (!block_ids || !num_selected) return MSA_ERR_INVALID_ARG;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool fused =
      num_kv_heads % k_idx->num_heads == 0 &&
      !index_uses_tc(rp, num_kv_heads / k_idx->num_heads, static_cast<int>(k_idx->dtype)) &&
      !index_uses_tc_pos(rp, num_kv_heads / k_idx->num_heads, static_cast<int>(k_idx->dtype),
                         flags);
  // counters: required on the decode and speculative routes, whether or not this shape uses them
  if (rp->max_q_len <= MSA_MAX_SPEC_DRAFT && (!counters || !aligned(counters, 4)))
    return MSA_ERR_INVALID_ARG;
  if (fused) {
    const FusedSelect fs{counters, block_ids, num_selected, top_k, init_blocks, local_blocks,
                         static_cast<int>(S)};
    return index_scores_impl(rp, q_idx, k_idx, num_kv_heads, max_blocks, flags, scores, dev_err,
                             st, &fs);
  }
  if (flags & MSA_SHARE_ACROSS_DRAFTS) return MSA_ERR_UNSUPPORTED;  // the fused route only
  const msa_status_t e = index_scores_impl(rp, q_idx, k_idx, num_kv_heads, max_blocks, flags,
                                           scores, dev_err, st, nullptr);
  if (e != MSA_OK) return e;
  return msa_select_blocks(rp, scores, num_kv_heads, max_blocks, top_k, init_blocks,
                           local_blocks, block_ids, num_selected, dev_err, stream);
}

msa_status_t msa_index_select(const msa_ragged_paged_t *rp, const void *q_idx,
                              const void *k_idx_cache, int32_t num_kv_heads,
                              int32_t num_idx_k_heads, int32_t max_blocks, int32_t top_k,
                              int32_t init_blocks, int32_t local_blocks, float *scores,
                              int32_t *block_ids, int32_t *num_selected, int32_t *counters,
                              int32_t *dev_err, struct CUstream_st *stream) {
  const msa_index_k_t k = bf16_index_k(k_idx_cache, num_idx_k_heads);
  return msa_index_select_k(rp, q_idx, &k, num_kv_heads, max_blocks, top_k, init_blocks,
                            local_blocks, 0u, scores, block_ids, num_selected, counters, dev_err,
                            stream);
}

msa_status_t msa_select_blocks(const msa_ragged_paged_t *rp, const float *scores,
                               int32_t num_kv_heads, int32_t max_blocks, int32_t top_k,
                               int32_t init_blocks, int32_t local_blocks, int32_t *block_ids,
                               int32_t *num_selected, int32_t *dev_err,
                               struct CUstream_st *stream) {
  const long long S = static_cast<long long>(top_k) + init_blocks + local_blocks;
  if (!ragged_ok(rp) || num_kv_heads < 1 || max_blocks < 1 || top_k < 0 || init_blocks < 0 ||
      local_blocks < 0 || S < 1 || S > (1 << 20))
    return MSA_ERR_INVALID_ARG;
  if (rp->total_q == 0) return MSA_OK;
  if (!scores || !block_ids || !num_selected) return MSA_ERR_INVALID_ARG;
  SelectArgs a;
  a.row_off = rp->input_row_offsets;
  a.cache_len = rp->cache_lengths;
  a.scores = scores;
  a.block_ids = block_ids;
  a.num_selected = num_selected;
  a.dev_err = dev_err;
  a.batch = rp->batch;
  a.total_q = rp->total_q;
  a.H_kv = num_kv_heads;
  a.max_blocks = max_blocks;
  a.top_k = top_k;
  a.init_blocks = init_blocks;
  a.local_blocks = local_blocks;
  a.S = static_cast<int>(S);
  return launch_select(a, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? MSA_OK
                                                                                 : MSA_ERR_CUDA;
}

msa_status_t msa_splitk_combine(const float *partial_o, const float *partial_lse,
                                int32_t num_splits, int32_t total_q, int32_t num_q_heads,
                                void *out, struct CUstream_st *stream) {
  if (num_splits < 1 || total_q < 0 || num_q_heads < 1) return MSA_ERR_INVALID_ARG;
  if (total_q == 0) return MSA_OK;
  if (!partial_o || !partial_lse || !out || !aligned(partial_o, 16) || !aligned(out, 8))
    return MSA_ERR_INVALID_ARG;
  return launch_combine(partial_o, partial_lse, num_splits, total_q, num_q_heads,
                        static_cast<uint16_t *>(out),
                        reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MSA_OK
             : MSA_ERR_CUDA;
}

}  // extern "C"

namespace {

// The selection to run inside the decode attention kernel (msa_select_sparse_attn_paged).
struct AttnSelect {
  const float *scores;
  int32_t *block_ids, *num_selected;
  int top_k, init_blocks, local_blocks;
  // the one-call decode step's flags (ready == nullptr: wait for the whole earlier launch)
  const int32_t *ready = nullptr;
  int32_t *epoch = nullptr, *step_done = nullptr;
  int H_idxk = 1;
};

// Whether msa_select_sparse_attn_paged selects inside the attention kernel for this shape: the
// decode route with one 16-row group per item.
bool select_in_attention(const msa_ragged_paged_t *rp, int num_q_heads, int num_kv_heads) {
  return rp->max_q_len == 1 && num_q_heads / num_kv_heads <= 16;
}

// Whether msa_select_sparse_attn_paged selects and plans in one launch for this shape: the
// speculative route with tiles of at most kMaxSpecTileTokens tokens.
bool select_with_plan(const msa_ragged_paged_t *rp, int S, int num_q_heads, int num_kv_heads,
                      int max_blocks, int num_splits, msa_kv_dtype_t kv_dtype) {
  if (rp->max_q_len <= 1 || rp->max_q_len > MSA_MAX_SPEC_DRAFT) return false;
  Route r;
  if (!make_route(rp, S, num_q_heads, num_kv_heads, max_blocks, num_splits,
                  num_sms_of_current_device(), kv_dtype == MSA_KV_FP8_E4M3, &r))
    return false;
  return r.stream && r.plan && r.qt <= kMaxSpecTileTokens &&
         select_plan_smem_bytes(max_blocks, r.cap, S) <= 200 * 1024;
}

// msa_sparse_attn_paged's body.  dry_run: validate only (nothing enqueued); sel: select inside
// the decode attention kernel (block_ids / num_selected are then its outputs).
msa_status_t attn_impl(const msa_ragged_paged_t *rp, const void *q, const void *k_cache,
                       const void *v_cache, msa_kv_dtype_t kv_dtype, const int32_t *block_ids,
                       const int32_t *num_selected, int32_t S, int32_t num_q_heads,
                       int32_t num_kv_heads, int32_t max_blocks, float scale, int32_t num_splits,
                       void *workspace, size_t workspace_bytes, void *out, int32_t *dev_err,
                       struct CUstream_st *stream, bool dry_run, const AttnSelect *sel) {
  if (ragged_ok(rp) && rp->total_q == 0 && S >= 1) return MSA_OK;  // nothing to attend
  if (!ragged_ok(rp) || !q || !k_cache || !v_cache || !block_ids || !num_selected ||
      S < 1 || num_kv_heads < 1 || num_q_heads < num_kv_heads ||
      num_q_heads % num_kv_heads != 0 || max_blocks < 1 || max_blocks > rp->max_pages_per_seq ||
      !(scale > 0.f) || !isfinite(scale) || num_splits < 0 || num_splits > kMaxSplits ||
      !(kv_dtype == MSA_KV_BF16 || kv_dtype == MSA_KV_FP8_E4M3) || !aligned(q, 16) ||
      !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16))
    return MSA_ERR_INVALID_ARG;
  if (!out && rp->max_q_len > MSA_MAX_SPEC_DRAFT) return MSA_ERR_INVALID_ARG;  // prefill: out
  const int G = num_q_heads / num_kv_heads;
  if (G > kMaxRows) return MSA_ERR_UNSUPPORTED;
  if (static_cast<long long>(rp->num_pages) * num_kv_heads >= (1LL << 31))
    return MSA_ERR_UNSUPPORTED;
  Route r;
  if (!make_route(rp, S, num_q_heads, num_kv_heads, max_blocks, num_splits,
                  num_sms_of_current_device(), kv_dtype == MSA_KV_FP8_E4M3, &r))
    return MSA_ERR_UNSUPPORTED;
  if (r.plan && (2 * ((max_blocks + 31) / 32) + r.cap) * 4 > 200 * 1024)
    return MSA_ERR_UNSUPPORTED;
  if (static_cast<long long>(rp->batch) * r.tiles > 0x7fffffffLL) return MSA_ERR_UNSUPPORTED;
  if (r.bytes > 0 && (!workspace || workspace_bytes < r.bytes || !aligned(workspace, 256)))
    return MSA_ERR_INVALID_ARG;
  // sel: on the decode route the attention kernel selects; on the speculative route one launch
  // selects and plans (tiles of at most kMaxSpecTileTokens tokens)
  if (sel && (!r.stream || (!r.plan && r.rg != 1) || (r.plan && r.qt > kMaxSpecTileTokens) ||
              (r.plan && select_plan_smem_bytes(max_blocks, r.cap, S) > 200 * 1024)))
    return MSA_ERR_UNSUPPORTED;
  if (dry_run) return MSA_OK;

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool fp8 = kv_dtype == MSA_KV_FP8_E4M3;

  if (r.plan && sel) {
    SelectPlanArgs p;
    p.row_off = rp->input_row_offsets;
    p.cache_len = rp->cache_lengths;
    p.scores = sel->scores;
    p.block_ids = sel->block_ids;
    p.num_selected = sel->num_selected;
    p.list = reinterpret_cast<int32_t *>(ws + r.off_list);
    p.masks = reinterpret_cast<uint32_t *>(ws + r.off_masks);
    p.counts = reinterpret_cast<int32_t *>(ws + r.off_counts);
    p.dev_err = dev_err;
    p.batch = rp->batch;
    p.max_q_len = rp->max_q_len;
    p.H_kv = num_kv_heads;
    p.S = S;
    p.max_blocks = max_blocks;
    p.qt = r.qt;
    p.tiles = r.tiles;
    p.cap = r.cap;
    p.top_k = sel->top_k;
    p.init_blocks = sel->init_blocks;
    p.local_blocks = sel->local_blocks;
    if (launch_select_plan(p, s) != cudaSuccess) return MSA_ERR_CUDA;
  } else if (r.plan) {
    PlanArgs p;
    p.row_off = rp->input_row_offsets;
    p.cache_len = rp->cache_lengths;
    p.block_ids = block_ids;
    p.num_selected = num_selected;
    p.list = reinterpret_cast<int32_t *>(ws + r.off_list);
    p.masks = reinterpret_cast<uint32_t *>(ws + r.off_masks);
    p.counts = reinterpret_cast<int32_t *>(ws + r.off_counts);
    p.dev_err = dev_err;
    p.batch = rp->batch;
    p.max_q_len = rp->max_q_len;
    p.H_kv = num_kv_heads;
    p.S = S;
    p.max_blocks = max_blocks;
    p.qt = r.qt;
    p.tiles = r.tiles;
    p.cap = r.cap;
    if (launch_plan(p, s) != cudaSuccess) return MSA_ERR_CUDA;
  }

  CUtensorMap kmap, vmap;
  const long long tiles = static_cast<long long>(rp->num_pages) * num_kv_heads;
  if (!page_tensor_map(&kmap, k_cache, tiles, fp8) || !page_tensor_map(&vmap, v_cache, tiles, fp8))
    return MSA_ERR_CUDA;

  AttnArgs a{};
  a.row_off = rp->input_row_offsets;
  a.cache_len = rp->cache_lengths;
  a.table = rp->kv_lookup_table;
  a.q = static_cast<const uint16_t *>(q);
  a.block_ids = block_ids;
  a.num_selected = num_selected;
  a.plan_list = reinterpret_cast<const int32_t *>(ws + r.off_list);
  a.plan_masks = reinterpret_cast<const uint32_t *>(ws + r.off_masks);
  a.plan_counts = reinterpret_cast<const int32_t *>(ws + r.off_counts);
  a.S = S;
  a.cap = r.cap;
  a.batch = rp->batch;
  a.total_q = rp->total_q;
  a.max_q_len = rp->max_q_len;
  a.max_pages = rp->max_pages_per_seq;
  a.num_pages = rp->num_pages;
  a.H_q = num_q_heads;
  a.H_kv = num_kv_heads;
  a.G = G;
  a.max_blocks = max_blocks;
  a.qt = r.qt;
  a.tiles = r.tiles;
  a.items = r.items;
  a.R = r.R;
  a.P = r.P;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.part_o = reinterpret_cast<float *>(ws + r.off_o);
  a.part_lse = reinterpret_cast<float *>(ws + r.off_lse);
  a.out = static_cast<uint16_t *>(out);
  // one partition: every item lies inside one CTA, which then writes the output itself
  a.direct = r.stream && r.splits == 1 && out != nullptr;
  a.dev_err = dev_err;
  const AttnSelect *in_kernel = r.plan ? nullptr : sel;  // decode: the attention selects
  a.scores = in_kernel ? in_kernel->scores : nullptr;
  a.sel_ids = in_kernel ? in_kernel->block_ids : nullptr;
  a.sel_counts = in_kernel ? in_kernel->num_selected : nullptr;
  a.top_k = in_kernel ? in_kernel->top_k : 0;
  a.init_blocks = in_kernel ? in_kernel->init_blocks : 0;
  a.local_blocks = in_kernel ? in_kernel->local_blocks : 0;
  a.ready = in_kernel ? in_kernel->ready : nullptr;
  a.epoch = in_kernel ? in_kernel->epoch : nullptr;
  a.step_done = in_kernel ? in_kernel->step_done : nullptr;
  a.H_idxk = in_kernel ? in_kernel->H_idxk : 1;
  if (r.tc)
    return launch_attention_tc(kmap, vmap, a, fp8, s) == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
  if (!r.stream)
    return launch_attention_tiles(kmap, vmap, a, fp8, r.rg, s) == cudaSuccess ? MSA_OK
                                                                             : MSA_ERR_CUDA;
  if (launch_attention_stream(kmap, vmap, a, fp8, r.rg, r.plan, r.grid, s) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (!out || a.direct) return MSA_OK;  // no partials, or the caller combines them itself
  if (launch_combine(a.part_o, a.part_lse, r.splits, rp->total_q, num_q_heads, a.out, s) !=
      cudaSuccess)
    return MSA_ERR_CUDA;
  return MSA_OK;
}

}  // namespace

extern "C" {

msa_status_t msa_sparse_attn_paged(const msa_ragged_paged_t *rp, const void *q,
                                   const void *k_cache, const void *v_cache,
                                   msa_kv_dtype_t kv_dtype, const int32_t *block_ids,
                                   const int32_t *num_selected, int32_t S, int32_t num_q_heads,
                                   int32_t num_kv_heads, int32_t max_blocks, float scale,
                                   int32_t num_splits, void *workspace, size_t workspace_bytes,
                                   void *out, int32_t *dev_err, struct CUstream_st *stream) {
  return attn_impl(rp, q, k_cache, v_cache, kv_dtype, block_ids, num_selected, S, num_q_heads,
                   num_kv_heads, max_blocks, scale, num_splits, workspace, workspace_bytes, out,
                   dev_err, stream, false, nullptr);
}

msa_status_t msa_select_sparse_attn_paged(
    const msa_ragged_paged_t *rp, const float *scores, int32_t top_k, int32_t init_blocks,
    int32_t local_blocks, const void *q, const void *k_cache, const void *v_cache,
    msa_kv_dtype_t kv_dtype, int32_t num_q_heads, int32_t num_kv_heads, int32_t max_blocks,
    float scale, int32_t num_splits, void *workspace, size_t workspace_bytes,
    int32_t *block_ids, int32_t *num_selected, void *out, int32_t *dev_err,
    struct CUstream_st *stream) {
  const long long S = static_cast<long long>(top_k) + init_blocks + local_blocks;
  if (!ragged_ok(rp) || top_k < 0 || init_blocks < 0 || local_blocks < 0 || S < 1 ||
      S > (1 << 20) || num_kv_heads < 1 || num_q_heads < num_kv_heads)
    return MSA_ERR_INVALID_ARG;
  if (rp->total_q == 0) return MSA_OK;
  if (!scores || !block_ids || !num_selected) return MSA_ERR_INVALID_ARG;
  const int Si = static_cast<int>(S);
  // everything validated before anything is enqueued
  const msa_status_t v = attn_impl(rp, q, k_cache, v_cache, kv_dtype, block_ids, num_selected,
                                   Si, num_q_heads, num_kv_heads, max_blocks, scale, num_splits,
                                   workspace, workspace_bytes, out, dev_err, stream, true,
                                   nullptr);
  if (v != MSA_OK) return v;
  if (select_in_attention(rp, num_q_heads, num_kv_heads) ||
      select_with_plan(rp, Si, num_q_heads, num_kv_heads, max_blocks, num_splits, kv_dtype)) {
    const AttnSelect sel{scores, block_ids, num_selected, top_k, init_blocks, local_blocks};
    return attn_impl(rp, q, k_cache, v_cache, kv_dtype, block_ids, num_selected, Si,
                     num_q_heads, num_kv_heads, max_blocks, scale, num_splits, workspace,
                     workspace_bytes, out, dev_err, stream, false, &sel);
  }
  const msa_status_t e = msa_select_blocks(rp, scores, num_kv_heads, max_blocks, top_k,
                                           init_blocks, local_blocks, block_ids, num_selected,
                                           dev_err, stream);
  if (e != MSA_OK) return e;
  return attn_impl(rp, q, k_cache, v_cache, kv_dtype, block_ids, num_selected, Si, num_q_heads,
                   num_kv_heads, max_blocks, scale, num_splits, workspace, workspace_bytes, out,
                   dev_err, stream, false, nullptr);
}

// ---------------------------------------------------------------- one-call decode step
// Words before the attention's workspace: the step epoch, the attention's done counter, the
// indexer's per-unit counters and the per-unit ready flags.
static size_t step_sync_bytes(const msa_ragged_paged_t *rp, int32_t num_idx_k_heads) {
  const size_t units = static_cast<size_t>(rp->batch) * rp->max_q_len * num_idx_k_heads;
  return (((2 + 2 * units) * sizeof(int32_t)) + 255) / 256 * 256;
}

size_t msa_decode_step_workspace_bytes(const msa_ragged_paged_t *rp, int32_t S,
                                       int32_t num_q_heads, int32_t num_kv_heads,
                                       int32_t num_idx_k_heads, int32_t max_blocks,
                                       int32_t num_splits) {
  if (!ragged_ok(rp) || num_idx_k_heads < 1) return 0;
  return step_sync_bytes(rp, num_idx_k_heads) +
         msa_attn_workspace_bytes(rp, S, num_q_heads, num_kv_heads, max_blocks, num_splits);
}

msa_status_t msa_decode_step(const msa_ragged_paged_t *rp, const void *q_idx,
                             const msa_index_k_t *k_idx, int32_t top_k, int32_t init_blocks,
                             int32_t local_blocks, const void *q, const void *k_cache,
                             const void *v_cache, msa_kv_dtype_t kv_dtype, int32_t num_q_heads,
                             int32_t num_kv_heads, int32_t max_blocks, float scale,
                             int32_t num_splits, void *workspace, size_t workspace_bytes,
                             float *scores, int32_t *block_ids, int32_t *num_selected, void *out,
                             int32_t *dev_err, struct CUstream_st *stream) {
  const long long S = static_cast<long long>(top_k) + init_blocks + local_blocks;
  if (!ragged_ok(rp) || !k_idx || k_idx->num_heads < 1 || top_k < 0 || init_blocks < 0 ||
      local_blocks < 0 || S < 1 || S > (1 << 20) || num_kv_heads < 1 ||
      num_q_heads < num_kv_heads)
    return MSA_ERR_INVALID_ARG;
  if (rp->total_q == 0) return MSA_OK;
  if (!scores || !block_ids || !num_selected || !workspace || !aligned(workspace, 256))
    return MSA_ERR_INVALID_ARG;
  const size_t sync = step_sync_bytes(rp, k_idx->num_heads);
  if (workspace_bytes < sync) return MSA_ERR_INVALID_ARG;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  void *attn_ws = ws + sync;
  const size_t attn_bytes = workspace_bytes - sync;
  const int Si = static_cast<int>(S);
  const bool fast = select_in_attention(rp, num_q_heads, num_kv_heads) &&
                    num_kv_heads % k_idx->num_heads == 0 &&
                    !index_uses_tc(rp, num_kv_heads / k_idx->num_heads,
                                   static_cast<int>(k_idx->dtype));
  if (!fast) {  // the two calls one after the other
    const msa_status_t v = attn_impl(rp, q, k_cache, v_cache, kv_dtype, block_ids,
                                     num_selected, Si, num_q_heads, num_kv_heads, max_blocks,
                                     scale, num_splits, attn_ws, attn_bytes, out, dev_err,
                                     stream, true, nullptr);
    if (v != MSA_OK) return v;
    const msa_status_t e = msa_index_scores_k(rp, q_idx, k_idx, num_kv_heads, max_blocks, 0u,
                                              scores, dev_err, stream);
    if (e != MSA_OK) return e;
    return msa_select_sparse_attn_paged(rp, scores, top_k, init_blocks, local_blocks, q,
                                        k_cache, v_cache, kv_dtype, num_q_heads, num_kv_heads,
                                        max_blocks, scale, num_splits, attn_ws, attn_bytes,
                                        block_ids, num_selected, out, dev_err, stream);
  }
  int32_t *words = reinterpret_cast<int32_t *>(ws);
  const size_t units = static_cast<size_t>(rp->batch) * rp->max_q_len * k_idx->num_heads;
  int32_t *epoch = words, *step_done = words + 1, *counters = words + 2;
  int32_t *ready = counters + units;
  AttnSelect sel{scores, block_ids, num_selected, top_k, init_blocks, local_blocks};
  sel.ready = ready;
  sel.epoch = epoch;
  sel.step_done = step_done;
  sel.H_idxk = k_idx->num_heads;
  const msa_status_t v = attn_impl(rp, q, k_cache, v_cache, kv_dtype, block_ids, num_selected,
                                   Si, num_q_heads, num_kv_heads, max_blocks, scale, num_splits,
                                   attn_ws, attn_bytes, out, dev_err, stream, true, &sel);
  if (v != MSA_OK) return v;
  FusedSelect fs{counters, nullptr, nullptr, top_k, init_blocks, local_blocks, Si};
  fs.publish = ready;
  fs.epoch = epoch;
  const msa_status_t e = index_scores_impl(rp, q_idx, k_idx, num_kv_heads, max_blocks, 0u,
                                           scores, dev_err,
                                           reinterpret_cast<cudaStream_t>(stream), &fs);
  if (e != MSA_OK) return e;
  return attn_impl(rp, q, k_cache, v_cache, kv_dtype, block_ids, num_selected, Si, num_q_heads,
                   num_kv_heads, max_blocks, scale, num_splits, attn_ws, attn_bytes, out,
                   dev_err, stream, false, &sel);
}

}  // extern "C"

// ---------------------------------------------------------------- latent sparse attention
namespace {

constexpr int kLatMaxSplits = 64;

bool leaf_ok(const msa_latent_leaf_t *l, int32_t batch) {
  return l && l->kv && l->cache_lengths && l->lookup_table && l->max_pages_per_seq >= 1 &&
         l->num_pages >= 1 && l->num_layers >= 1 && l->layer >= 0 && l->layer < l->num_layers &&
         aligned(l->kv, 16) && batch >= 1;
}

}  // namespace

extern "C" {

size_t msa_latent_workspace_bytes(int32_t total_q, int32_t num_heads, int32_t num_splits) {
  if (total_q < 1 || num_heads < 1 || num_splits <= 1) return 0;
  const size_t rows = static_cast<size_t>(num_splits) * total_q * num_heads;
  return round_up(rows * kHeadDim * sizeof(float), 256) + round_up(rows * sizeof(float), 256);
}

int32_t msa_latent_default_splits(int32_t total_q, int32_t num_heads, int32_t window,
                                  int32_t n_entries, int32_t num_sms) {
  if (total_q < 1 || num_heads < 1 || window < 1 || n_entries < 0 || num_sms < 1) return 1;
  const long long items =
      static_cast<long long>(total_q) * ((num_heads + latent_rows_per_cta() - 1) /
                                         latent_rows_per_cta());
  const long long want = (2LL * num_sms + items - 1) / items;
  const long long tiles = (static_cast<long long>(window) + n_entries +
                           latent_tile_positions() - 1) / latent_tile_positions();
  long long s = std::min<long long>(want, std::max<long long>(1, tiles / 2));
  s = std::max<long long>(1, std::min<long long>(s, kLatMaxSplits));
  return static_cast<int32_t>(s);
}

msa_status_t msa_latent_sparse_attn_paged(
    const int32_t *input_row_offsets, int32_t batch, int32_t total_q, int32_t max_q_len,
    const void *q, int32_t num_heads, const msa_latent_leaf_t *swa, int32_t window,
    const msa_latent_leaf_t *comp, const int32_t *comp_indices, int32_t n_entries,
    const float *attn_sink, float scale, int32_t num_splits, void *workspace,
    size_t workspace_bytes, void *out, int32_t *dev_err, struct CUstream_st *stream) {
  if (!input_row_offsets || batch < 1 || total_q < 0 || max_q_len < 1 || num_heads < 1 ||
      !leaf_ok(swa, batch) || !leaf_ok(comp, batch) || window < 1 || n_entries < 0 ||
      (n_entries > 0 && (!comp_indices || !aligned(comp_indices, 4))) || !attn_sink ||
      !(scale > 0.f) || !isfinite(scale) || num_splits < 0 || num_splits > kLatMaxSplits)
    return MSA_ERR_INVALID_ARG;
  if (total_q == 0) return MSA_OK;
  if (!q || !out || !aligned(q, 16) || !aligned(out, 16)) return MSA_ERR_INVALID_ARG;
  if ((num_heads + latent_rows_per_cta() - 1) / latent_rows_per_cta() > 65535)
    return MSA_ERR_UNSUPPORTED;
  const int splits = num_splits > 0 ? num_splits
                                    : msa_latent_default_splits(total_q, num_heads, window,
                                                                n_entries,
                                                                num_sms_of_current_device());
  const size_t need = msa_latent_workspace_bytes(total_q, num_heads, splits);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 256)))
    return MSA_ERR_INVALID_ARG;
  LatentArgs a;
  a.row_off = input_row_offsets;
  a.batch = batch;
  a.total_q = total_q;
  a.max_q_len = max_q_len;
  a.q = static_cast<const uint16_t *>(q);
  a.H = num_heads;
  a.swa_kv = static_cast<const uint16_t *>(swa->kv);
  a.swa_len = swa->cache_lengths;
  a.swa_table = swa->lookup_table;
  a.swa_pages = swa->num_pages;
  a.swa_layers = swa->num_layers;
  a.swa_layer = swa->layer;
  a.swa_max_pages = swa->max_pages_per_seq;
  a.window = window;
  a.comp_kv = static_cast<const uint16_t *>(comp->kv);
  a.comp_len = comp->cache_lengths;
  a.comp_table = comp->lookup_table;
  a.comp_pages = comp->num_pages;
  a.comp_layers = comp->num_layers;
  a.comp_layer = comp->layer;
  a.comp_max_pages = comp->max_pages_per_seq;
  a.comp_idx = comp_indices;
  a.n_entries = n_entries;
  a.sink = attn_sink;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.splits = splits;
  const size_t rows = static_cast<size_t>(splits) * total_q * num_heads;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  a.part_o = need ? reinterpret_cast<float *>(ws) : nullptr;
  a.part_lse = need ? reinterpret_cast<float *>(ws + round_up(rows * kHeadDim * sizeof(float),
                                                              256))
                    : nullptr;
  a.out = static_cast<uint16_t *>(out);
  a.dev_err = dev_err;
  return launch_latent_attention(a, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MSA_OK
             : MSA_ERR_CUDA;
}

}  // extern "C"
