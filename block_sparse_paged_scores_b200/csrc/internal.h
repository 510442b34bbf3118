// internal.h — argument blocks and launchers shared between the kernels and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "msa.h"

namespace msa {

constexpr int kBlock = 128;    // tokens per block == tokens per page
constexpr int kHeadDim = 128;  // head dim of q / k / v / q_idx / k_idx

// ---- stage 1: block scores (indexer.cu)
constexpr int kIdxBf16 = 0, kIdxFp8 = 1, kIdxFp4 = 2;  // index-K formats (msa_idx_dtype_t)
struct IndexerArgs {
  const int32_t *row_off, *cache_len, *table;
  const uint16_t *q_idx;  // bf16 bits [total_q, H_kv, 128]
  int idx_fmt;               // kIdxBf16 / kIdxFp8 / kIdxFp4
  const void *k_idx_scale;   // fp8: f32 [pages, H_idxk, 128]; fp4: u8 [pages, H_idxk, 128, 4]
  float *scores;          // [total_q, H_kv, max_blocks]
  int32_t *dev_err;
  int batch, max_q_len, max_pages, num_pages, H_kv, H_idxk, max_blocks;
  int qt;     // query tokens per tile
  int tiles;  // tiles per sequence
  int chunk;   // pages per CTA
  int chunks;  // CTAs per (sequence, tile, index-K head)
  // Selection fused into the decode indexer (counters == nullptr: scores only).  The CTAs of one
  // (sequence, tile, index-K head) count themselves out on counters[(b * tiles + tile) * H_idxk
  // + hk]; the last one selects for the unit's rows and puts the counter back to zero.
  int32_t *counters;
  int32_t *block_ids, *num_selected;  // [total_q, H_kv, S], [total_q, H_kv]
  int top_k, init_blocks, local_blocks, S;
  // Top-k shared across each sequence's new tokens: one tile of one token (the first) per
  // sequence is scored, and the fused selection writes every token's row from it.
  int share;
  // One-call decode step (publish != nullptr, counters set, no fused selection): the last CTA
  // of every unit publishes publish[unit] = *epoch + 1 (release) once the unit's scores are
  // written, so that the attention launch, already running, can select that unit's rows.
  int32_t *publish;
  const int32_t *epoch;
};
// mt = 16-row MMA tiles per CTA (1 or 2)
cudaError_t launch_index_scores(const CUtensorMap &kidx_map, const IndexerArgs &a, int mt,
                                int chunks, cudaStream_t s);
// prefill on tcgen05 (indexer_tc.cu): tiles of qt tokens x (H_kv / H_idxk) heads <= 128 rows,
// every visible page of the tile in one CTA
cudaError_t launch_index_scores_tc(const CUtensorMap &kidx_map, const IndexerArgs &a,
                                   cudaStream_t s);
// speculative route on tcgen05 (indexer_tc.cu): a page's 128 positions as M and the unit's
// qt x (H_kv / H_idxk) <= 32 rows as N = 32; the warp-MMA kernel's grid of chunks
cudaError_t launch_index_scores_tc_pos(const CUtensorMap &kidx_map, const IndexerArgs &a,
                                       int chunks, cudaStream_t s);

// ---- stage 2: selection (select.cu)
struct SelectArgs {
  const int32_t *row_off, *cache_len;
  const float *scores;
  int32_t *block_ids, *num_selected, *dev_err;
  int batch, total_q, H_kv, max_blocks, top_k, init_blocks, local_blocks, S;
};
cudaError_t launch_select(const SelectArgs &a, cudaStream_t s);

// ---- per-tile union of the tokens' selections (plan.cu)
struct PlanArgs {
  const int32_t *row_off, *cache_len, *block_ids, *num_selected;
  int32_t *list;     // [items, cap] ascending block ids
  uint32_t *masks;   // [items, cap] bit i: token tok0 + i selected the block
  int32_t *counts;   // [items]
  int32_t *dev_err;
  int batch, max_q_len, H_kv, S, max_blocks, qt, tiles, cap;
};
cudaError_t launch_plan(const PlanArgs &a, cudaStream_t s);

// ---- the speculative route's selection and plan in one launch (select_plan.cu): one CTA of qt
// warps per (sequence, query tile, KV head); writes what select.cu and plan.cu write
constexpr int kMaxSpecTileTokens = 8;  // tokens per speculative query tile (warps per CTA)
struct SelectPlanArgs {
  const int32_t *row_off, *cache_len;
  const float *scores;
  int32_t *block_ids, *num_selected;  // [total_q, H_kv, S], [total_q, H_kv]
  int32_t *list;                      // [items, cap]
  uint32_t *masks;                    // [items, cap]
  int32_t *counts;                    // [items]
  int32_t *dev_err;
  int batch, max_q_len, H_kv, S, max_blocks, qt, tiles, cap;
  int top_k, init_blocks, local_blocks;
};
size_t select_plan_smem_bytes(int max_blocks, int cap, int S);
cudaError_t launch_select_plan(const SelectPlanArgs &a, cudaStream_t s);

// ---- stage 3: sparse paged attention (attention_stream.cu: decode / speculative,
//      attention_tile.cu: prefill)
struct AttnArgs {
  const int32_t *row_off, *cache_len, *table;
  const uint16_t *q;  // bf16 bits [total_q, H_q, 128]
  const int32_t *block_ids, *num_selected;  // decode route: the selection itself
  const int32_t *plan_list;                 // other routes: the per-tile union
  const uint32_t *plan_masks;
  const int32_t *plan_counts;
  int S, cap;  // cap: work-list slots per item (decode: S; others: the union capacity)
  int batch, total_q, max_q_len, max_pages, num_pages, H_q, H_kv, G, max_blocks;
  int qt, tiles;
  int items;    // batch * tiles * H_kv
  long long R;  // persistent kernel: work-list slots per CTA
  int P;        // persistent kernel: most CTAs one item's slots can span
  float scale_log2;          // scale * log2(e)
  float *part_o, *part_lse;  // persistent kernel: [P][total_q][H_q][128] and [P][total_q][H_q]
  uint16_t *out;             // bf16 bits [total_q, H_q, 128]: tile kernels, and the persistent
                             // kernel when `direct`
  int direct;                // persistent kernel with P == 1 (every item inside one CTA): write
                             // O / l to `out` instead of partials (no combine follows)
  // Selection inside the decode attention kernel (sel_ids != nullptr): every CTA first selects
  // the rows of its items from `scores` into sel_ids / sel_counts (== block_ids / num_selected).
  const float *scores;
  int32_t *sel_ids, *sel_counts;
  int top_k, init_blocks, local_blocks;
  // One-call decode step (ready != nullptr, with the selection inside): the kernel does not
  // wait for the whole indexer launch; each row's scores are read once its unit's flag
  // ready[b * H_idxk + g % H_idxk] equals *epoch + 1 (acquire, bounded wait).  The last CTA
  // to finish counting on *step_done sets it back to zero and advances *epoch.
  const int32_t *ready;
  int32_t *epoch, *step_done;
  int H_idxk;
  int32_t *dev_err;
};
// rg = 16-row groups (1..4); plan = read the per-tile union instead of the selection
cudaError_t launch_attention_stream(const CUtensorMap &kmap, const CUtensorMap &vmap,
                                    const AttnArgs &a, bool fp8, int rg, bool plan, int grid,
                                    cudaStream_t s);
cudaError_t launch_attention_tiles(const CUtensorMap &kmap, const CUtensorMap &vmap,
                                   const AttnArgs &a, bool fp8, int rg, cudaStream_t s);
// prefill on tcgen05 (attention_tc.cu): tiles of qt tokens x G heads <= 128 rows; BF16 KV, or
// e4m3 KV converted to f16 in shared memory (f16 MMAs)
bool attention_tc_supported(int G, int qt);
cudaError_t launch_attention_tc(const CUtensorMap &kmap, const CUtensorMap &vmap,
                                const AttnArgs &a, bool fp8, cudaStream_t s);

// ---- latent sparse attention (latent.cu)
struct LatentArgs {
  const int32_t *row_off;
  int batch, total_q, max_q_len;
  const uint16_t *q;  // bf16 bits [total_q, H, 128]
  int H;
  // sliding-window leaf: bf16 [swa_pages, swa_layers, 128, 128], swa_len = prior tokens
  const uint16_t *swa_kv;
  const int32_t *swa_len, *swa_table;
  int swa_pages, swa_layers, swa_layer, swa_max_pages, window;
  // compressed leaf: bf16 [comp_pages, comp_layers, 128, 128], comp_len = its entries
  const uint16_t *comp_kv;
  const int32_t *comp_len, *comp_table;
  int comp_pages, comp_layers, comp_layer, comp_max_pages;
  const int32_t *comp_idx;  // [total_q, n_entries], -1 = padding
  int n_entries;
  const float *sink;  // [H]
  float scale_log2;
  int splits;                // position-list splits (grid.z); 1: the kernel writes `out`
  float *part_o, *part_lse;  // [splits][total_q][H][128], [splits][total_q][H]
  uint16_t *out;             // bf16 bits [total_q, H, 128]
  int32_t *dev_err;
};
int latent_rows_per_cta();
int latent_tile_positions();
// enqueues the attention and, with more than one split, the combine
cudaError_t launch_latent_attention(const LatentArgs &a, cudaStream_t s);

// ---- split-K combine (combine.cu)
cudaError_t launch_combine(const float *part_o, const float *part_lse, int splits, int total_q,
                           int H_q, uint16_t *out, cudaStream_t s);

// Sets the dynamic shared-memory limit of `func` once per device.
cudaError_t ensure_smem_limit(const void *func, int bytes);

// Launch with programmatic stream serialization: the kernel may start while its predecessor
// in the stream finishes; every kernel of this library calls pdl_wait() before it touches
// global memory that an earlier kernel may write or read.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace msa
