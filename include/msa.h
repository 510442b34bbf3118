/*
 * msa.h — C ABI of libmsa.so: MiniMax-M3 block-sparse attention (MSA) over a paged KV cache,
 * native to NVIDIA B200 (sm_100a).
 *
 * The path has three stages, one entry point each, plus the split-K combine:
 *   msa_index_scores      block scores: max over a 128-token block of raw q_idx . k_idx
 *   msa_select_blocks     forced init/local blocks + top-k of the rest, ascending
 *   msa_index_select      the first two in one call (one launch on the decode routes)
 *   msa_select_sparse_attn_paged  the last two in one call (one launch on the decode route)
 *   msa_sparse_attn_paged softmax attention over the selected pages (decode / speculative /
 *                         prefill routes picked from max_q_len), split-K + combine inside
 *   msa_splitk_combine    log-sum-exp merge of split-K partials into the ragged output
 *
 * Sources (page title, section):
 *   [msa]    Mojo module "msa" (Graph-op bindings for the MiniMax-M3 block-sparse attention
 *            kernels): module summary, the two graph ops, "Three attention routes",
 *            MAX_SPEC_DRAFT.
 *   [ferrox] ferrox-core "Module block_sparse": "Four rules", "The block size is an ABI",
 *            BlockSparseConfig, block_sparse_select, positions_of_blocks.
 *   [latent] Mojo "Struct_latent_sparse_attention_ragged_paged": the ragged / paged argument
 *            set (input_row_offsets, cache_lengths, kv_lookup_table, scale).
 *   [trtllm] TensorRT-LLM "DeepSeekSparseAttentionConfig": indexer_k_dtype (scaled FP8 / FP4
 *            index-K caches).
 *
 * Conventions shared by every entry point
 *   - Head dim and page size are both 128 and fixed ([msa] summary; [ferrox] "The block size
 *     is an ABI").  Index-K is BF16 ([msa]) or a scaled FP8 / FP4 format ([trtllm],
 *     msa_index_scores_k); main K/V is BF16 or scale-free FP8 e4m3 ([msa]).
 *   - Every pointer argument named "device" must point to device memory owned by the caller.
 *     The library allocates no device memory, never synchronises, and never reads device
 *     memory from the host.  Every call only enqueues work on `stream` and returns.
 *   - Host-side validation happens before anything is enqueued; a call that returns anything
 *     but MSA_OK has enqueued nothing.  A failed launch returns MSA_ERR_CUDA.
 *   - `dev_err` (device int32, nullable): kernels OR a bit mask of MSA_DEVERR_* into it when
 *     they meet a device-side value outside the declared bounds; the offending work is skipped
 *     (never read out of bounds, never trap).  The caller zeroes it and reads it when it likes.
 *   - Outputs must not alias inputs.
 *   - Query row t of sequence b is row input_row_offsets[b] + i, at position
 *     p = cache_lengths[b] + i ([msa] "Three attention routes", speculative route).  The new
 *     tokens' k / v / k_idx rows are already in the cache at [cache_lengths[b], L_b) with
 *     L_b = cache_lengths[b] + q_len_b.  Block j covers positions [128 j, 128 j + 128) and is
 *     stored in page kv_lookup_table[b * max_pages_per_seq + j].  A query at p sees the
 *     nb(p) = p / 128 + 1 blocks whose first position is <= p.
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t == struct CUstream_st*; NULL = the legacy default stream */

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

#define MSA_BLOCK 128    /* tokens per block == tokens per page ([ferrox] MINIMAX_BLOCK_SIZE) */
#define MSA_HEAD_DIM 128 /* [msa] summary: head_dim 128 */
#define MSA_MAX_SPEC_DRAFT 8 /* [msa] MAX_SPEC_DRAFT: largest max_q_len of the speculative route */

typedef enum {
    MSA_OK = 0,
    MSA_ERR_INVALID_ARG = 1, /* a null pointer, a size out of range, a too-small workspace */
    MSA_ERR_UNSUPPORTED = 2, /* valid but not built: e.g. a GQA group above the kernel limit */
    MSA_ERR_CUDA = 3         /* the CUDA runtime refused a launch or a tensor-map encode */
} msa_status_t;

typedef enum { MSA_KV_BF16 = 0, MSA_KV_FP8_E4M3 = 1 } msa_kv_dtype_t;

/* Bits OR-ed into *dev_err by the kernels. */
#define MSA_DEVERR_PAGE_ID 1u      /* a page id outside [0, num_pages): that block is skipped */
#define MSA_DEVERR_LENGTHS 2u      /* q_len_b > max_q_len, q_len_b < 0 or nb(p) > max_blocks */
#define MSA_DEVERR_BLOCK_ID 4u     /* a selected id outside [0, nb(p)) or not ascending */
#define MSA_DEVERR_NUM_SELECTED 8u /* num_selected outside [0, S] */
#define MSA_DEVERR_TIMEOUT 16u     /* a pipeline wait gave up (bounded spin); output invalid */

/* The ragged batch and its page table ([latent] argument set; [msa] routes). */
typedef struct {
    const int32_t *input_row_offsets; /* device [batch + 1], non-decreasing, [0] == 0 */
    const int32_t *cache_lengths;     /* device [batch], prior tokens of each sequence */
    const int32_t *kv_lookup_table;   /* device [batch * max_pages_per_seq] physical page ids */
    int32_t batch;                    /* host: number of sequences, >= 1 */
    int32_t total_q;                  /* host: input_row_offsets[batch] */
    int32_t max_q_len;                /* host: max over b of q_len_b; picks the route */
    int32_t max_pages_per_seq;        /* host: row stride of kv_lookup_table */
    int32_t num_pages;                /* host: pages in each paged cache pool */
} msa_ragged_paged_t;

/*
 * msa_index_scores — stage 1 ([ferrox] "Four rules": a block's score is the MAX over its
 * positions, no softmax scale, one index head per KV head; [msa]: the indexer op, single
 * BF16 index-K head).
 *
 *   scores[t, g, j] = max over pos in [128 j, min(128 j + 127, p)] of
 *                     sum_c q_idx[t, g, c] * k_idx[page(b, j), g % num_idx_k_heads, pos - 128 j, c]
 *   for j < nb(p); -inf for nb(p) <= j < max_blocks.  FP32 accumulation of exact BF16
 *   products.  Positions > p (and so every position >= L_b) never enter the max.
 *
 *   q_idx        device bf16 [total_q, num_kv_heads, 128], 16-byte aligned
 *   k_idx_cache  device bf16 [num_pages, num_idx_k_heads, 128 tokens, 128], 16-byte aligned
 *   num_idx_k_heads  1 (one index-K head shared by all index-query heads) or num_kv_heads
 *   max_blocks   row length of `scores`; must be >= nb(p) of every query and
 *                <= max_pages_per_seq; a larger nb(p) sets MSA_DEVERR_LENGTHS and is clipped
 *   scores       device fp32 [total_q, num_kv_heads, max_blocks] (output)
 */
MSA_API msa_status_t msa_index_scores(const msa_ragged_paged_t *rp, const void *q_idx,
                              const void *k_idx_cache, int32_t num_kv_heads,
                              int32_t num_idx_k_heads, int32_t max_blocks, float *scores,
                              int32_t *dev_err, struct CUstream_st *stream);

/*
 * msa_select_blocks — stage 2 ([ferrox] "Four rules": first init_blocks and newest
 * local_blocks forced in, before any scoring; block_sparse_select returns ids ascending;
 * BlockSparseConfig {top_k, init_blocks, local_blocks}).
 *
 *   F = {j < min(init_blocks, nb)} U {max(0, nb - local_blocks) <= j < nb}, nb = nb(p)
 *   C = [0, nb) \ F;  T = the top_k blocks of C by score (equal scores: the lower id first;
 *   -0.0 equals +0.0); all of C when |C| <= top_k.
 *   block_ids[t, g, :] = F U T ascending, then -1 up to S = init + local + top_k;
 *   num_selected[t, g] = |F U T| (>= 1: the selection is never empty).
 *
 *   scores        device fp32 [total_q, num_kv_heads, max_blocks] (as msa_index_scores)
 *   block_ids     device int32 [total_q, num_kv_heads, S] (output)
 *   num_selected  device int32 [total_q, num_kv_heads] (output)
 *   init_blocks, local_blocks, top_k >= 0 with S >= 1; max_blocks <= 65536.
 */
MSA_API msa_status_t msa_select_blocks(const msa_ragged_paged_t *rp, const float *scores,
                               int32_t num_kv_heads, int32_t max_blocks, int32_t top_k,
                               int32_t init_blocks, int32_t local_blocks, int32_t *block_ids,
                               int32_t *num_selected, int32_t *dev_err,
                               struct CUstream_st *stream);

/*
 * msa_index_select — stages 1 and 2 in one call: exactly msa_index_scores followed by
 * msa_select_blocks with the same arguments ([ferrox] "Four rules"; block_sparse_select), with
 * bit-identical scores, block_ids and num_selected.
 *
 * On the decode and speculative routes (max_q_len <= MSA_MAX_SPEC_DRAFT) it is one launch: the
 * CTAs that score one (sequence, tile of query tokens, index-K head) count themselves out on
 * `counters`, and the last one selects for that unit's rows, so the selection needs no launch
 * of its own.  Two cases enqueue the two stages one after the other instead and do not touch
 * `counters`: the prefill route, and the speculative route with a BF16 index-K cache, the
 * top-k per token and units of more than 16 rows (tokens of a tile x index-query heads of one
 * index-K head), which score on the tensor cores.
 *
 *   scores, block_ids, num_selected  as msa_index_scores / msa_select_blocks (all outputs;
 *                  `scores` stays valid after the call, as the selection's input)
 *   counters      device int32 [msa_index_select_counters(rp, num_idx_k_heads)], 4-byte
 *                 aligned, owned by the caller.  It must be all zero when the call's kernel
 *                 starts; the kernel leaves it all zero when it ends, so the caller zeroes it
 *                 once and reuses it.  Two calls in flight at once (on different streams) must
 *                 not share one counters array: their counts would mix.  Required on the decode
 *                 and speculative routes (MSA_ERR_INVALID_ARG when NULL there).
 *   Validation is that of both stages; max_blocks <= max_pages_per_seq.
 */
MSA_API size_t msa_index_select_counters(const msa_ragged_paged_t *rp, int32_t num_idx_k_heads);
MSA_API msa_status_t msa_index_select(const msa_ragged_paged_t *rp, const void *q_idx,
                              const void *k_idx_cache, int32_t num_kv_heads,
                              int32_t num_idx_k_heads, int32_t max_blocks, int32_t top_k,
                              int32_t init_blocks, int32_t local_blocks, float *scores,
                              int32_t *block_ids, int32_t *num_selected, int32_t *counters,
                              int32_t *dev_err, struct CUstream_st *stream);

/*
 * Scaled index-K caches ([trtllm] TensorRT-LLM "DeepSeekSparseAttentionConfig", field
 * indexer_k_dtype: fp8 stores one E4M3 byte per element with a per-128 float32 scale, 132 B per
 * token; fp4 packs two E2M1 codes per byte with a per-32 UE8M0 exponent, 68 B per token).
 *
 * Element c of token `tok` of (page, head) tile r = page * num_heads + head is
 *   MSA_IDX_BF16      codes bf16 [r][tok][c]
 *   MSA_IDX_FP8_E4M3  e4m3(codes u8 [r][tok][c]) * scales f32 [r][tok]
 *   MSA_IDX_FP4_E2M1  e2m1(nibble) * 2^(scales u8 [r][tok][c / 32] - 127), the nibble being the
 *                     low half of codes u8 [r][tok][c / 2] for even c, the high half for odd c
 * (e4m3: the "fn" variant, bias 7, no infinities; e2m1: bias 1, values 0 .. 6; UE8M0 0xFF is
 * NaN).  The scales tensor of one tile is 512 contiguous bytes in both scaled formats.  Scores
 * are the max over positions of sum_c q_idx[c] * element(c), accumulated in fp32; the scaled
 * formats multiply q_idx (converted to f16 after a power-of-two prescale that keeps every row
 * below 2^15 in magnitude, undone exactly) with the codes (converted to f16 exactly) and apply
 * the scales to the fp32 products.  A q_idx element of magnitude below 2^-14 (after the
 * prescale) is rounded to f16's subnormal grid (absolute error <= 2^-25).
 */
typedef enum {
    MSA_IDX_BF16 = 0,
    MSA_IDX_FP8_E4M3 = 1, /* e4m3 codes + one f32 scale per token */
    MSA_IDX_FP4_E2M1 = 2  /* e2m1 code pairs + one UE8M0 exponent per 32 elements */
} msa_idx_dtype_t;

typedef struct {
    msa_idx_dtype_t dtype;
    const void *codes;  /* device, 16-byte aligned: bf16 [num_pages, num_heads, 128, 128] |
                           u8 [num_pages, num_heads, 128, 128] | u8 [num_pages, num_heads, 128,
                           64] */
    const void *scales; /* device, 16-byte aligned: NULL (bf16) | f32 [num_pages, num_heads,
                           128] | u8 [num_pages, num_heads, 128, 4] */
    int32_t num_heads;  /* 1 or num_kv_heads (as num_idx_k_heads) */
} msa_index_k_t;

/*
 * msa_index_scores_k / msa_index_select_k — msa_index_scores / msa_index_select over an index-K
 * cache in any msa_idx_dtype_t (the BF16 entry points are these with MSA_IDX_BF16 and flags 0;
 * their results are bit-identical).  Scaled formats run the warp-MMA indexer on every route
 * (the tensor-core indexers, of the prefill route and of speculative units of more than 16
 * rows, take BF16 only).
 *
 * flags: 0, or MSA_SHARE_ACROSS_DRAFTS ([trtllm] index_share_for_mtp_iteration: reuse the
 * indexer top-k across draft tokens instead of recomputing it for each), accepted on the
 * decode and speculative routes (max_q_len <= MSA_MAX_SPEC_DRAFT; MSA_ERR_INVALID_ARG
 * otherwise).  Then only the first new token of each sequence is scored (the other rows of
 * `scores` are not written), and msa_index_select_k selects for every new token t of the
 * sequence its own forced blocks (init / local, for its own position) together with the top_k
 * of the first token's candidates (its visible blocks minus its own forced blocks) by the
 * first token's scores, ascending.  Those blocks lie below the first token's position, so every
 * later token can read them.  num_selected[t] <= S as ever.
 */
#define MSA_SHARE_ACROSS_DRAFTS 1u

MSA_API msa_status_t msa_index_scores_k(const msa_ragged_paged_t *rp, const void *q_idx,
                                        const msa_index_k_t *k_idx, int32_t num_kv_heads,
                                        int32_t max_blocks, uint32_t flags, float *scores,
                                        int32_t *dev_err, struct CUstream_st *stream);
MSA_API msa_status_t msa_index_select_k(const msa_ragged_paged_t *rp, const void *q_idx,
                                        const msa_index_k_t *k_idx, int32_t num_kv_heads,
                                        int32_t max_blocks, int32_t top_k, int32_t init_blocks,
                                        int32_t local_blocks, uint32_t flags, float *scores,
                                        int32_t *block_ids, int32_t *num_selected,
                                        int32_t *counters, int32_t *dev_err,
                                        struct CUstream_st *stream);

/*
 * msa_sparse_attn_paged — stage 3 ([ferrox] positions_of_blocks: the selected blocks'
 * positions, ascending and causally clipped; "an ordinary masked pass over the positions
 * those blocks cover"; [msa] "Three attention routes").
 *
 *   For query head h (KV head g = h / (num_q_heads / num_kv_heads)) of row t at position p:
 *   P = positions of the blocks in block_ids[t, g, :num_selected[t, g]] that are <= p,
 *   out[t, h] = sum_{pos in P} softmax_pos(scale * q[t, h] . k[pos]) v[pos],
 *   FP32 accumulation, output rounded to BF16.
 *
 *   Route from rp->max_q_len: 1 -> decode (no causal mask needed: p = L_b - 1); 2..8 ->
 *   speculative decode (per-token causal mask); > 8 -> prefill (per-token causal mask).
 *   Speculative and prefill steps first build, in `workspace`, each query tile's union of its
 *   tokens' selected blocks with a per-token mask, so that a page is read once per tile.
 *   Decode / speculative work is a list of (sequence, query tile, KV head, selected block)
 *   entries cut into `num_splits` equal contiguous split-K partitions (0 = one per SM and at
 *   least 8 blocks per partition, a persistent launch); their partials live in `workspace` and
 *   this call also enqueues the combine that writes `out`.  With a single partition the
 *   attention kernel writes `out` itself and no combine is enqueued.  Prefill runs one CTA per
 *   (sequence, query tile, KV head) and ignores num_splits.
 *
 *   q            device bf16 [total_q, num_q_heads, 128]
 *   k_cache, v_cache  device [num_pages, num_kv_heads, 128 tokens, 128] of kv_dtype,
 *                16-byte aligned
 *   block_ids, num_selected  as produced by msa_select_blocks with width S
 *   max_blocks   an upper bound on nb(p) of every query (as for msa_index_scores)
 *   workspace    device, >= msa_attn_workspace_bytes(...) bytes, 256-byte aligned;
 *                may be NULL when that size is 0
 *   out          device bf16 [total_q, num_q_heads, 128] (output), 16-byte aligned.  On the
 *                decode and speculative routes `out` may be NULL: the call then leaves the
 *                split-K partials in `workspace` (see msa_attn_partials) and enqueues no
 *                combine.
 *   num_q_heads % num_kv_heads == 0; the group size num_q_heads / num_kv_heads <= 64.
 */
MSA_API msa_status_t msa_sparse_attn_paged(const msa_ragged_paged_t *rp, const void *q,
                                   const void *k_cache, const void *v_cache,
                                   msa_kv_dtype_t kv_dtype, const int32_t *block_ids,
                                   const int32_t *num_selected, int32_t S, int32_t num_q_heads,
                                   int32_t num_kv_heads, int32_t max_blocks, float scale,
                                   int32_t num_splits, void *workspace, size_t workspace_bytes,
                                   void *out, int32_t *dev_err, struct CUstream_st *stream);

/*
 * msa_select_sparse_attn_paged — stages 2 and 3 in one call: exactly msa_select_blocks
 * followed by msa_sparse_attn_paged with the same arguments ([ferrox] block_sparse_select,
 * positions_of_blocks; [msa] "Three attention routes"), with bit-identical block_ids and
 * num_selected and the same output.
 *
 * On the decode route (max_q_len == 1) with a GQA group of at most 16 the selection runs inside
 * the attention launch: each CTA of the persistent kernel first selects the rows of the items in
 * its share of the work, then streams them, so the selection needs no launch of its own.  On the
 * speculative route (tiles of at most 8 tokens) one launch selects every token's row and builds
 * each query tile's union plan, which msa_sparse_attn_paged would otherwise build in a launch of
 * its own.  On the prefill route it enqueues the two stages one after the other.
 *
 *   scores, top_k, init_blocks, local_blocks  as msa_select_blocks (S = init + local + top_k)
 *   block_ids, num_selected  device int32 [total_q, num_kv_heads, S] / [total_q, num_kv_heads]
 *                  (outputs, as msa_select_blocks writes them)
 *   the rest      as msa_sparse_attn_paged.
 *   Validation is that of both stages, all of it before anything is enqueued.
 */
MSA_API msa_status_t msa_select_sparse_attn_paged(
    const msa_ragged_paged_t *rp, const float *scores, int32_t top_k, int32_t init_blocks,
    int32_t local_blocks, const void *q, const void *k_cache, const void *v_cache,
    msa_kv_dtype_t kv_dtype, int32_t num_q_heads, int32_t num_kv_heads, int32_t max_blocks,
    float scale, int32_t num_splits, void *workspace, size_t workspace_bytes,
    int32_t *block_ids, int32_t *num_selected, void *out, int32_t *dev_err,
    struct CUstream_st *stream);

/*
 * msa_decode_step — one step of the path in one call: msa_index_scores_k (no flags), then
 * msa_select_sparse_attn_paged, with the same results (scores, block_ids, num_selected, out)
 * ([msa] "Three attention routes", [ferrox] block_sparse_select, positions_of_blocks).
 *
 * On the decode route with the selection inside the attention (max_q_len == 1, a GQA group of
 * at most 16), the attention launch does not wait for the whole indexer launch: the last CTA of
 * each (sequence, index-K head) unit of the indexer publishes a flag once the unit's scores are
 * written, and each attention CTA selects a row as soon as its unit's flag is up (a bounded
 * wait), so the CTAs that start while the indexer's last units are still running begin early.
 * On the other routes the two calls run one after the other.
 *
 *   q_idx, index_k, scores  as msa_index_scores_k (scores: output)
 *   top_k .. out, dev_err, stream  as msa_select_sparse_attn_paged
 *   workspace    device, >= msa_decode_step_workspace_bytes(...) bytes, 256-byte aligned.  Its
 *                first msa_decode_step_workspace_bytes(...) - msa_attn_workspace_bytes(...)
 *                bytes hold the step's flags and counters: zero them once before the first
 *                call (every call leaves them ready for the next one) and again after a call
 *                that reports a device error.  Calls sharing one workspace run on one stream.
 */
MSA_API size_t msa_decode_step_workspace_bytes(const msa_ragged_paged_t *rp, int32_t S,
                                               int32_t num_q_heads, int32_t num_kv_heads,
                                               int32_t num_idx_k_heads, int32_t max_blocks,
                                               int32_t num_splits);
MSA_API msa_status_t msa_decode_step(const msa_ragged_paged_t *rp, const void *q_idx,
                                     const msa_index_k_t *index_k, int32_t top_k,
                                     int32_t init_blocks, int32_t local_blocks, const void *q,
                                     const void *k_cache, const void *v_cache,
                                     msa_kv_dtype_t kv_dtype, int32_t num_q_heads,
                                     int32_t num_kv_heads, int32_t max_blocks, float scale,
                                     int32_t num_splits, void *workspace, size_t workspace_bytes,
                                     float *scores, int32_t *block_ids, int32_t *num_selected,
                                     void *out, int32_t *dev_err, struct CUstream_st *stream);

/*
 * msa_sparse_attn_paged_noalloc — msa_sparse_attn_paged for callers that cannot provide a
 * workspace.  (This entry point has no counterpart on the pages: it is a deployment aid.)
 *
 * Some callers cannot allocate device memory when they call in: a host runtime whose device
 * memory plan is fixed before it starts serving and has no allocator to call afterwards, or a
 * plugin interface that passes only an operation's inputs and outputs.  This entry point takes
 * the same arguments as msa_sparse_attn_paged minus `workspace` / `workspace_bytes`, and keeps
 * that scratch in a device array that is part of the library itself: MSA_NOALLOC_SCRATCH_BYTES
 * on every GPU the library is loaded on, held until the process exits.  It allocates nothing.
 *
 *   - `out` is required (MSA_ERR_INVALID_ARG when NULL): the split-K partials stay in the
 *     library's own array, which the caller cannot reach, so the combine always runs.
 *   - A shape whose msa_attn_workspace_bytes exceeds MSA_NOALLOC_SCRATCH_BYTES is rejected
 *     with MSA_ERR_UNSUPPORTED before anything is enqueued (use msa_sparse_attn_paged with a
 *     workspace of your own for it).
 *   - The first call on a device looks the array's device address up (with that device
 *     current) and keeps it for that device's current context; a call in a new context (after
 *     cudaDeviceReset, for instance) looks it up again.  Make the first call on each device,
 *     and the first after a reset, before any stream capture.
 *   - Every call on a device shares the one array and it keeps the last call's contents
 *     (nothing in it needs to start at zero).  Calls whose work overlaps on the GPU race on
 *     it: run them on one stream, or order them.
 */
#define MSA_NOALLOC_SCRATCH_BYTES (32u << 20) /* 32 MiB */

MSA_API msa_status_t msa_sparse_attn_paged_noalloc(
    const msa_ragged_paged_t *rp, const void *q, const void *k_cache, const void *v_cache,
    msa_kv_dtype_t kv_dtype, const int32_t *block_ids, const int32_t *num_selected, int32_t S,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t max_blocks, float scale,
    int32_t num_splits, void *out, int32_t *dev_err, struct CUstream_st *stream);

/*
 * msa_splitk_combine — merge split-K partials ([msa] "Three attention routes": at more than
 * one partition the partials key on the ragged global query row and a combine writes the
 * ragged output).
 *
 *   out[t, h] = sum_s w_s o_s[t, h] / sum_s w_s,  w_s = exp(lse_s[t, h] - max_s lse_s[t, h]);
 *   partitions with lse = -inf (no position) weigh nothing; a row with none at all gets 0.
 *
 *   partial_o    device fp32 [num_splits, total_q, num_q_heads, 128]: each partition's
 *                softmax-normalised output over its own positions
 *   partial_lse  device fp32 [num_splits, total_q, num_q_heads]: natural log of each
 *                partition's sum of exp(scale * q . k)
 *   out          device bf16 [total_q, num_q_heads, 128] (output)
 */
MSA_API msa_status_t msa_splitk_combine(const float *partial_o, const float *partial_lse,
                                int32_t num_splits, int32_t total_q, int32_t num_q_heads,
                                void *out, struct CUstream_st *stream);

/*
 * msa_selftest_bounded_wait — a diagnostic (the pages have no counterpart): runs the bounded
 * pipeline wait that every pipelined kernel of this library uses on barriers that nothing ever
 * completes, so that its give-up path can be checked on a GPU without hanging it.
 *
 * One CTA: a first waiter gives up after `limit_us` microseconds, ORs MSA_DEVERR_TIMEOUT into
 * *dev_err and raises the CTA's abort flag; a second waiter (limit 4 x limit_us) leaves as soon
 * as it sees that flag; a last wait on a completed phase returns at once.  The kernel returns
 * normally and the context stays usable.
 *
 *   limit_us  1 .. 1000000
 *   dev_err   device int32 (nullable), as for the other entry points
 *   result    device uint32 [5], 4-byte aligned (output): [0] first waiter (1 = the phase
 *             completed, 2 = gave up), [1] its wait in microseconds, [2] / [3] the same for the
 *             second waiter, [4] the wait on the completed phase (1 = returned true)
 */
MSA_API msa_status_t msa_selftest_bounded_wait(uint32_t limit_us, int32_t *dev_err,
                                               uint32_t *result, struct CUstream_st *stream);

/*
 * msa_latent_sparse_attn_paged — latent sparse attention ([latent] Mojo
 * "Struct_latent_sparse_attention_ragged_paged": sparse attention over a shared K = V latent
 * read from two paged leaves, the sliding-window leaf by position range and the compressed
 * leaf by an explicit per-query entry list, with a per-head attention sink in the
 * denominator).
 *
 *   For query row t = input_row_offsets[b] + i at position p = swa->cache_lengths[b] + i and
 *   head h:  out[t, h] = sum_x e^(z_x) v_x / (e^(attn_sink[h]) + sum_x e^(z_x)),
 *   z_x = scale * q[t, h] . v_x, over the latent rows v_x of
 *     - the window leaf at positions max(0, p - window + 1) .. p (the new tokens' rows are
 *       already in that leaf), and
 *     - the compressed leaf at positions comp_indices[t, e] >= 0 (e < n_entries; -1 is
 *       padding, every listed entry counts); an entry >= comp->cache_lengths[b] sets
 *       MSA_DEVERR_BLOCK_ID and is skipped.
 *   Position x of leaf L for sequence b is row x % 128 of page L->lookup_table[b *
 *   L->max_pages_per_seq + x / 128], layer L->layer.  FP32 accumulation, BF16 output.
 *
 *   q            device bf16 [total_q, num_heads, 128], 16-byte aligned
 *   leaves       msa_latent_leaf_t (below); kv 16-byte aligned
 *   comp_indices device int32 [total_q, n_entries] (may be NULL when n_entries == 0)
 *   attn_sink    device f32 [num_heads]
 *   window >= 1; n_entries >= 0; scale > 0
 *   num_splits   0 = a count that fills the GPU (msa_latent_default_splits), else 1 .. 64:
 *                each query's list of rows (window, then entries) is cut into that many equal
 *                shares; with more than one the partials live in `workspace` (at least
 *                msa_latent_workspace_bytes bytes, 256-byte aligned) and a combine follows
 *   out          device bf16 [total_q, num_heads, 128], 16-byte aligned
 */
typedef struct {
    const void *kv;               /* device bf16 [num_pages, num_layers, 128 tokens, 128] */
    const int32_t *cache_lengths; /* device [batch]: window leaf: prior tokens; compressed
                                     leaf: its entries */
    const int32_t *lookup_table;  /* device [batch * max_pages_per_seq], -1 = no page */
    int32_t max_pages_per_seq;
    int32_t num_pages;
    int32_t num_layers;
    int32_t layer;                /* 0 .. num_layers - 1 */
} msa_latent_leaf_t;

MSA_API msa_status_t msa_latent_sparse_attn_paged(
    const int32_t *input_row_offsets, int32_t batch, int32_t total_q, int32_t max_q_len,
    const void *q, int32_t num_heads, const msa_latent_leaf_t *swa, int32_t window,
    const msa_latent_leaf_t *comp, const int32_t *comp_indices, int32_t n_entries,
    const float *attn_sink, float scale, int32_t num_splits, void *workspace,
    size_t workspace_bytes, void *out, int32_t *dev_err, struct CUstream_st *stream);

/* Host-only helpers (no device work, no CUDA call). */

/* Bytes of `workspace` msa_latent_sparse_attn_paged needs (0 for a single split). */
MSA_API size_t msa_latent_workspace_bytes(int32_t total_q, int32_t num_heads,
                                          int32_t num_splits);
/* The split count msa_latent_sparse_attn_paged uses when num_splits == 0: enough CTAs for two
 * per SM, at most one share per two 64-row tiles of the longest list and at most 64. */
MSA_API int32_t msa_latent_default_splits(int32_t total_q, int32_t num_heads, int32_t window,
                                          int32_t n_entries, int32_t num_sms);

/* Bytes of `workspace` that msa_sparse_attn_paged needs for this shape (0 when none). */
MSA_API size_t msa_attn_workspace_bytes(const msa_ragged_paged_t *rp, int32_t S,
                                        int32_t num_q_heads, int32_t num_kv_heads,
                                        int32_t max_blocks, int32_t num_splits);

/* The split-K partition count the decode / speculative routes use when num_splits == 0 for
 * `batch` sequences of `max_q_len` new tokens: one partition per SM, fewer when the work list
 * (batch x num_kv_heads x S x max_q_len entries) has under 8 entries per SM; 1 for prefill. */
MSA_API int32_t msa_default_num_splits(int32_t batch, int32_t max_q_len, int32_t num_kv_heads,
                               int32_t S, int32_t num_sms);

/* Where msa_sparse_attn_paged keeps its split-K partials in `workspace` for this shape:
 * returns the number of split indices (the num_splits argument msa_splitk_combine takes) and
 * stores the byte offsets of partial_o [n, total_q, H_q, 128] and partial_lse [n, total_q,
 * H_q] (both fp32); returns 0 when the route writes `out` directly (prefill) or on invalid
 * arguments.  The offsets may be NULL. */
MSA_API int32_t msa_attn_partials(const msa_ragged_paged_t *rp, int32_t S, int32_t num_q_heads,
                                  int32_t num_kv_heads, int32_t max_blocks, int32_t num_splits,
                                  size_t *partial_o_offset, size_t *partial_lse_offset);

/* A static, human-readable name of a status code. */
MSA_API const char *msa_status_string(msa_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */
