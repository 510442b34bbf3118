/*
 * CPU oracle for MiniMax-M3 block-sparse attention (MSA) over a paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  The parity tests, the smoke check and the benchmark's
 * CPU-baseline / reference arm are the only callers.  Nothing on the GPU product path
 * links, loads or calls this file, and this file includes nothing from that path.
 *
 * It is the method's definition written out as plain loops with fp64 arithmetic:
 * no tiling, no fusion, no reordering beyond what the definition states.
 *
 * Sources (page title, section):
 *   [msa]     Mojo module "msa" (Graph-op bindings for the MiniMax-M3 block-sparse
 *             attention kernels): module summary (BF16, head_dim 128, page 128 == block,
 *             single index-K head, scale-free FP8 e4m3 main KV, FP32 accumulation) and the
 *             "Three attention routes" list (query position = cache_lengths[batch] +
 *             tok_in_seq; logical KV start of a selected block = block id * BN).
 *   [trtllm]  TensorRT-LLM "DeepSeekSparseAttentionConfig", field indexer_k_dtype (the
 *             scaled FP8 / FP4 index-K formats; below, before stage 1).
 *   [ferrox]  ferrox-core "Module block_sparse": "Four rules" (max over the block, no
 *             softmax scale, per-KV-head selection, forced init/local blocks),
 *             "The block size is an ABI", and the functions block_sparse_select
 *             (ascending) and positions_of_blocks (ascending, causally clipped).
 *
 * Readings where the pages are silent (each one also listed in the design notes):
 *   - top_k counts only the non-forced candidates; the selection is forced ∪ top_k(rest).
 *   - equal scores: the lower block id wins.
 *   - a query's position is p = cache_lengths[b] + i; the new tokens' k / v / k_idx rows
 *     already sit in the cache at [cache_lengths[b], cache_lengths[b] + q_len_b).
 *   - "newest local_blocks" is relative to the query's own position: blocks
 *     nb(p)-local .. nb(p)-1 with nb(p) = p/128 + 1.
 *   - a block's score takes only the positions <= p; blocks with none score -inf.
 *   - GQA: query head h reads KV head g = h / (H_q / H_kv); index-query head g reads
 *     index-K head g % H_idxk.
 *
 * Memory layouts (the same host bytes the GPU path consumes):
 *   q        bf16 bits  [total_q][H_q][128]
 *   q_idx    bf16 bits  [total_q][H_kv][128]
 *   k_idx    bf16 bits  [num_pages][H_idxk][128 tokens][128], or
 *            fp8: e4m3 bytes [num_pages][H_idxk][128 tokens][128] + f32 [..][128 tokens],
 *            fp4: e2m1 pairs [num_pages][H_idxk][128 tokens][64] + ue8m0 [..][128 tokens][4]
 *   k, v     bf16 bits or e4m3 bytes [num_pages][H_kv][128 tokens][128]
 *   table    int32      [batch][max_pages]  (logical block j of sequence b -> page)
 *   scores   fp64       [total_q][H_kv][max_blocks]
 *   ids      int32      [total_q][H_kv][S] ascending, padded with -1; counts [total_q][H_kv]
 *   out      fp64       [total_q][H_q][128]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_BLOCK 128 /* [ferrox] "The block size is an ABI": block = page = 128 tokens */
#define ORC_D 128     /* [msa] module summary: head_dim 128 */

/* bf16 -> value: the bf16 bits are the top half of an IEEE binary32. */
double orc_bf16_value(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* e4m3 ("fn" variant: bias 7, no infinities, S.1111.111 is NaN) -> value. */
double orc_e4m3_value(uint8_t x)
{
    int sign = x >> 7;
    int e = (x >> 3) & 15;
    int m = x & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6); /* subnormal: 0.m * 2^(1-7) */
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* ---------------------------------------------------------------------------------------
 * Scaled index-K formats: TensorRT-LLM "DeepSeekSparseAttentionConfig", field
 * indexer_k_dtype.  fp8: one E4M3 byte per element and one float32 scale for the token's 128
 * elements (132 B per token); fp4: two E2M1 codes per byte and one UE8M0 exponent per 32
 * elements (68 B per token).  Readings where the page is silent: element c of a token's fp4
 * codes is in byte c / 2, in the low nibble when c is even; the exponent byte x stands for
 * 2^(x - 127); an element's value is its code's value times its scale.
 * ------------------------------------------------------------------------------------- */

/* E2M1 (1 sign bit, 2 exponent bits with bias 1, 1 mantissa bit; no inf, no NaN) -> value. */
double orc_e2m1_value(uint8_t code)
{
    int sign = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double v = (e == 0) ? 0.5 * m                          /* subnormal: 0.m * 2^(1-1) */
                        : ldexp(1.0 + 0.5 * m, e - 1);     /* 1.m * 2^(e-1) */
    return sign ? -v : v;
}

/* UE8M0 (8 exponent bits, bias 127, no sign, no mantissa; 0xFF is NaN) -> value. */
double orc_ue8m0_value(uint8_t x)
{
    if (x == 0xFF)
        return NAN;
    return ldexp(1.0, (int)x - 127);
}

#define ORC_IDX_BF16 0
#define ORC_IDX_FP8 1
#define ORC_IDX_FP4 2

/* Element c of index-K row r (r = (page * H_idxk + head) * 128 + token) in format fmt:
 * bf16 codes [rows][128] u16; fp8 codes [rows][128] u8 with scales [rows] f32; fp4 codes
 * [rows][64] u8 with exponents [rows][4] u8. */
static double idx_k_value(int fmt, const void *codes, const void *scales, size_t r, int c)
{
    if (fmt == ORC_IDX_FP8) {
        float s;
        memcpy(&s, (const uint8_t *)scales + r * sizeof(float), sizeof s);
        return orc_e4m3_value(((const uint8_t *)codes)[r * ORC_D + c]) * (double)s;
    }
    if (fmt == ORC_IDX_FP4) {
        uint8_t byte = ((const uint8_t *)codes)[r * (ORC_D / 2) + c / 2];
        uint8_t code = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
        uint8_t e = ((const uint8_t *)scales)[r * (ORC_D / 32) + c / 32];
        return orc_e2m1_value(code) * orc_ue8m0_value(e);
    }
    return orc_bf16_value(((const uint16_t *)codes)[r * ORC_D + c]);
}

/* Query position of row i of sequence b: [msa] "Three attention routes",
 * speculative route: position = cache_lengths[batch] + tok_in_seq. */
static int query_position(const int32_t *cache_len, int b, int i) { return cache_len[b] + i; }

/* Blocks visible to a query at position p: those whose first position is <= p. */
static int visible_blocks(int p) { return p / ORC_BLOCK + 1; }

/* ---------------------------------------------------------------------------------------
 * Stage 1: block scores.  [ferrox] "Four rules": a block's score is the MAX over its
 * positions of the raw dot product q_idx . k_idx, with no softmax scale; one index head
 * scores for one KV head.
 * ------------------------------------------------------------------------------------- */
void orc_index_scores(int batch, const int32_t *row_off, const int32_t *cache_len,
                      const int32_t *table, int max_pages, const uint16_t *q_idx,
                      int k_idx_fmt, const void *k_idx, const void *k_idx_scale, int H_kv,
                      int H_idxk, int max_blocks, double *scores)
{
    for (int b = 0; b < batch; ++b) {
        int q_len = row_off[b + 1] - row_off[b];
#pragma omp parallel for collapse(2) schedule(dynamic)
        for (int i = 0; i < q_len; ++i) {
            for (int g = 0; g < H_kv; ++g) {
                int t = row_off[b] + i;
                int p = query_position(cache_len, b, i);
                int nb = visible_blocks(p);
                int hk = g % H_idxk;
                const uint16_t *qv = q_idx + ((size_t)t * H_kv + g) * ORC_D;
                double *srow = scores + ((size_t)t * H_kv + g) * max_blocks;
                for (int j = 0; j < max_blocks; ++j) {
                    double best = -INFINITY;
                    if (j < nb) {
                        int page = table[(size_t)b * max_pages + j];
                        int last = j * ORC_BLOCK + ORC_BLOCK - 1;
                        if (last > p)
                            last = p;
                        for (int pos = j * ORC_BLOCK; pos <= last; ++pos) {
                            int tok = pos - j * ORC_BLOCK;
                            size_t r = ((size_t)page * H_idxk + hk) * ORC_BLOCK + (size_t)tok;
                            double dot = 0.0;
                            for (int c = 0; c < ORC_D; ++c)
                                dot += orc_bf16_value(qv[c]) *
                                       idx_k_value(k_idx_fmt, k_idx, k_idx_scale, r, c);
                            if (dot > best)
                                best = dot;
                        }
                    }
                    srow[j] = best;
                }
            }
        }
    }
}

/* ---------------------------------------------------------------------------------------
 * Stage 2: selection.  [ferrox] "Four rules": the first init_blocks and the newest
 * local_blocks are force-included; block_sparse_select returns the blocks ascending.
 * The rest is the top_k of the remaining blocks by score (ties: lower id first).
 * ------------------------------------------------------------------------------------- */
typedef struct {
    double score;
    int id;
} orc_cand;

static int cand_order(const void *a, const void *b)
{
    const orc_cand *x = (const orc_cand *)a, *y = (const orc_cand *)b;
    if (x->score > y->score)
        return -1;
    if (x->score < y->score)
        return 1;
    return (x->id < y->id) ? -1 : (x->id > y->id);
}

void orc_select_blocks(int batch, const int32_t *row_off, const int32_t *cache_len, int H_kv,
                       int max_blocks, const double *scores, int top_k, int init_blocks,
                       int local_blocks, int S, int32_t *ids, int32_t *counts)
{
    for (int b = 0; b < batch; ++b) {
        int q_len = row_off[b + 1] - row_off[b];
        for (int i = 0; i < q_len; ++i) {
            int t = row_off[b] + i;
            int nb = visible_blocks(query_position(cache_len, b, i));
            for (int g = 0; g < H_kv; ++g) {
                const double *srow = scores + ((size_t)t * H_kv + g) * max_blocks;
                char *chosen = (char *)calloc((size_t)nb, 1);
                orc_cand *cand = (orc_cand *)malloc(sizeof(orc_cand) * (size_t)nb);
                int nc = 0;
                for (int j = 0; j < nb; ++j) {
                    int forced = (j < init_blocks) || (j >= nb - local_blocks);
                    if (forced)
                        chosen[j] = 1;
                    else {
                        cand[nc].score = srow[j];
                        cand[nc].id = j;
                        ++nc;
                    }
                }
                qsort(cand, (size_t)nc, sizeof(orc_cand), cand_order);
                for (int r = 0; r < nc && r < top_k; ++r)
                    chosen[cand[r].id] = 1;
                int32_t *out = ids + ((size_t)t * H_kv + g) * S;
                int n = 0;
                for (int j = 0; j < nb; ++j)
                    if (chosen[j])
                        out[n++] = j;
                counts[(size_t)t * H_kv + g] = n;
                for (int r = n; r < S; ++r)
                    out[r] = -1;
                free(chosen);
                free(cand);
            }
        }
    }
}

/* ---------------------------------------------------------------------------------------
 * Stage 2 with the indexer top-k shared across draft tokens: TensorRT-LLM
 * "DeepSeekSparseAttentionConfig", field index_share_for_mtp_iteration ("reuse the indexer
 * Top-K across MTP draft steps instead of recomputing it each step").  Reading: the top-k is
 * computed once per (sequence, KV head), for the sequence's first new token, over that
 * token's candidates (its visible blocks minus its own forced blocks), from that token's
 * scores; every new token of the sequence then selects its own forced blocks ([ferrox] "Four
 * rules") together with that shared top-k, ascending.  The shared blocks lie below the first
 * token's position, so every later token of the sequence can see them.
 * ------------------------------------------------------------------------------------- */
void orc_select_blocks_shared(int batch, const int32_t *row_off, const int32_t *cache_len,
                              int H_kv, int max_blocks, const double *scores, int top_k,
                              int init_blocks, int local_blocks, int S, int32_t *ids,
                              int32_t *counts)
{
    for (int b = 0; b < batch; ++b) {
        int q_len = row_off[b + 1] - row_off[b];
        if (q_len <= 0)
            continue;
        int t0 = row_off[b];
        int nb0 = visible_blocks(query_position(cache_len, b, 0));
        int nb_last = visible_blocks(query_position(cache_len, b, q_len - 1));
        for (int g = 0; g < H_kv; ++g) {
            /* the shared top-k: the first token's candidates by its own scores */
            const double *srow = scores + ((size_t)t0 * H_kv + g) * max_blocks;
            char *shared = (char *)calloc((size_t)nb_last, 1);
            orc_cand *cand = (orc_cand *)malloc(sizeof(orc_cand) * (size_t)nb0);
            int nc = 0;
            for (int j = 0; j < nb0; ++j) {
                int forced0 = (j < init_blocks) || (j >= nb0 - local_blocks);
                if (!forced0) {
                    cand[nc].score = srow[j];
                    cand[nc].id = j;
                    ++nc;
                }
            }
            qsort(cand, (size_t)nc, sizeof(orc_cand), cand_order);
            for (int r = 0; r < nc && r < top_k; ++r)
                shared[cand[r].id] = 1;
            /* every token: its own forced blocks and the shared top-k */
            for (int i = 0; i < q_len; ++i) {
                int t = row_off[b] + i;
                int nb = visible_blocks(query_position(cache_len, b, i));
                int32_t *out = ids + ((size_t)t * H_kv + g) * S;
                int n = 0;
                for (int j = 0; j < nb; ++j) {
                    int forced = (j < init_blocks) || (j >= nb - local_blocks);
                    if (forced || shared[j])
                        out[n++] = j;
                }
                counts[(size_t)t * H_kv + g] = n;
                for (int r = n; r < S; ++r)
                    out[r] = -1;
            }
            free(shared);
            free(cand);
        }
    }
}

/* ---------------------------------------------------------------------------------------
 * Stage 3: attention over the positions the selected blocks cover, ascending and causally
 * clipped ([ferrox] positions_of_blocks), with softmax(scale * q . k) in fp64 ("an
 * ordinary masked pass over the positions those blocks cover").
 * ------------------------------------------------------------------------------------- */
static double kv_value(const void *cache, int fp8, size_t idx)
{
    if (fp8)
        return orc_e4m3_value(((const uint8_t *)cache)[idx]);
    return orc_bf16_value(((const uint16_t *)cache)[idx]);
}

void orc_attention(int batch, const int32_t *row_off, const int32_t *cache_len,
                   const int32_t *table, int max_pages, const uint16_t *q, const void *k_cache,
                   const void *v_cache, int kv_fp8, int H_q, int H_kv, const int32_t *ids,
                   const int32_t *counts, int S, double scale, double *out)
{
    int G = H_q / H_kv;
    for (int b = 0; b < batch; ++b) {
        int q_len = row_off[b + 1] - row_off[b];
#pragma omp parallel for collapse(2) schedule(dynamic)
        for (int i = 0; i < q_len; ++i) {
            for (int h = 0; h < H_q; ++h) {
                int t = row_off[b] + i;
                int p = query_position(cache_len, b, i);
                int g = h / G;
                const int32_t *sel = ids + ((size_t)t * H_kv + g) * S;
                int nsel = counts[(size_t)t * H_kv + g];
                const uint16_t *qv = q + ((size_t)t * H_q + h) * ORC_D;
                /* positions_of_blocks: every position of every selected block, <= p */
                int cap = nsel * ORC_BLOCK;
                double *z = (double *)malloc(sizeof(double) * (size_t)(cap > 0 ? cap : 1));
                size_t *row = (size_t *)malloc(sizeof(size_t) * (size_t)(cap > 0 ? cap : 1));
                int np = 0;
                for (int s = 0; s < nsel; ++s) {
                    int j = sel[s];
                    int page = table[(size_t)b * max_pages + j];
                    for (int pos = j * ORC_BLOCK; pos < (j + 1) * ORC_BLOCK && pos <= p; ++pos) {
                        size_t r = ((size_t)page * H_kv + g) * ORC_BLOCK + (size_t)(pos - j * ORC_BLOCK);
                        double dot = 0.0;
                        for (int c = 0; c < ORC_D; ++c)
                            dot += orc_bf16_value(qv[c]) * kv_value(k_cache, kv_fp8, r * ORC_D + c);
                        z[np] = scale * dot;
                        row[np] = r;
                        ++np;
                    }
                }
                double m = -INFINITY;
                for (int x = 0; x < np; ++x)
                    if (z[x] > m)
                        m = z[x];
                double l = 0.0;
                double acc[ORC_D];
                for (int c = 0; c < ORC_D; ++c)
                    acc[c] = 0.0;
                for (int x = 0; x < np; ++x) {
                    double w = exp(z[x] - m);
                    l += w;
                    for (int c = 0; c < ORC_D; ++c)
                        acc[c] += w * kv_value(v_cache, kv_fp8, row[x] * ORC_D + c);
                }
                double *o = out + ((size_t)t * H_q + h) * ORC_D;
                for (int c = 0; c < ORC_D; ++c)
                    o[c] = (np > 0) ? acc[c] / l : NAN; /* softmax over nothing: NaN */
                free(z);
                free(row);
            }
        }
    }
}

/* ---------------------------------------------------------------------------------------
 * Latent sparse attention: Mojo "Struct_latent_sparse_attention_ragged_paged" (the
 * mo.latent_sparse_attention.ragged.paged op): sparse attention over a K = V latent shared by
 * all query heads, read from two paged leaves, the sliding-window leaf by position range and
 * the compressed leaf by an explicit per-query entry list, with a per-head attention sink in
 * the softmax denominator.
 *
 * Readings where the page gives only the op's arguments:
 *   - the latent is 128 wide, both leaves are paged like the main cache (128 tokens a page,
 *     page(b, pos) = table[b][pos / 128]) with a layer axis: [pages][layers][128][128] bf16,
 *     and `layer` picks the layer;
 *   - the window of the query at position p = swa_cache_lengths[b] + i is the `window`
 *     positions ending at p (inclusive), clipped at 0; the new tokens are already in that leaf;
 *   - comp_indices [total_q][n_entries] lists logical positions of the sequence's compressed
 *     leaf; -1 is padding; every listed entry counts (as listed);
 *   - the sink of head h adds exp(sink[h]) to the denominator (natural-log domain, not scaled)
 *     and contributes no value:
 *       out = sum_x e^(z_x) v_x / (e^(sink) + sum_x e^(z_x)),  z_x = scale * q . v_x.
 * ------------------------------------------------------------------------------------- */
void orc_latent_attention(int batch, const int32_t *row_off, const uint16_t *q, int H,
                          int window, const uint16_t *swa_kv, int swa_layers, int swa_layer,
                          const int32_t *swa_len, const int32_t *swa_table, int swa_max_pages,
                          const uint16_t *comp_kv, int comp_layers, int comp_layer,
                          const int32_t *comp_table, int comp_max_pages,
                          const int32_t *comp_idx, int n_entries, const float *sink,
                          double scale, double *out)
{
    for (int b = 0; b < batch; ++b) {
        int q_len = row_off[b + 1] - row_off[b];
#pragma omp parallel for collapse(2) schedule(dynamic)
        for (int i = 0; i < q_len; ++i) {
            for (int h = 0; h < H; ++h) {
                int t = row_off[b] + i;
                int p = swa_len[b] + i;
                int w0 = p - window + 1;
                if (w0 < 0)
                    w0 = 0;
                int n = (p - w0 + 1) + n_entries;
                const uint16_t **rows = (const uint16_t **)malloc(sizeof(*rows) * (size_t)n);
                int np = 0;
                for (int pos = w0; pos <= p; ++pos) {
                    int page = swa_table[(size_t)b * swa_max_pages + pos / ORC_BLOCK];
                    rows[np++] = swa_kv + (((size_t)page * swa_layers + swa_layer) * ORC_BLOCK +
                                           (size_t)(pos % ORC_BLOCK)) * ORC_D;
                }
                for (int e = 0; e < n_entries; ++e) {
                    int pos = comp_idx[(size_t)t * n_entries + e];
                    if (pos < 0)
                        continue;
                    int page = comp_table[(size_t)b * comp_max_pages + pos / ORC_BLOCK];
                    rows[np++] = comp_kv + (((size_t)page * comp_layers + comp_layer) *
                                                ORC_BLOCK + (size_t)(pos % ORC_BLOCK)) * ORC_D;
                }
                const uint16_t *qv = q + ((size_t)t * H + h) * ORC_D;
                double *z = (double *)malloc(sizeof(double) * (size_t)(np > 0 ? np : 1));
                double m = (double)sink[h];
                for (int x = 0; x < np; ++x) {
                    double dot = 0.0;
                    for (int c = 0; c < ORC_D; ++c)
                        dot += orc_bf16_value(qv[c]) * orc_bf16_value(rows[x][c]);
                    z[x] = scale * dot;
                    if (z[x] > m)
                        m = z[x];
                }
                double l = exp((double)sink[h] - m); /* the sink: denominator only */
                double acc[ORC_D];
                for (int c = 0; c < ORC_D; ++c)
                    acc[c] = 0.0;
                for (int x = 0; x < np; ++x) {
                    double w = exp(z[x] - m);
                    l += w;
                    for (int c = 0; c < ORC_D; ++c)
                        acc[c] += w * orc_bf16_value(rows[x][c]);
                }
                double *o = out + ((size_t)t * H + h) * ORC_D;
                for (int c = 0; c < ORC_D; ++c)
                    o[c] = acc[c] / l;
                free(z);
                free(rows);
            }
        }
    }
}
