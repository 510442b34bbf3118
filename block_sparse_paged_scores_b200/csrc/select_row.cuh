// select_row.cuh — the selection of one (query row, KV head), done by one warp.
//
// ferrox-core "Module block_sparse": the first init_blocks and the newest local_blocks are
// force-included before any scoring (that is what keeps the selection non-empty), and
// block_sparse_select returns the blocks each KV head may read, ascending.  The remaining
// blocks compete on score; equal scores go to the lower block id.
//
// The candidates' scores become order-preserving uint32 keys held in registers; the exact
// top_k-th largest key is then built bit by bit from the top (32 rounds of "how many keys are
// >= this prefix", one warp reduction each, no atomics).  One ascending pass over the block ids
// keeps the forced blocks, every candidate above that threshold, and the lowest-id candidates
// equal to it until top_k are taken, so the output comes out in ascending order with no sort.
//
// Used by the selection kernel (select.cu) and by the decode indexer's last CTA of each
// (sequence, tile, index head) (indexer.cu), which reads scores other CTAs wrote in the same
// launch and so loads them from L2 (CG = true).
#pragma once

#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace msa {

template <bool CG>
__device__ __forceinline__ float load_score(const float *p) {
  if (CG) return __ldcg(p);
  return *p;
}

// Keys of the candidate blocks (0 for blocks that are not candidates: every real key is at
// least score_key(-inf) = 0x007fffff > 0).  KPL keys per lane stay in registers; KPL == 0
// reads them from memory on every pass (any number of blocks).
template <int KPL, bool CG>
struct SelKeys {
  uint32_t k[KPL > 0 ? KPL : 1];
  __device__ __forceinline__ void load(const float *srow, int nb, int lane, int init_e,
                                       int local_lo) {
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
      const int j = i * 32 + lane;
      k[i] = (j < nb && j >= init_e && j < local_lo) ? score_key(load_score<CG>(srow + j)) : 0u;
    }
  }
  // number of candidate keys >= x (over the warp); four independent partial counts
  __device__ __forceinline__ uint32_t count_ge(uint32_t x, const float *srow, int lane,
                                               int init_e, int local_lo) const {
    uint32_t c = 0;
    if (KPL > 0) {
      uint32_t c4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int i = 0; i < KPL; ++i) c4[i & 3] += k[i] >= x;
      c = (c4[0] + c4[1]) + (c4[2] + c4[3]);
    } else {
      for (int j = init_e + lane; j < local_lo; j += 32)
        c += score_key(load_score<CG>(srow + j)) >= x;
    }
    return __reduce_add_sync(0xffffffffu, c);
  }
  // largest and smallest candidate key over the warp
  __device__ __forceinline__ void range(const float *srow, int lane, int init_e, int local_lo,
                                        uint32_t &kmax, uint32_t &kmin) const {
    uint32_t hi = 0u, lo = 0xffffffffu;
    if (KPL > 0) {
#pragma unroll
      for (int i = 0; i < KPL; ++i) {
        hi = max(hi, k[i]);
        if (k[i] != 0u) lo = min(lo, k[i]);
      }
    } else {
      for (int j = init_e + lane; j < local_lo; j += 32) {
        const uint32_t key = score_key(load_score<CG>(srow + j));
        hi = max(hi, key);
        lo = min(lo, key);
      }
    }
    kmax = __reduce_max_sync(0xffffffffu, hi);
    kmin = __reduce_min_sync(0xffffffffu, lo);
  }
};

// One warp selects for one (row, KV head): srow = its nb visible scores (nb >= 1), out = its S
// id slots; returns the number selected (lane-uniform).  S >= init + local + top_k.
//
// nb_out > nb (the indexer top-k shared across a sequence's draft tokens: TensorRT-LLM
// "DeepSeekSparseAttentionConfig", index_share_for_mtp_iteration): srow and nb are the first
// draft token's, whose candidates and top-k they give; the output is for a later token that
// sees nb_out blocks: its own forced blocks of [0, nb_out) together with that top-k.
template <int KPL, bool CG>
__device__ __forceinline__ int select_row(const float *srow, int nb, int top_k, int init_blocks,
                                          int local_blocks, int S, int32_t *out,
                                          int32_t *dev_err, int lane, int nb_out = 0) {
  const unsigned lt_mask = (1u << lane) - 1u;
  if (nb_out < nb) nb_out = nb;
  // forced: [0, init_e) and [local_lo, nb); candidates: [init_e, local_lo)
  const int init_e = min(init_blocks, nb);
  const int local_lo = max(init_e, nb - local_blocks);
  const int n_cand = local_lo - init_e;
  const bool take_all = n_cand <= top_k;
  // the output row's own forced blocks: [0, init_o) and [local_o, nb_out)
  const int init_o = min(init_blocks, nb_out);
  const int local_o = max(init_o, nb_out - local_blocks);

  SelKeys<KPL, CG> keys;
  uint32_t T = 0xffffffffu;  // top_k == 0: no candidate passes
  int need_eq = 0;
  if (!take_all && top_k > 0) {
    keys.load(srow, nb, lane, init_e, local_lo);
    // T = the top_k-th largest candidate key: the largest x with count(key >= x) >= top_k,
    // built one bit at a time from the top.  Every candidate key lies in [kmin, kmax], so T
    // shares their common leading bits and only the bits below can still be open.
    const uint32_t k = static_cast<uint32_t>(top_k);
    uint32_t kmax, kmin;
    keys.range(srow, lane, init_e, local_lo, kmax, kmin);
    const uint32_t diff = kmax ^ kmin;
    const int top = diff == 0u ? -1 : 31 - __clz(diff);  // highest bit where they differ
    T = top < 0 ? kmax : (kmax & ~((2u << top) - 1u));
    for (int bit = top; bit >= 0; --bit) {
      const uint32_t x = T | (1u << bit);
      if (keys.count_ge(x, srow, lane, init_e, local_lo) >= k) T = x;
    }
    const uint32_t above =
        T == 0xffffffffu ? 0u : keys.count_ge(T + 1u, srow, lane, init_e, local_lo);
    need_eq = static_cast<int>(k - above);  // how many candidates equal to T are taken
  }

  // one ascending pass: forced, above T, and the lowest-id candidates equal to T
  int nsel = 0, eq_seen = 0;
  auto pass = [&](int i, uint32_t key_reg) {
    const int j = i * 32 + lane;
    const bool cand = j < nb && j >= init_e && j < local_lo;
    const bool forced = j < nb_out && (j < init_o || j >= local_o);
    bool take;
    if (take_all) {
      take = forced || cand;
    } else {
      const uint32_t key =
          KPL > 0 ? key_reg : (cand ? score_key(load_score<CG>(srow + j)) : 0u);
      const bool eq = cand && key == T;
      const unsigned eqm = __ballot_sync(0xffffffffu, eq);
      const int eq_rank = eq_seen + __popc(eqm & lt_mask);
      take = forced || (cand && key > T) || (eq && eq_rank < need_eq);
      eq_seen += __popc(eqm);
    }
    const unsigned tm = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int pos = nsel + __popc(tm & lt_mask);
      if (pos < S) out[pos] = j;
    }
    nsel += __popc(tm);
  };
  const int passes = (nb_out + 31) / 32;
  if (KPL > 0) {
#pragma unroll
    for (int i = 0; i < (KPL > 0 ? KPL : 1); ++i)
      if (i < passes) pass(i, keys.k[i]);
  } else {
    for (int i = 0; i < passes; ++i) pass(i, 0u);
  }
  if (nsel > S) {  // cannot happen when S >= init + local + top_k
    if (lane == 0) report(dev_err, MSA_DEVERR_NUM_SELECTED);
    nsel = S;
  }
  for (int q = nsel + lane; q < S; q += 32) out[q] = -1;
  return nsel;
}

}  // namespace msa
