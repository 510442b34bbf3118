// select_row.cuh — the selection of one (query row, KV head), done by one warp.
//
// ferrox-core "Module block_sparse": the first init_blocks and the newest local_blocks are
// force-included before any scoring (that is what keeps the selection non-empty), and
// block_sparse_select returns the blocks each KV head may read, ascending.  The remaining
// blocks compete on score; equal scores go to the lower block id.
//
// The candidates' scores become order-preserving uint32 keys held in registers; the exact
// top_k-th largest key is then built from the top, two bits a round (at most 16 rounds of "how
// many keys are >= each of three prefixes", three warp reductions in flight, no atomics).  The
// search stops early when a prefix has exactly top_k keys at or above it: those keys are then
// the top_k, whatever the lower bits (with continuous scores this happens once the prefix
// separates the top_k-th key from the next one, after about half the bits).  One ascending pass
// over the block ids keeps the forced blocks, every candidate above the threshold, and the
// lowest-id candidates equal to it until top_k are taken, so the output comes out in ascending
// order with no sort.
//
// Used by the selection kernel (select.cu), by the speculative selection-and-plan kernel
// (select_plan.cu), by the decode attention's prologue (attention_stream.cu, which hands it the
// scores it loaded already: select_row_from), and by the decode indexer's last CTA of each
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
  // score(i): the score of block 32 i + lane
  template <typename Score>
  __device__ __forceinline__ void load(Score score, int nb, int lane, int init_e, int local_lo) {
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
      const int j = i * 32 + lane;
      k[i] = (j < nb && j >= init_e && j < local_lo) ? score_key(score(i)) : 0u;
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
  // numbers of candidate keys >= x1, >= x2 and >= x3 (three reductions in flight at once)
  __device__ __forceinline__ void count_ge3(uint32_t x1, uint32_t x2, uint32_t x3,
                                            const float *srow, int lane, int init_e,
                                            int local_lo, uint32_t &c1, uint32_t &c2,
                                            uint32_t &c3) const {
    uint32_t a1 = 0, a2 = 0, a3 = 0;
    if (KPL > 0) {
#pragma unroll
      for (int i = 0; i < KPL; ++i) {
        a1 += k[i] >= x1;
        a2 += k[i] >= x2;
        a3 += k[i] >= x3;
      }
    } else {
      for (int j = init_e + lane; j < local_lo; j += 32) {
        const uint32_t key = score_key(load_score<CG>(srow + j));
        a1 += key >= x1;
        a2 += key >= x2;
        a3 += key >= x3;
      }
    }
    c1 = __reduce_add_sync(0xffffffffu, a1);
    c2 = __reduce_add_sync(0xffffffffu, a2);
    c3 = __reduce_add_sync(0xffffffffu, a3);
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
//
// For callers that keep more per selected block, emit is told of each one in one of two ways:
// emit.taken(pos, j, i) by the lane that takes block j = 32 i + lane as the pos-th selected
// block; or emit.gathered(pos, j, i, src, valid), called by every lane of the warp together,
// where a valid lane writes the pos-th selected block j = 32 i + src (lane src holds it).
struct NoEmit {
  __device__ __forceinline__ void taken(int, int, int) const {}
  __device__ __forceinline__ void gathered(int, int, int, int, bool) const {}
};

// Position of the set bit of rank r (0: the lowest) in m (r < popc(m)).
__device__ __forceinline__ int nth_set_bit(uint32_t m, int r) {
  int b = 0;
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const int c = __popc(m & ((1u << w) - 1u));
    if (r >= c) {
      r -= c;
      m >>= w;
      b += w;
    }
  }
  return b;
}
//
// select_row_from takes the row's scores through score(i) (block 32 i + lane) when KPL > 0, for
// callers that loaded them already; select_row reads them from srow.
template <int KPL, bool CG, typename Emit, typename Score>
__device__ __forceinline__ int select_row_from(Score score, const float *srow, int nb, int top_k,
                                               int init_blocks, int local_blocks, int S,
                                               int32_t *out, int32_t *dev_err, int lane,
                                               int nb_out, Emit emit) {
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
    keys.load(score, nb, lane, init_e, local_lo);
    // T = the top_k-th largest candidate key: the largest x with count(key >= x) >= top_k,
    // built one bit at a time from the top.  Every candidate key lies in [kmin, kmax], so T
    // shares their common leading bits and only the bits below can still be open.
    const uint32_t k = static_cast<uint32_t>(top_k);
    uint32_t kmax, kmin;
    keys.range(srow, lane, init_e, local_lo, kmax, kmin);
    const uint32_t diff = kmax ^ kmin;
    const int top = diff == 0u ? -1 : 31 - __clz(diff);  // highest bit where they differ
    T = top < 0 ? kmax : (kmax & ~((2u << top) - 1u));
    bool exact = false;  // exactly top_k keys are >= T
    int bit = top;
    // two bits a round: the largest of the digits 1..3 whose prefix keeps >= top_k keys
    // (digit 0 keeps T, which has >= top_k keys by construction)
    for (; bit >= 1; bit -= 2) {
      const uint32_t x1 = T | (1u << (bit - 1)), x2 = T | (2u << (bit - 1)),
                     x3 = T | (3u << (bit - 1));
      uint32_t c1, c2, c3;
      keys.count_ge3(x1, x2, x3, srow, lane, init_e, local_lo, c1, c2, c3);
      const uint32_t c = c3 >= k ? c3 : (c2 >= k ? c2 : c1);
      if (c >= k) {
        T = c3 >= k ? x3 : (c2 >= k ? x2 : x1);
        if (c == k) {
          exact = true;
          break;
        }
      }
    }
    if (!exact && bit == 0) {  // the last bit on its own
      const uint32_t x = T | 1u;
      const uint32_t c = keys.count_ge(x, srow, lane, init_e, local_lo);
      if (c >= k) {
        T = x;
        exact = c == k;
      }
    }
    if (exact) {
      // take every key >= T (T > 0: it has a bit set): keys > T - 1, none by equality
      T -= 1u;
      need_eq = 0;
    } else {
      const uint32_t above =
          T == 0xffffffffu ? 0u : keys.count_ge(T + 1u, srow, lane, init_e, local_lo);
      need_eq = static_cast<int>(k - above);  // how many candidates equal to T are taken
    }
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
      if (pos < S) {
        out[pos] = j;
        emit.taken(pos, j, i);
      }
    }
    nsel += __popc(tm);
  };
  const int passes = (nb_out + 31) / 32;
  if (KPL > 0 && need_eq == 0) {
    // No candidate is taken by equality (take_all, or the early exit, or no tie at T): every
    // pass's take mask is independent of the others, so all ballots go out together; then
    // lane q writes the q-th selected block (q = lane, lane + 32, ...), found from the prefix
    // of the passes' counts and a rank search in its pass's mask: no divergent stores.
    constexpr int KP = KPL > 0 ? KPL : 1;
    unsigned tm[KP];
    int first[KP];  // selected blocks before pass i
#pragma unroll
    for (int i = 0; i < KP; ++i) {
      const int j = i * 32 + lane;
      const bool cand = j < nb && j >= init_e && j < local_lo;
      const bool forced = j < nb_out && (j < init_o || j >= local_o);
      const bool take = i < passes && (forced || (cand && (take_all || keys.k[i] > T)));
      tm[i] = __ballot_sync(0xffffffffu, take);
    }
#pragma unroll
    for (int i = 0; i < KP; ++i) {
      first[i] = nsel;
      nsel += __popc(tm[i]);
    }
    const int nout = min(nsel, S);
    for (int q0 = 0; q0 < nout; q0 += 32) {
      const int q = q0 + lane;
      int ii = 0;
      uint32_t mi = tm[0];
      int base = 0;
#pragma unroll
      for (int i = 1; i < KP; ++i) {
        if (first[i] <= q) {
          ii = i;
          mi = tm[i];
          base = first[i];
        }
      }
      const bool valid = q < nout;
      const int src = valid ? nth_set_bit(mi, q - base) : 0;
      const int j = ii * 32 + src;
      if (valid) out[q] = j;
      emit.gathered(q, j, ii, src, valid);
    }
  } else if (KPL > 0) {
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

template <int KPL, bool CG, typename Emit = NoEmit>
__device__ __forceinline__ int select_row(const float *srow, int nb, int top_k, int init_blocks,
                                          int local_blocks, int S, int32_t *out,
                                          int32_t *dev_err, int lane, int nb_out = 0,
                                          Emit emit = Emit()) {
  auto score = [&](int i) { return load_score<CG>(srow + i * 32 + lane); };
  return select_row_from<KPL, CG>(score, srow, nb, top_k, init_blocks, local_blocks, S, out,
                                  dev_err, lane, nb_out, emit);
}

}  // namespace msa
