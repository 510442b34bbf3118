// select.cu — stage 2: forced blocks + top-k of the rest, ascending.
//
// ferrox-core "Module block_sparse": the first init_blocks and the newest local_blocks are
// force-included before any scoring (that is what keeps the selection non-empty), and
// block_sparse_select returns the blocks each KV head may read, ascending.  The remaining
// blocks compete on score; equal scores go to the lower block id.
//
// One warp per (query row, KV head).  The candidates' scores become order-preserving uint32
// keys held in registers; the exact top_k-th largest key is then built bit by bit from the top
// (32 rounds of "how many keys are >= this prefix", one warp reduction each, no atomics).  One
// ascending pass over the block ids keeps the forced blocks, every candidate above that
// threshold, and the lowest-id candidates equal to it until top_k are taken, so the output
// comes out in ascending order with no sort.
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace msa {

namespace {

constexpr int kWarps = 4;

__device__ __forceinline__ int find_sequence(const int32_t *row_off, int batch, int t) {
  int lo = 0, hi = batch;  // row_off[lo] <= t < row_off[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (row_off[mid] <= t)
      lo = mid;
    else
      hi = mid;
  }
  return lo;
}

// Keys of the candidate blocks (0 for blocks that are not candidates: every real key is at
// least score_key(-inf) = 0x007fffff > 0).  KPL keys per lane stay in registers; KPL == 0
// reads them from memory on every pass (any number of blocks).
template <int KPL>
struct Keys {
  uint32_t k[KPL > 0 ? KPL : 1];
  __device__ __forceinline__ void load(const float *srow, int nb, int lane, int init_e,
                                       int local_lo) {
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
      const int j = i * 32 + lane;
      k[i] = (j < nb && j >= init_e && j < local_lo) ? score_key(srow[j]) : 0u;
    }
  }
  // number of candidate keys >= x (over the warp)
  __device__ __forceinline__ uint32_t count_ge(uint32_t x, const float *srow, int nb, int lane,
                                               int init_e, int local_lo) const {
    uint32_t c = 0;
    if (KPL > 0) {
#pragma unroll
      for (int i = 0; i < KPL; ++i) c += k[i] >= x;
    } else {
      for (int j = init_e + lane; j < local_lo; j += 32) c += score_key(srow[j]) >= x;
    }
    return __reduce_add_sync(0xffffffffu, c);
  }
  __device__ __forceinline__ uint32_t key(int i, int j, const float *srow, int init_e,
                                          int local_lo) const {
    if (KPL > 0) return k[i];
    return (j >= init_e && j < local_lo) ? score_key(srow[j]) : 0u;
  }
};

template <int KPL>
__global__ void __launch_bounds__(32 * kWarps) select_kernel(const SelectArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long item = static_cast<long long>(blockIdx.x) * kWarps + warp;
  if (item >= static_cast<long long>(a.total_q) * a.H_kv) return;
  const int t = static_cast<int>(item / a.H_kv);
  const unsigned lt_mask = (1u << lane) - 1u;

  const int b = find_sequence(a.row_off, a.batch, t);
  const int p = a.cache_len[b] + (t - a.row_off[b]);
  int nb = (p < 0 ? 0 : p) / kBlock + 1;
  if (nb > a.max_blocks) {
    if (lane == 0) report(a.dev_err, MSA_DEVERR_LENGTHS);
    nb = a.max_blocks;
  }
  const float *srow = a.scores + static_cast<size_t>(item) * a.max_blocks;
  int32_t *out = a.block_ids + static_cast<size_t>(item) * a.S;

  // forced: [0, init_e) and [local_lo, nb); candidates: [init_e, local_lo)
  const int init_e = min(a.init_blocks, nb);
  const int local_lo = max(init_e, nb - a.local_blocks);
  const int n_cand = local_lo - init_e;
  const bool take_all = n_cand <= a.top_k;

  Keys<KPL> keys;
  uint32_t T = 0xffffffffu;  // top_k == 0: no candidate passes
  int need_eq = 0;
  if (!take_all && a.top_k > 0) {
    keys.load(srow, nb, lane, init_e, local_lo);
    // T = the top_k-th largest candidate key: the largest x with count(key >= x) >= top_k,
    // built one bit at a time from the top.
    const uint32_t k = static_cast<uint32_t>(a.top_k);
    T = 0;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t x = T | (1u << bit);
      if (keys.count_ge(x, srow, nb, lane, init_e, local_lo) >= k) T = x;
    }
    const uint32_t above = T == 0xffffffffu
                               ? 0u
                               : keys.count_ge(T + 1u, srow, nb, lane, init_e, local_lo);
    need_eq = static_cast<int>(k - above);  // how many candidates equal to T are taken
  }

  // one ascending pass: forced, above T, and the lowest-id candidates equal to T
  int nsel = 0, eq_seen = 0;
  const int passes = (nb + 31) / 32;
  for (int i = 0; i < passes; ++i) {
    const int j = i * 32 + lane;
    const bool in = j < nb;
    const bool cand = in && j >= init_e && j < local_lo;
    bool take;
    if (take_all) {
      take = in;
    } else {
      uint32_t key = 0;
      if (KPL > 0) {
#pragma unroll
        for (int q = 0; q < (KPL > 0 ? KPL : 1); ++q)
          if (q == i) key = keys.key(q, j, srow, init_e, local_lo);
      } else {
        key = cand ? score_key(srow[j]) : 0u;
      }
      const bool eq = cand && key == T;
      const unsigned eqm = __ballot_sync(0xffffffffu, eq);
      const int eq_rank = eq_seen + __popc(eqm & lt_mask);
      take = (in && !cand) || (cand && key > T) || (eq && eq_rank < need_eq);
      eq_seen += __popc(eqm);
    }
    const unsigned tm = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int pos = nsel + __popc(tm & lt_mask);
      if (pos < a.S) out[pos] = j;
    }
    nsel += __popc(tm);
  }
  if (nsel > a.S) {  // cannot happen when S == init + local + top_k
    if (lane == 0) report(a.dev_err, MSA_DEVERR_NUM_SELECTED);
    nsel = a.S;
  }
  for (int q = nsel + lane; q < a.S; q += 32) out[q] = -1;
  if (lane == 0) a.num_selected[item] = nsel;
}

}  // namespace

cudaError_t launch_select(const SelectArgs &a, cudaStream_t s) {
  const long long items = static_cast<long long>(a.total_q) * a.H_kv;
  const unsigned blocks = static_cast<unsigned>((items + kWarps - 1) / kWarps);
  const dim3 grid(blocks), block(32 * kWarps);
  if (a.max_blocks <= 4 * 32) return launch_pdl(select_kernel<4>, grid, block, 0, s, a);
  if (a.max_blocks <= 16 * 32) return launch_pdl(select_kernel<16>, grid, block, 0, s, a);
  if (a.max_blocks <= 32 * 32) return launch_pdl(select_kernel<32>, grid, block, 0, s, a);
  return launch_pdl(select_kernel<0>, grid, block, 0, s, a);
}

}  // namespace msa
