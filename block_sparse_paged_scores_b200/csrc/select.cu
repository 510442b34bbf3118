// select.cu — stage 2: forced blocks + top-k of the rest, ascending.
//
// ferrox-core "Module block_sparse": the first init_blocks and the newest local_blocks are
// force-included before any scoring (that is what keeps the selection non-empty), and
// block_sparse_select returns the blocks each KV head may read, ascending.  The remaining
// blocks compete on score; equal scores go to the lower block id.
//
// One warp per (query row, KV head).  The k-th largest candidate key is found exactly by a
// radix select over order-preserving uint32 keys (4 passes of 8 bits, a 256-bin shared-memory
// histogram per warp); one ascending pass over the block ids then keeps the forced blocks,
// every candidate above the threshold key, and the lowest-id candidates equal to it until k
// are taken.  The output comes out in ascending order with no sort.
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

__global__ void __launch_bounds__(32 * kWarps) select_kernel(const SelectArgs a) {
  __shared__ uint32_t hist_all[kWarps][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long item = static_cast<long long>(blockIdx.x) * kWarps + warp;
  if (item >= static_cast<long long>(a.total_q) * a.H_kv) return;
  const int t = static_cast<int>(item / a.H_kv);
  uint32_t *hist = hist_all[warp];
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

  const int init_e = min(a.init_blocks, nb);
  const int local_lo = max(0, nb - a.local_blocks);
  const int n_forced = init_e + (nb - local_lo) - max(0, init_e - local_lo);
  const int n_cand = nb - n_forced;
  const bool take_all = n_cand <= a.top_k;
  auto forced = [&](int j) { return j < init_e || j >= local_lo; };

  // ---- radix select of the top_k-th largest candidate key: threshold T, and how many of
  // the candidates equal to T are still needed (need_eq).
  uint32_t T = 0xffffffffu;  // top_k == 0: no candidate passes
  int need_eq = 0;
  if (!take_all && a.top_k > 0) {
    uint32_t prefix = 0, pmask = 0;
    int kk = a.top_k;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int q = lane; q < 256; q += 32) hist[q] = 0;
      __syncwarp();
      for (int j = lane; j < nb; j += 32) {
        if (forced(j)) continue;
        const uint32_t key = score_key(srow[j]);
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncwarp();
      // lane L owns digits 255-8L .. 248-8L (descending), so a lane prefix sum counts the
      // candidates whose digit is larger.
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        c[q] = hist[255 - 8 * lane - q];
        sum += c[q];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      const uint32_t excl = incl - sum;
      const bool mine = excl < static_cast<uint32_t>(kk) && static_cast<uint32_t>(kk) <= incl;
      const unsigned bal = __ballot_sync(0xffffffffu, mine);
      int digit = 0, above = 0;
      if (mine) {
        uint32_t run = excl;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (run + c[q] >= static_cast<uint32_t>(kk)) {
            digit = 255 - 8 * lane - q;
            above = static_cast<int>(run);
            break;
          }
          run += c[q];
        }
      }
      const int src = bal ? __ffs(bal) - 1 : 0;
      digit = __shfl_sync(0xffffffffu, digit, src);
      above = __shfl_sync(0xffffffffu, above, src);
      kk -= above;
      prefix |= static_cast<uint32_t>(digit) << shift;
      pmask |= 255u << shift;
      __syncwarp();
    }
    T = prefix;
    need_eq = kk;
  }

  // ---- one ascending pass: forced, above T, and the lowest-id ties at T.
  int nsel = 0, eq_seen = 0;
  for (int base = 0; base < nb; base += 32) {
    const int j = base + lane;
    const bool in = j < nb;
    const bool f = in && forced(j);
    bool take;
    if (take_all) {
      take = in;
    } else {
      const bool cand = in && !f;
      const uint32_t key = cand ? score_key(srow[j]) : 0u;
      const bool eq = cand && key == T;
      const unsigned eqm = __ballot_sync(0xffffffffu, eq);
      const int eq_rank = eq_seen + __popc(eqm & lt_mask);
      take = f || (cand && key > T) || (eq && eq_rank < need_eq);
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
  select_kernel<<<blocks, 32 * kWarps, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace msa
