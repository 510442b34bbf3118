// select.cu — stage 2: forced blocks + top-k of the rest, ascending.
//
// ferrox-core "Module block_sparse": the first init_blocks and the newest local_blocks are
// force-included before any scoring, and block_sparse_select returns the blocks each KV head
// may read, ascending; equal scores go to the lower block id.  One warp per (query row, KV
// head); the per-row algorithm (an exact bitwise threshold search over register-held keys, then
// one ascending compaction pass) is select_row in select_row.cuh.
#include "select_row.cuh"

namespace msa {

namespace {

constexpr int kWarps = 4;

// The sequence of row t: the largest b < batch with row_off[b] <= t, by a warp-wide 32-ary
// search (one load per lane per level: one level up to 32 sequences, two up to 1024).
__device__ __forceinline__ int find_sequence(const int32_t *row_off, int batch, int t, int lane) {
  int lo = 0, n = batch;  // row_off[lo] <= t, and t < row_off[lo + n] unless lo + n == batch
  while (n > 1) {
    const int step = (n + 31) / 32;
    const bool le = lane * step < n && row_off[lo + lane * step] <= t;
    const unsigned m = __ballot_sync(0xffffffffu, le);  // lane 0 always set
    const int last = 31 - __clz(m);
    lo += last * step;
    n = min(step, n - last * step);
  }
  return lo;
}

template <int KPL>
__global__ void __launch_bounds__(32 * kWarps) select_kernel(const SelectArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long item = static_cast<long long>(blockIdx.x) * kWarps + warp;
  if (item >= static_cast<long long>(a.total_q) * a.H_kv) return;
  const int t = static_cast<int>(item / a.H_kv);

  const int b = find_sequence(a.row_off, a.batch, t, lane);
  const int p = a.cache_len[b] + (t - a.row_off[b]);
  int nb = (p < 0 ? 0 : p) / kBlock + 1;
  if (nb > a.max_blocks) {
    if (lane == 0) report(a.dev_err, MSA_DEVERR_LENGTHS);
    nb = a.max_blocks;
  }
  const float *srow = a.scores + static_cast<size_t>(item) * a.max_blocks;
  int32_t *out = a.block_ids + static_cast<size_t>(item) * a.S;
  const int nsel = select_row<KPL, false>(srow, nb, a.top_k, a.init_blocks, a.local_blocks, a.S,
                                          out, a.dev_err, lane);
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
