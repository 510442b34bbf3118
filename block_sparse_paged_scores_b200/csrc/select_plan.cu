// select_plan.cu — stages 2 and the speculative route's per-tile plan in one launch.
//
// ferrox-core "Module block_sparse" (forced init / local blocks, top-k of the rest, ascending)
// for every token of a speculative query tile, and Mojo module "msa", "Three attention routes"
// (the speculative route masks causally per token inside the kernel, driven by each tile's
// union of selected blocks): the same block_ids / num_selected as the selection kernel, and the
// same union list, token masks and counts as the plan kernel, from one CTA per (sequence, query
// tile, KV head) instead of a warp per row followed by a warp per tile.
//
// Warp i selects token tok0 + i's row (select_row); every block it takes goes into a
// shared-memory bitmap of the tile's union and into the warp's id list.  Then one warp turns the
// bitmap into union indices (a prefix of the words' popcounts), each warp ORs its token's bit
// into the masks of its blocks, and the CTA writes the fixed-capacity CSR row.
#include "select_row.cuh"

namespace msa {

namespace {

struct TileEmit {
  uint32_t *bitmap;  // the tile's union
  int *ids;          // this warp's selected ids, by position
  __device__ __forceinline__ void put(int pos, int j) const {
    ids[pos] = j;
    atomicOr(&bitmap[j >> 5], 1u << (j & 31));
  }
  __device__ __forceinline__ void taken(int pos, int j, int) const { put(pos, j); }
  __device__ __forceinline__ void gathered(int pos, int j, int, int, bool valid) const {
    if (valid) put(pos, j);
  }
};

template <int KPL>
__global__ void __launch_bounds__(32 * kMaxSpecTileTokens)
    select_plan_kernel(const SelectPlanArgs a) {
  extern __shared__ uint32_t sm[];
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y, y = blockIdx.x;
  const int b = y / a.tiles, tile = y % a.tiles;
  const size_t item = static_cast<size_t>(y) * a.H_kv + g;
  const int words = (a.max_blocks + 31) >> 5;
  uint32_t *bitmap = sm;                                   // [words]
  uint32_t *wprefix = sm + words;                          // [words]
  uint32_t *mask_s = sm + 2 * words;                       // [cap]
  int *nsel_s = reinterpret_cast<int *>(mask_s + a.cap);   // [qt] tokens' counts, then U
  int *ids_s = nsel_s + kMaxSpecTileTokens + 1;            // [qt][S]

  const int row0 = a.row_off[b];
  int q_len = a.row_off[b + 1] - row0;
  if (q_len < 0 || q_len > a.max_q_len) {
    if (threadIdx.x == 0 && g == 0 && tile == 0) report(a.dev_err, MSA_DEVERR_LENGTHS);
    q_len = q_len < 0 ? 0 : a.max_q_len;
  }
  const int tok0 = tile * a.qt;
  if (tok0 >= q_len) {  // a tile past the sequence's end: no rows, an empty union
    if (threadIdx.x == 0) a.counts[item] = 0;
    return;
  }
  const int ntok = min(a.qt, q_len - tok0);
  const int cl = a.cache_len[b];
  for (int w = threadIdx.x; w < words; w += blockDim.x) bitmap[w] = 0;
  __syncthreads();

  // ---- each token's selection (as the selection kernel: same arguments, same output)
  if (warp < ntok) {
    const int t = row0 + tok0 + warp;
    const int p = cl + tok0 + warp;
    int nb = (p < 0 ? 0 : p) / kBlock + 1;
    if (nb > a.max_blocks) {
      if (lane == 0) report(a.dev_err, MSA_DEVERR_LENGTHS);
      nb = a.max_blocks;
    }
    const size_t row = static_cast<size_t>(t) * a.H_kv + g;
    const TileEmit emit{bitmap, ids_s + warp * a.S};
    const int n = select_row<KPL, false>(a.scores + row * a.max_blocks, nb, a.top_k,
                                         a.init_blocks, a.local_blocks, a.S,
                                         a.block_ids + row * a.S, a.dev_err, lane, 0, emit);
    if (lane == 0) {
      a.num_selected[row] = n;
      nsel_s[warp] = min(n, a.S);
    }
  }
  __syncthreads();

  // ---- union indices: exclusive prefix of the words' popcounts
  if (warp == 0) {
    uint32_t carry = 0;
    for (int base = 0; base < words; base += 32) {
      const int w = base + lane;
      const uint32_t c = w < words ? __popc(bitmap[w]) : 0u;
      uint32_t incl = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      if (w < words) wprefix[w] = carry + incl - c;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) nsel_s[kMaxSpecTileTokens] = min(static_cast<int>(carry), a.cap);
  }
  __syncthreads();
  const int U = nsel_s[kMaxSpecTileTokens];
  for (int e = threadIdx.x; e < U; e += blockDim.x) mask_s[e] = 0;
  __syncthreads();

  // ---- token masks: token i's bit on every union entry it selected
  if (warp < ntok) {
    const int n = nsel_s[warp];
    for (int pos = lane; pos < n; pos += 32) {
      const int j = ids_s[warp * a.S + pos];
      const uint32_t w = bitmap[j >> 5];
      const int e = static_cast<int>(wprefix[j >> 5]) + __popc(w & ((1u << (j & 31)) - 1u));
      if (e < U) atomicOr(&mask_s[e], 1u << warp);
    }
  }
  __syncthreads();

  // ---- the CSR row
  int32_t *list = a.list + item * a.cap;
  uint32_t *masks = a.masks + item * a.cap;
  for (int w = threadIdx.x; w < words; w += blockDim.x) {
    uint32_t bits = bitmap[w];
    int e = static_cast<int>(wprefix[w]);
    while (bits) {
      const int k = __ffs(bits) - 1;
      bits &= bits - 1;
      if (e < U) {
        list[e] = w * 32 + k;
        masks[e] = mask_s[e];
      }
      ++e;
    }
  }
  if (threadIdx.x == 0) a.counts[item] = U;
}

}  // namespace

size_t select_plan_smem_bytes(int max_blocks, int cap, int S) {
  const size_t words = (static_cast<size_t>(max_blocks) + 31) / 32;
  return (2 * words + cap + kMaxSpecTileTokens + 1 +
          static_cast<size_t>(kMaxSpecTileTokens) * S) *
         sizeof(uint32_t);
}

cudaError_t launch_select_plan(const SelectPlanArgs &a, cudaStream_t s) {
  const size_t smem = select_plan_smem_bytes(a.max_blocks, a.cap, a.S);
  const dim3 grid(a.batch * a.tiles, a.H_kv), block(32 * a.qt);
  auto go = [&](auto kernel) -> cudaError_t {
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(kernel),
                                      static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    return launch_pdl(kernel, grid, block, smem, s, a);
  };
  if (a.max_blocks <= 8 * 32) return go(&select_plan_kernel<8>);
  if (a.max_blocks <= 16 * 32) return go(&select_plan_kernel<16>);
  if (a.max_blocks <= 32 * 32) return go(&select_plan_kernel<32>);
  return go(&select_plan_kernel<0>);
}

}  // namespace msa
