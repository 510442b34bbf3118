// plan.cu — per query tile, the ascending union of the tokens' selected blocks and, for each
// union entry, the bit mask of the tile's tokens that selected it.
//
// Mojo module "msa", "Three attention routes": the speculative route masks causally per token
// inside the kernel, and the prefill route is driven by a device-built CSR of the selected
// blocks.  Here every (sequence, query tile, KV head) item gets a fixed-capacity row of that
// CSR (capacity = min(max_blocks, tile tokens x S)), so the attention kernel reads each
// selected page once per tile and applies each token's own selection as a mask.
//
// One warp per item: a shared-memory bitmap of the blocks marks the union, a warp prefix sum
// of the word popcounts gives each block its union index, and each token ORs its bit into
// the mask of every block it selected.
#include <climits>

#include "internal.h"
#include "ptx.cuh"

namespace msa {

namespace {

__global__ void __launch_bounds__(32) plan_kernel(const PlanArgs a) {
  extern __shared__ uint32_t psm[];
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x;
  const int g = blockIdx.y, y = blockIdx.x;
  const int b = y / a.tiles, tile = y % a.tiles;
  const size_t item = static_cast<size_t>(y) * a.H_kv + g;
  const int words = (a.max_blocks + 31) >> 5;
  uint32_t *bitmap = psm;                 // [words]
  uint32_t *wprefix = psm + words;        // [words] union entries before each word
  uint32_t *mask_s = psm + 2 * words;     // [cap]

  const int row0 = a.row_off[b];
  int q_len = a.row_off[b + 1] - row0;
  if (q_len < 0 || q_len > a.max_q_len) {
    if (lane == 0 && g == 0 && tile == 0) report(a.dev_err, MSA_DEVERR_LENGTHS);
    q_len = q_len < 0 ? 0 : a.max_q_len;
  }
  const int tok0 = tile * a.qt;
  if (tok0 >= q_len) {
    if (lane == 0) a.counts[item] = 0;
    return;
  }
  const int ntok = min(a.qt, q_len - tok0);
  const int cl = a.cache_len[b];
  // the tokens' selection counts, one lane each (ntok <= 32), read all at once
  int n_l = 0;
  if (lane < ntok) {
    n_l = a.num_selected[static_cast<size_t>(row0 + tok0 + lane) * a.H_kv + g];
    if (n_l < 0 || n_l > a.S) {
      report(a.dev_err, MSA_DEVERR_NUM_SELECTED);
      n_l = n_l < 0 ? 0 : a.S;
    }
  }
  // Every (token, slot) pair of the tile, kR per lane at a time, so that the loads of all the
  // tokens' ids are in flight together; `fn(i, j)` is called for each valid id j of token i.
  constexpr int kR = 8;
  const int total = ntok * a.S;
  auto for_each_id = [&](auto fn) {
    for (int k0 = 0; k0 < total; k0 += 32 * kR) {
      int jr[kR], ir[kR];
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        const int k = k0 + r * 32 + lane;
        const int i = k < total ? k / a.S : 0, sl = k - i * a.S;
        const int n = __shfl_sync(0xffffffffu, n_l, i);
        ir[r] = i;
        jr[r] = (k < total && sl < n)
                    ? a.block_ids[(static_cast<size_t>(row0 + tok0 + i) * a.H_kv + g) * a.S + sl]
                    : INT_MIN;
      }
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        if (jr[r] == INT_MIN) continue;
        const int nb = (cl + tok0 + ir[r]) / kBlock + 1;
        fn(ir[r], jr[r], jr[r] >= 0 && jr[r] < nb && jr[r] < a.max_blocks);
      }
    }
  };

  for (int w = lane; w < words; w += 32) bitmap[w] = 0;
  __syncwarp();
  // mark the union
  for_each_id([&](int, int j, bool valid) {
    if (!valid) {
      report(a.dev_err, MSA_DEVERR_BLOCK_ID);
      return;
    }
    atomicOr(&bitmap[j >> 5], 1u << (j & 31));
  });
  __syncwarp();
  // exclusive prefix of the word popcounts
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
  const int U = min(static_cast<int>(carry), a.cap);
  for (int e = lane; e < U; e += 32) mask_s[e] = 0;
  __syncwarp();
  // token masks
  for_each_id([&](int i, int j, bool valid) {
    if (!valid) return;
    const uint32_t w = bitmap[j >> 5];
    const int e = static_cast<int>(wprefix[j >> 5]) + __popc(w & ((1u << (j & 31)) - 1u));
    if (e < U) atomicOr(&mask_s[e], 1u << i);
  });
  __syncwarp();
  // write the CSR row
  int32_t *list = a.list + item * a.cap;
  uint32_t *masks = a.masks + item * a.cap;
  for (int w = lane; w < words; w += 32) {
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
  if (lane == 0) a.counts[item] = U;
}

}  // namespace

cudaError_t launch_plan(const PlanArgs &a, cudaStream_t s) {
  const int words = (a.max_blocks + 31) / 32;
  const size_t smem = (2 * static_cast<size_t>(words) + a.cap) * sizeof(uint32_t);
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(&plan_kernel),
                                    static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(a.batch * a.tiles, a.H_kv);
  return launch_pdl(plan_kernel, grid, dim3(32), smem, s, a);
}

}  // namespace msa
