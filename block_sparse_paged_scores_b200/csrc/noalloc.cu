// noalloc.cu — msa_sparse_attn_paged without a caller-provided workspace.
//
// Some callers cannot hand this library a workspace: a host runtime whose device memory plan
// is fixed before it starts serving and has no allocator to call afterwards, or a plugin
// interface that passes only the operation's inputs and outputs.  For them the split-K
// partials and the per-tile block lists live in one file-scope device array instead.  That
// array is part of the library image: every GPU on which the library is loaded holds it
// until the process exits, so it is kept to a modest, stated size (MSA_NOALLOC_SCRATCH_BYTES).
// This file calls no allocator; it only looks the array's device address up.
#include <mutex>

#include "internal.h"

namespace msa {

namespace {

__device__ __align__(256) uint8_t g_noalloc_scratch[MSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// The array's device address on the current device.  In host code the symbol itself is only
// a host-side stand-in, so the address is asked of the runtime once per device (with that
// device current) and kept.
cudaError_t scratch_address(void **out) {
  static void *addr[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace

}  // namespace msa

extern "C" msa_status_t msa_sparse_attn_paged_noalloc(
    const msa_ragged_paged_t *rp, const void *q, const void *k_cache, const void *v_cache,
    msa_kv_dtype_t kv_dtype, const int32_t *block_ids, const int32_t *num_selected, int32_t S,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t max_blocks, float scale,
    int32_t num_splits, void *out, int32_t *dev_err, struct CUstream_st *stream) {
  if (!rp || S < 1 || num_kv_heads < 1 || num_q_heads < num_kv_heads || max_blocks < 1 ||
      num_splits < 0)
    return MSA_ERR_INVALID_ARG;
  const size_t need =
      msa_attn_workspace_bytes(rp, S, num_q_heads, num_kv_heads, max_blocks, num_splits);
  if (need > static_cast<size_t>(MSA_NOALLOC_SCRATCH_BYTES)) return MSA_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  if (msa::scratch_address(&scratch) != cudaSuccess) return MSA_ERR_CUDA;
  // Nothing in the workspace has to start at zero: every byte the kernels read is written
  // earlier in the same call, so the previous call's leftovers do no harm.
  return msa_sparse_attn_paged(rp, q, k_cache, v_cache, kv_dtype, block_ids, num_selected, S,
                               num_q_heads, num_kv_heads, max_blocks, scale, num_splits, scratch,
                               MSA_NOALLOC_SCRATCH_BYTES, out, dev_err, stream);
}
