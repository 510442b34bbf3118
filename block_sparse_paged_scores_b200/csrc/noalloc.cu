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

// The driver's id of the current context (unique for the life of the process, never reused),
// reached through the runtime's entry-point table so that the library needs no link against
// libcuda.  0 when it cannot be had.
unsigned long long current_context_id() {
  using GetCurrentFn = CUresult (*)(CUcontext *);
  using GetIdFn = CUresult (*)(CUcontext, unsigned long long *);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// The array's device address in the current context.  In host code the symbol itself is only
// a host-side stand-in, so the address is asked of the runtime with the device current, and
// kept per device together with the id of the context it belongs to: a new context on the
// device (after cudaDeviceReset, say) reloads the module, and the address is looked up again.
cudaError_t scratch_address(void **out) {
  struct Entry {
    unsigned long long ctx;
    void *addr;
  };
  static Entry cache[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev].addr || ctx == 0 || cache[dev].ctx != ctx) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    cache[dev].addr = p;
    // read after the lookup, which makes the device's primary context current if no context
    // was yet (the id read before it was then 0)
    cache[dev].ctx = current_context_id();
  }
  *out = cache[dev].addr;
  return cudaSuccess;
}

}  // namespace

}  // namespace msa

extern "C" msa_status_t msa_sparse_attn_paged_noalloc(
    const msa_ragged_paged_t *rp, const void *q, const void *k_cache, const void *v_cache,
    msa_kv_dtype_t kv_dtype, const int32_t *block_ids, const int32_t *num_selected, int32_t S,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t max_blocks, float scale,
    int32_t num_splits, void *out, int32_t *dev_err, struct CUstream_st *stream) {
  // `out` is required here: with out == NULL the split-K partials would stay in the library's
  // own array, where the caller cannot reach them.
  if (!rp || !out || S < 1 || num_kv_heads < 1 || num_q_heads < num_kv_heads ||
      max_blocks < 1 || num_splits < 0)
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
