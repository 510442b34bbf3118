// selftest.cu — msa_selftest_bounded_wait: the bounded pipeline wait every pipelined kernel of
// this library uses (ptx.cuh, mbar_wait), made to run out on purpose so that its give-up path
// can be checked on a GPU without hanging it.
//
// One CTA of two warps and three mbarriers.  Nothing ever arrives on the first two:
//   warp 0  waits on barrier 0 with the caller's limit; it gives up, reports
//           MSA_DEVERR_TIMEOUT and raises the CTA's abort flag, as a pipeline role does;
//   warp 1  waits on barrier 1 with four times that limit; it leaves as soon as it sees the
//           abort flag, as the other roles of a pipeline do;
// and then one thread arrives on barrier 2 and waits on it: a wait on a completed phase
// returns at once.  Every wait here ends by itself; nothing traps.
#include "internal.h"
#include "ptx.cuh"

namespace msa {

namespace {

__global__ void __launch_bounds__(64) bounded_wait_selftest_kernel(int32_t *dev_err,
                                                                   uint32_t *result,
                                                                   uint64_t limit_ns) {
  __shared__ uint64_t bar[3];
  __shared__ volatile int abort_flag, no_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(&bar[i], 1);
    abort_flag = 0;
    no_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (lane == 0) {
    const uint64_t t0 = global_timer_ns();
    bool ok;
    if (warp == 0) {
      ok = mbar_wait(&bar[0], 0, &abort_flag, limit_ns);
      if (!ok) {
        report(dev_err, MSA_DEVERR_TIMEOUT);
        abort_flag = 1;
      }
    } else {
      ok = mbar_wait(&bar[1], 0, &abort_flag, 4 * limit_ns);
    }
    const uint64_t us = (global_timer_ns() - t0) / 1000ull;
    result[2 * warp] = ok ? 1u : 2u;  // 1: the phase completed, 2: the wait gave up
    result[2 * warp + 1] = static_cast<uint32_t>(us < 0xffffffffull ? us : 0xffffffffull);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive(&bar[2]);
    result[4] = mbar_wait(&bar[2], 0, &no_abort, limit_ns) ? 1u : 2u;
  }
}

}  // namespace

}  // namespace msa

extern "C" msa_status_t msa_selftest_bounded_wait(uint32_t limit_us, int32_t *dev_err,
                                                  uint32_t *result, struct CUstream_st *stream) {
  if (!result || limit_us < 1 || limit_us > 1000000u ||
      (reinterpret_cast<uintptr_t>(result) & 3u) != 0)
    return MSA_ERR_INVALID_ARG;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  msa::bounded_wait_selftest_kernel<<<1, 64, 0, s>>>(dev_err, result,
                                                     static_cast<uint64_t>(limit_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}
