// combine.cu — split-K combine.
//
// Mojo module "msa", "Three attention routes": with more than one split-K partition the
// partials are keyed on the ragged global query row and a combine writes the ragged output.
// Each partition carries its softmax-normalised output o_s and the natural log of its sum of
// exponentials lse_s; the merge weighs o_s by exp(lse_s - max_s lse_s).
//
// One warp per (query row, head); each lane owns 4 of the 128 dims (one float4 per split).
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace msa {

namespace {

constexpr int kWarps = 8;
constexpr int kPre = 2;  // partitions whose outputs are loaded with the log-sum-exps

// One warp per (row, head).  All partitions' log-sum-exps are fetched at once (one lane
// each).  With at most kPre partitions their output float4s are fetched with them (one that
// turns out empty is loaded but not used), so that the warp waits for one memory latency;
// with more, every non-empty partition's output is issued before any is used (two latencies,
// and no loads of empty partitions).
__global__ void __launch_bounds__(32 * kWarps)
    combine_kernel(const float *__restrict__ part_o, const float *__restrict__ part_lse,
                   int splits, long long rows, uint16_t *__restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f, M = -INFINITY;  // running max of the log-sum-exps seen so far
  float4 pre[kPre];
#pragma unroll
  for (int s = 0; s < kPre; ++s)
    if (splits <= kPre && s < splits)
      pre[s] = reinterpret_cast<const float4 *>(part_o + (s * rows + row) * kHeadDim)[lane];
  for (int s0 = 0; s0 < splits; s0 += 32) {
    const int n = min(32, splits - s0);
    const float my_lse = lane < n ? part_lse[(s0 + lane) * rows + row] : -INFINITY;
    float m = my_lse;
#pragma unroll
    for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (m == -INFINITY) continue;
    const float m_new = fmaxf(M, m);
    const float keep = M == -INFINITY ? 0.f : expf(M - m_new);  // rescale earlier chunks
    acc.x *= keep;
    acc.y *= keep;
    acc.z *= keep;
    acc.w *= keep;
    wsum *= keep;
    M = m_new;
    const float w_lane = my_lse == -INFINITY ? 0.f : expf(my_lse - m_new);
#pragma unroll 8
    for (int s = 0; s < n; ++s) {
      const float w = __shfl_sync(0xffffffffu, w_lane, s);
      if (w == 0.f) continue;
      float4 o;
      if (splits <= kPre) {
#pragma unroll
        for (int t = 0; t < kPre; ++t)
          if (t == s) o = pre[t];
      } else {
        o = reinterpret_cast<const float4 *>(part_o + ((s0 + s) * rows + row) * kHeadDim)[lane];
      }
      acc.x += w * o.x;
      acc.y += w * o.y;
      acc.z += w * o.z;
      acc.w += w * o.w;
      wsum += w;
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint2 packed;
  packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  reinterpret_cast<uint2 *>(out + row * kHeadDim)[lane] = packed;
}

}  // namespace

cudaError_t launch_combine(const float *part_o, const float *part_lse, int splits, int total_q,
                           int H_q, uint16_t *out, cudaStream_t s) {
  const long long rows = static_cast<long long>(total_q) * H_q;
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((rows + kWarps - 1) / kWarps);
  return launch_pdl(combine_kernel, dim3(blocks), dim3(32 * kWarps), 0, s, part_o, part_lse,
                    splits, rows, out);
}

}  // namespace msa
