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

__global__ void __launch_bounds__(32 * kWarps)
    combine_kernel(const float *__restrict__ part_o, const float *__restrict__ part_lse,
                   int splits, long long rows, uint16_t *__restrict__ out) {
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  float m = -INFINITY;
  for (int s = lane; s < splits; s += 32) m = fmaxf(m, part_lse[s * rows + row]);
#pragma unroll
  for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < splits; ++s) {
      const float lse = part_lse[s * rows + row];
      if (lse == -INFINITY) continue;
      const float w = expf(lse - m);
      const float4 o = reinterpret_cast<const float4 *>(part_o + (s * rows + row) * kHeadDim)[lane];
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
  combine_kernel<<<blocks, 32 * kWarps, 0, s>>>(part_o, part_lse, splits, rows, out);
  return cudaGetLastError();
}

}  // namespace msa
