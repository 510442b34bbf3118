// latent.cu — latent sparse attention over two paged leaves.
//
// Mojo "Struct_latent_sparse_attention_ragged_paged" (the mo.latent_sparse_attention.ragged.
// paged op): attention over a K = V latent shared by every query head, read from a sliding-
// window leaf by position range and from a compressed leaf by an explicit per-query entry list,
// with a per-head attention sink in the softmax denominator:
//   out[t, h] = sum_x e^(z_x) v_x / (e^(sink[h]) + sum_x e^(z_x)),   z_x = scale * q[t, h] . v_x
// over x in the window [p - window + 1, p] (p = swa_cache_lengths[b] + i, clipped at 0) and the
// entries comp_indices[t, :] that are >= 0.
//
// One CTA per (query token, group of 64 heads, split of the token's position list).  The list
// is the window positions followed by the entry slots; a split takes an equal share of it.
// K = V rows (256 bytes) are gathered with 16-byte cp.async into a 3-stage ring of 64-row tiles
// (the 16-byte chunks XOR-swizzled by row, so that ldmatrix reads are conflict-free); every
// thread computes the page lookups of its own rows two tiles ahead.  Four warps each own 16
// heads: S = Q K^T and O += P V on bf16 mma.sync with fp32 accumulators, the same smem tile
// serving as K (ldmatrix) and as V (ldmatrix.trans), an online softmax in the exp2 domain.  The
// sink enters split 0's state as a position of its own with no value (m = sink, l = 1), so the
// split-K combine counts it exactly once.  A single split writes the bf16 output itself.
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace msa {

namespace {

constexpr int kLatWarps = 4;
constexpr int kLatThreads = 32 * kLatWarps;
constexpr int kLatRows = 16 * kLatWarps;  // heads per CTA
constexpr int kLatTile = 64;              // positions per tile
constexpr int kLatStages = 3;
constexpr uint32_t kLatTileBytes = kLatTile * 256;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Byte offset of 16-byte chunk ch (0..15) of row r in a tile of 256-byte rows: the low three
// bits of the chunk index are XOR-ed with the row index mod 8.
__device__ __forceinline__ uint32_t lat_off(int r, int ch) {
  return static_cast<uint32_t>(r) * 256u +
         (static_cast<uint32_t>((ch & 8) | ((ch & 7) ^ (r & 7))) << 4);
}

__global__ void __launch_bounds__(kLatThreads) latent_attn_kernel(const LatentArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x, hg = blockIdx.y, split = blockIdx.z;

  extern __shared__ __align__(128) uint8_t lat_smem[];
  uint8_t(*tiles)[kLatTileBytes] = reinterpret_cast<uint8_t(*)[kLatTileBytes]>(lat_smem);
  uint8_t(*valid_s)[kLatTile] =
      reinterpret_cast<uint8_t(*)[kLatTile]>(lat_smem + kLatStages * kLatTileBytes);
  __shared__ int seq_s;

  // the sequence of row t (binary search over the row offsets)
  if (threadIdx.x == 0) {
    int lo = 0, hi = a.batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.row_off[mid] <= t) lo = mid;
      else hi = mid - 1;
    }
    seq_s = lo;
  }
  __syncthreads();
  const int b = seq_s;
  const int i = t - a.row_off[b];
  int swa_prior = a.swa_len[b];
  int comp_len = a.comp_len[b];
  if (swa_prior < 0 || comp_len < 0 || i < 0 || i >= a.max_q_len) {
    if (threadIdx.x == 0 && hg == 0 && split == 0) report(a.dev_err, MSA_DEVERR_LENGTHS);
    swa_prior = max(swa_prior, 0);
    comp_len = max(comp_len, 0);
  }
  const int p = swa_prior + i;
  const int w0 = max(0, p - a.window + 1);
  const int nw = p - w0 + 1;
  const int n_list = nw + a.n_entries;
  const int per = (n_list + a.splits * kLatTile - 1) / (a.splits * kLatTile) * kLatTile;
  const int lo = split * per, hi = min(n_list, lo + per);
  const int n_tiles = hi > lo ? (hi - lo + kLatTile - 1) / kLatTile : 0;
  const int32_t *entries = a.comp_idx + static_cast<size_t>(t) * a.n_entries;

  // ---- the row of list index idx: a global address, or nullptr (padding / out of range)
  auto row_ptr = [&](int idx, bool report_bad) -> const uint16_t * {
    if (idx >= hi) return nullptr;
    if (idx < nw) {
      const int pos = w0 + idx;
      const int pg = pos / kBlock < a.swa_max_pages
                         ? a.swa_table[static_cast<size_t>(b) * a.swa_max_pages + pos / kBlock]
                         : -1;
      if (pg < 0 || pg >= a.swa_pages) {
        if (report_bad) report(a.dev_err, MSA_DEVERR_PAGE_ID);
        return nullptr;
      }
      return a.swa_kv + ((static_cast<size_t>(pg) * a.swa_layers + a.swa_layer) * kBlock +
                         (pos % kBlock)) * kHeadDim;
    }
    const int e = entries[idx - nw];
    if (e < 0) return nullptr;  // padding
    if (e >= comp_len) {
      if (report_bad) report(a.dev_err, MSA_DEVERR_BLOCK_ID);
      return nullptr;
    }
    const int pg = e / kBlock < a.comp_max_pages
                       ? a.comp_table[static_cast<size_t>(b) * a.comp_max_pages + e / kBlock]
                       : -1;
    if (pg < 0 || pg >= a.comp_pages) {
      if (report_bad) report(a.dev_err, MSA_DEVERR_PAGE_ID);
      return nullptr;
    }
    return a.comp_kv + ((static_cast<size_t>(pg) * a.comp_layers + a.comp_layer) * kBlock +
                        (e % kBlock)) * kHeadDim;
  };
  // ---- gather tile k into its stage: thread tid copies chunk tid % 16 of rows tid / 16 + 8 j
  const int ch = threadIdx.x & 15, r0 = threadIdx.x >> 4;
  auto issue = [&](int k) {
    if (k < n_tiles) {
      const int st = k % kLatStages;
      const uint32_t base = smem_u32(tiles[st]);
#pragma unroll
      for (int j = 0; j < kLatTile / 8; ++j) {
        const int r = r0 + 8 * j;
        const uint16_t *src = row_ptr(lo + k * kLatTile + r, ch == 0 && hg == 0);
        cp_async16(base + lat_off(r, ch), src ? src + ch * 8 : a.q, src != nullptr);
        if (ch == 0) valid_s[st][r] = src != nullptr;
      }
    }
    cp_async_commit();
  };

  // ---- Q fragments of this warp's 16 heads (rows g and g + 8, dims 16 ks + 2 c (+ 8))
  const int g = lane >> 2, c = lane & 3;
  const int h0 = hg * kLatRows + warp * 16;
  uint32_t qa[8][4];
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      const int h = h0 + g + (q4 & 1) * 8;
      const int d = 16 * ks + 2 * c + (q4 >> 1) * 8;
      qa[ks][q4] = h < a.H ? *reinterpret_cast<const uint32_t *>(
                                 a.q + (static_cast<size_t>(t) * a.H + h) * kHeadDim + d)
                           : 0u;
    }
  // the sink is split 0's first "position": m = sink, l = 1, no value
  float m_run[2], l_run[2];
#pragma unroll
  for (int sl = 0; sl < 2; ++sl) {
    const int h = h0 + g + 8 * sl;
    const bool own_sink = split == 0 && h < a.H;
    m_run[sl] = own_sink ? a.sink[h] * kLog2e : -INFINITY;
    l_run[sl] = own_sink ? 1.f : 0.f;
  }
  float o[16][4];
#pragma unroll
  for (int dn = 0; dn < 16; ++dn)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[dn][e] = 0.f;

  issue(0);
  issue(1);
  for (int k = 0; k < n_tiles; ++k) {
    issue(k + 2);
    cp_async_wait<2>();
    __syncthreads();
    const int st = k % kLatStages;
    const uint32_t tb = smem_u32(tiles[st]);
    // S = Q K^T over the tile's 64 positions
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
    const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(tb + lat_off(16 * np + (mi >> 1) * 8 + rr, 2 * ks + (mi & 1)), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qa[ks], b0, b1);
        mma_bf16(s[2 * np + 1], qa[ks], b2, b3);
      }
    // masked online softmax (exp2 domain), rows g (slot 0) and g + 8 (slot 1)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool ok = valid_s[st][8 * nt + 2 * c + (e & 1)] != 0;
        s[nt][e] = ok ? s[nt][e] * a.scale_log2 : -INFINITY;
        mx[e >> 1] = fmaxf(mx[e >> 1], s[nt][e]);
      }
    float alpha[2], m_use[2];
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
      mx[sl] = fmaxf(mx[sl], __shfl_xor_sync(0xffffffffu, mx[sl], 1));
      mx[sl] = fmaxf(mx[sl], __shfl_xor_sync(0xffffffffu, mx[sl], 2));
      const float m_new = fmaxf(m_run[sl], mx[sl]);
      m_use[sl] = m_new == -INFINITY ? 0.f : m_new;
      alpha[sl] = m_run[sl] == -INFINITY ? 0.f : fast_exp2(m_run[sl] - m_use[sl]);
      m_run[sl] = m_new;
    }
    float ps[2] = {0.f, 0.f};
    uint32_t pa[4][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p0 = fast_exp2(s[nt][0] - m_use[0]), p1 = fast_exp2(s[nt][1] - m_use[0]);
      const float p2 = fast_exp2(s[nt][2] - m_use[1]), p3 = fast_exp2(s[nt][3] - m_use[1]);
      const uint32_t lo01 = pack_bf16x2(p0, p1), hi23 = pack_bf16x2(p2, p3);
      // the row sums add the rounded P the P V MMA reads
      const float2 f01 = bf16x2_to_float2(lo01), f23 = bf16x2_to_float2(hi23);
      ps[0] += f01.x + f01.y;
      ps[1] += f23.x + f23.y;
      pa[nt >> 1][(nt & 1) * 2 + 0] = lo01;
      pa[nt >> 1][(nt & 1) * 2 + 1] = hi23;
    }
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
      ps[sl] += __shfl_xor_sync(0xffffffffu, ps[sl], 1);
      ps[sl] += __shfl_xor_sync(0xffffffffu, ps[sl], 2);
      l_run[sl] = l_run[sl] * alpha[sl] + ps[sl];
    }
#pragma unroll
    for (int dn = 0; dn < 16; ++dn) {
      o[dn][0] *= alpha[0];
      o[dn][1] *= alpha[0];
      o[dn][2] *= alpha[1];
      o[dn][3] *= alpha[1];
    }
    // O += P V, V = the same tile read transposed
#pragma unroll
    for (int kp = 0; kp < 4; ++kp)
#pragma unroll
      for (int dp = 0; dp < 8; ++dp) {
        uint32_t v0, v1, v2, v3;
        ldsm_x4_t(tb + lat_off(16 * kp + (mi & 1) * 8 + rr, 2 * dp + (mi >> 1)), v0, v1, v2,
                  v3);
        mma_bf16(o[2 * dp], pa[kp], v0, v1);
        mma_bf16(o[2 * dp + 1], pa[kp], v2, v3);
      }
    __syncthreads();  // the stage is free for the tile three ahead
  }
  cp_async_wait<0>();

  // ---- epilogue: O / l in bf16 (one split), else the normalised partial and its log-sum-exp
#pragma unroll
  for (int sl = 0; sl < 2; ++sl) {
    const int h = h0 + g + 8 * sl;
    if (h >= a.H) continue;
    const float inv = l_run[sl] > 0.f ? 1.f / l_run[sl] : 0.f;
    const size_t row = static_cast<size_t>(t) * a.H + h;
    if (a.splits == 1) {
#pragma unroll
      for (int dn = 0; dn < 16; ++dn)
        *reinterpret_cast<uint32_t *>(a.out + row * kHeadDim + 8 * dn + 2 * c) =
            pack_bf16x2(o[dn][2 * sl] * inv, o[dn][2 * sl + 1] * inv);
    } else {
      const size_t prow = static_cast<size_t>(split) * a.total_q * a.H + row;
#pragma unroll
      for (int dn = 0; dn < 16; ++dn)
        *reinterpret_cast<float2 *>(a.part_o + prow * kHeadDim + 8 * dn + 2 * c) =
            make_float2(o[dn][2 * sl] * inv, o[dn][2 * sl + 1] * inv);
      if (c == 0)
        a.part_lse[prow] =
            l_run[sl] > 0.f ? (m_run[sl] + log2f(l_run[sl])) * 0.69314718055994530942f
                            : -INFINITY;
    }
  }
}

}  // namespace

int latent_rows_per_cta() { return kLatRows; }
int latent_tile_positions() { return kLatTile; }

cudaError_t launch_latent_attention(const LatentArgs &a, cudaStream_t s) {
  const dim3 grid(a.total_q, (a.H + kLatRows - 1) / kLatRows, a.splits);
  constexpr size_t smem = kLatStages * (kLatTileBytes + kLatTile);
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(&latent_attn_kernel),
                                    static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  e = launch_pdl(latent_attn_kernel, grid, dim3(kLatThreads), smem, s, a);
  if (e != cudaSuccess || a.splits == 1) return e;
  return launch_combine(a.part_o, a.part_lse, a.splits, a.total_q, a.H, a.out, s);
}

}  // namespace msa
