// attention_tc.cu — stage 3 for prefill on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// ferrox-core "Module block_sparse": an ordinary masked pass over the positions the selected
// blocks cover (ascending, causally clipped).  Mojo module "msa", "Three attention routes":
// above 8 new tokens the step is a prefill driven by a device-built CSR of the selected
// blocks, with each token's causal diagonal at cache_lengths[b] + its index; BF16 operands,
// FP32 accumulation.
//
// One CTA per (sequence, query tile, KV head).  The tile's 128 rows are 128 / G tokens x the
// KV head's G query heads (the MMA's M = 128); the CTA walks the tile's union of selected
// blocks (plan.cu) once and every token keeps only the blocks it selected itself.
//
//   warp 0    producer: TMA loads of each block's K and V page tiles (128-byte swizzle) into a
//             2-stage ring
//   warp 1    TMEM owner and MMA issuer (one thread): S = Q K^T into one of two TMEM S
//             buffers (M = N = 128, K = 16 x 8), then O += P V into the TMEM O accumulator
//             (P from shared memory, V as an N-major operand); tcgen05.commit signals each
//   warps 2-5 softmax: one query row per thread (its TMEM lane); masks, online softmax in
//             the exp2 domain, P as bf16 into shared memory (the MMA's K-major 128-byte
//             swizzled layout), O rescaled in TMEM only when a row's max grew; zeroes the
//             rows of a last page past the sequence end in V (0 * NaN is NaN); epilogue
//             O / l -> bf16.
//
// TMEM columns: S buffers [0, 128) and [128, 256), O [256, 384) of a 512-column allocation.
#include <math.h>

#include "attn_common.cuh"

namespace msa {

namespace {

constexpr int kTcRows = 128;                     // MMA M: query rows of the tile
constexpr uint32_t kTcTile = 32768;              // one (page, head) bf16 tile
constexpr uint32_t kTcHalf = 16384;              // one swizzled [128][128 B] box
constexpr int kTcStages = 2;
constexpr uint32_t kTcStage = 2 * kTcTile;       // K + V
constexpr uint32_t kTcQBytes = 2 * kTcHalf;      // Q: 128 rows x 128 dims bf16
constexpr uint32_t kTcPBytes = 2 * kTcHalf;      // P: 128 rows x 128 positions bf16
constexpr uint32_t kTcCols = 512;                // TMEM columns allocated
constexpr uint32_t kColS0 = 0, kColO = 256;
constexpr int kTcThreads = 6 * 32;

constexpr size_t tc_smem_bytes() {
  return 1024 + kTcStages * kTcStage + kTcQBytes + kTcPBytes +
         (2 * kTcStages + 2 + 2 + 1 + 1 + 1) * sizeof(uint64_t) + kTcStages * 3 * sizeof(int) + 64;
}

// S = Q K^T: A = Q (K-major, 128 rows), B = K tile (K-major, 128 positions), K = 128 dims.
// O += P V: A = P (K-major, 128 rows, K = 128 positions), B = V tile (N-major: 128 dims
// contiguous in two 64-dim boxes 16 KiB apart; 8-position groups 1 KiB apart).
constexpr uint32_t kIdescQK = umma_idesc_bf16(128, 128, false);
constexpr uint32_t kIdescPV = umma_idesc_bf16(128, 128, true);

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int kstep) {
  // 16 bf16 of K per step: steps 0-3 inside the first 64-column box, 4-7 in the second
  return umma_desc_sw128(base + (kstep >> 2) * kTcHalf + (kstep & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t nmajor_desc(uint32_t base, int kstep) {
  // 16 positions (rows) per step
  return umma_desc_sw128(base + kstep * 16 * 128, kTcHalf, 1024);
}

__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const AttnArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  const int b = blockIdx.x / a.tiles, tile = blockIdx.x % a.tiles;
  const bool reporter = threadIdx.x == 0 && g == 0 && tile == 0;

  const int row0 = a.row_off[b];
  int q_len = a.row_off[b + 1] - row0;
  if (q_len < 0 || q_len > a.max_q_len) {
    if (reporter) report(a.dev_err, MSA_DEVERR_LENGTHS);
    q_len = q_len < 0 ? 0 : a.max_q_len;
  }
  const int tok0 = tile * a.qt;
  if (tok0 >= q_len) return;
  const int ntok = min(a.qt, q_len - tok0);
  const int rows = ntok * a.G;
  const int t0 = row0 + tok0;
  int cl = a.cache_len[b];
  if (cl < 0) {
    if (reporter) report(a.dev_err, MSA_DEVERR_LENGTHS);
    cl = 0;
  }
  const int L = cl + q_len;
  const size_t item = static_cast<size_t>(blockIdx.x) * a.H_kv + g;
  const int32_t *list = a.plan_list + item * a.cap;
  const uint32_t *masks = a.plan_masks + item * a.cap;
  const int nblk = min(max(a.plan_counts[item], 0), a.cap);

  if (nblk == 0) {  // a tile whose tokens selected nothing: invalid selection input
    if (threadIdx.x == 0) report(a.dev_err, MSA_DEVERR_NUM_SELECTED);
    for (int idx = threadIdx.x; idx < rows * (kHeadDim / 4); idx += blockDim.x) {
      const int r = idx / (kHeadDim / 4), d4 = idx % (kHeadDim / 4);
      const size_t orow = static_cast<size_t>(t0 + r / a.G) * a.H_q + g * a.G + r % a.G;
      reinterpret_cast<uint2 *>(a.out + orow * kHeadDim)[d4] = make_uint2(0, 0);
    }
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;                               // [2][K 32 KiB | V 32 KiB]
  uint8_t *qs = stages + kTcStages * kTcStage;          // Q, K-major SW128
  uint8_t *ps = qs + kTcQBytes;                         // P, K-major SW128
  uint64_t *kv_full = reinterpret_cast<uint64_t *>(ps + kTcPBytes);
  uint64_t *kv_empty = kv_full + kTcStages;
  uint64_t *s_full = kv_empty + kTcStages;  // [2]
  uint64_t *s_free = s_full + 2;            // [2]
  uint64_t *p_full = s_free + 2;
  uint64_t *o_done = p_full + 1;
  uint64_t *mma_done = o_done + 1;
  int *st_j = reinterpret_cast<int *>(mma_done + 1);
  uint32_t *st_mask = reinterpret_cast<uint32_t *>(st_j + kTcStages);
  int *st_ok = reinterpret_cast<int *>(st_mask + kTcStages);
  uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(st_ok + kTcStages);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_base_s + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);  // one arrival per softmax warp
    }
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_s, kTcCols);
    tmem_relinquish();
  }
  // Q rows (tok * G + head) into shared memory in the MMA's K-major swizzled layout
  stage_q<false, kTcRows>(qs, a.q, t0, rows, a.G, a.H_q, g, threadIdx.x, blockDim.x);
  fence_async_shared();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_base_s;

  if (warp == 0) {
    // ============================================================== producer
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&vmap);
    }
    bool dead = false;
    for (int base = 0; base < nblk && !dead; base += 32) {
      int j = -1, page = -1;
      uint32_t msk = 0u;
      if (base + lane < nblk) {
        j = list[base + lane];
        msk = masks[base + lane];
        if (j >= 0 && j < a.max_blocks) page = a.table[static_cast<size_t>(b) * a.max_pages + j];
      }
      const int cnt = min(32, nblk - base);
      for (int k = 0; k < cnt; ++k) {
        const int jj = __shfl_sync(0xffffffffu, j, k);
        const int pg = __shfl_sync(0xffffffffu, page, k);
        const uint32_t mm = __shfl_sync(0xffffffffu, msk, k);
        if (lane == 0) {
          const int i = base + k;
          const int s = i % kTcStages;
          if (i >= kTcStages &&
              !mbar_wait(&kv_empty[s], ((i / kTcStages) - 1) & 1, abort_flag)) {
            report(a.dev_err, MSA_DEVERR_TIMEOUT);
            *abort_flag = 1;
            dead = true;
          } else {
            const bool jok = jj >= 0 && jj < a.max_blocks;
            const bool ok = jok && pg >= 0 && pg < a.num_pages;
            st_j[s] = jj;
            st_mask[s] = mm;
            st_ok[s] = ok;
            if (ok) {
              mbar_arrive_expect_tx(&kv_full[s], kTcStage);
              const int c2 = pg * a.H_kv + g;
              uint8_t *kd = stages + s * kTcStage, *vd = kd + kTcTile;
              tma_load_3d(kd, &kmap, &kv_full[s], 0, 0, c2);
              tma_load_3d(kd + kTcHalf, &kmap, &kv_full[s], 64, 0, c2);
              tma_load_3d(vd, &vmap, &kv_full[s], 0, 0, c2);
              tma_load_3d(vd + kTcHalf, &vmap, &kv_full[s], 64, 0, c2);
            } else {
              // an unusable page: the stage is filled with zeros so that its block adds
              // nothing (its scores are masked below as well)
              report(a.dev_err, jok ? MSA_DEVERR_PAGE_ID : MSA_DEVERR_BLOCK_ID);
              uint4 *z = reinterpret_cast<uint4 *>(stages + s * kTcStage);
              for (uint32_t w = 0; w < kTcStage / 16; ++w) z[w] = make_uint4(0, 0, 0, 0);
              fence_async_shared();
              mbar_arrive(&kv_full[s]);
            }
          }
        }
        dead = __shfl_sync(0xffffffffu, dead, 0);
        if (dead) break;
      }
    }
  } else if (warp == 1) {
    // ============================================================== MMA issuer
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(qs), p_addr = smem_u32(ps);
      auto pv = [&](int jb) {
        if (!mbar_wait(p_full, jb & 1, abort_flag)) {
          report(a.dev_err, MSA_DEVERR_TIMEOUT);
          *abort_flag = 1;
          return;
        }
        tc_fence_after();
        const uint32_t v_addr = smem_u32(stages + (jb % kTcStages) * kTcStage + kTcTile);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          umma_bf16_ss(tbase + kColO, kmajor_desc(p_addr, ks), nmajor_desc(v_addr, ks), kIdescPV,
                       (jb > 0 || ks > 0) ? 1u : 0u);
        umma_commit(o_done);
        umma_commit(&kv_empty[jb % kTcStages]);
      };
      for (int i = 0; i < nblk && !*abort_flag; ++i) {
        const int s = i % kTcStages, sb = i & 1;
        if (!mbar_wait(&kv_full[s], (i / kTcStages) & 1, abort_flag) ||
            (i >= 2 && !mbar_wait(&s_free[sb], ((i >> 1) - 1) & 1, abort_flag))) {
          report(a.dev_err, MSA_DEVERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(stages + s * kTcStage);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          umma_bf16_ss(tbase + kColS0 + sb * 128, kmajor_desc(q_addr, ks),
                       kmajor_desc(k_addr, ks), kIdescQK, ks > 0 ? 1u : 0u);
        umma_commit(&s_full[sb]);
        if (i >= 1) pv(i - 1);
      }
      if (!*abort_flag) pv(nblk - 1);
      // every tcgen05 operation of this thread done before the TMEM is released
      umma_commit(mma_done);
      if (!mbar_wait(mma_done, 0, abort_flag)) report(a.dev_err, MSA_DEVERR_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ============================================================== softmax warps
    const int quarter = warp & 3;        // TMEM lanes 32 * quarter .. + 31
    const int r = quarter * 32 + lane;   // this thread's query row
    const uint32_t lane_addr = tbase + (static_cast<uint32_t>(quarter * 32) << 16);
    const int tl = r / a.G;
    const bool valid = r < rows;
    const int prow = valid ? cl + tok0 + tl : -1;
    const uint32_t tbit = valid ? (1u << tl) : 0u;
    float m_run = -INFINITY, l_run = 0.f;
    for (int i = 0; i < nblk; ++i) {
      const int s = i % kTcStages, sb = i & 1;
      bool live = mbar_wait(&kv_full[s], (i / kTcStages) & 1, abort_flag) &&
                  mbar_wait(&s_full[sb], (i >> 1) & 1, abort_flag);
      if (!live) {
        report(a.dev_err, MSA_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
      tc_fence_after();
      const int j = st_j[s];
      const uint32_t msk = st_mask[s];
      const bool use = live && st_ok[s] && (msk & tbit);
      const int pos0 = j * kBlock;
      // pass 1: row max over the visible positions of this block
      float mx = -INFINITY;
      const uint32_t s_addr = lane_addr + kColS0 + sb * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(s_addr + c * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (use && pos0 + c * 32 + e <= prow) mx = fmaxf(mx, __uint_as_float(v[e]));
      }
      const float m_new = fmaxf(m_run, mx * a.scale_log2);
      const float base = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = fast_exp2(m_run - base);  // 0 while nothing was visible
      // P must not be overwritten before the previous PV has read it
      if (i >= 1 && !mbar_wait(o_done, (i - 1) & 1, abort_flag)) {
        report(a.dev_err, MSA_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
      tc_fence_after();
      // pass 2: P = exp2(scale log2e S - m) as bf16 into the swizzled P tile
      float psum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(s_addr + c * 32, v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int p0 = pos0 + c * 32 + e;
          const float x0 = (use && p0 <= prow) ? __uint_as_float(v[e]) * a.scale_log2 - base
                                               : -INFINITY;
          const float x1 = (use && p0 + 1 <= prow)
                               ? __uint_as_float(v[e + 1]) * a.scale_log2 - base
                               : -INFINITY;
          const float e0 = fast_exp2(x0), e1 = fast_exp2(x1);
          psum += e0 + e1;
          pk[e >> 1] = pack_bf16x2(e0, e1);
        }
        // positions c*32 .. c*32+31 = four 16-byte chunks of row r
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int chunk = c * 4 + q4;  // 0..15 (8 positions each)
          *reinterpret_cast<uint4 *>(ps + sw128(r, chunk, kTcHalf)) =
              make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);  // S buffer may be overwritten
      l_run = l_run * alpha + psum;
      m_run = m_new;
      // O *= alpha where the row max grew (only once O holds something)
      if (i >= 1 && __any_sync(0xffffffffu, alpha < 1.f)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(lane_addr + kColO + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
          tmem_st32(lane_addr + kColO + c * 32, v);
        }
        tmem_wait_st();
      }
      // positions past the sequence end in a last page: V rows there become zeros
      if (pos0 + kBlock > L && live && st_ok[s]) {
        const int first = max(L - pos0, 0);
        uint8_t *vt = stages + s * kTcStage + kTcTile;
        for (int idx = quarter * 32 + lane; idx < (kBlock - first) * 16; idx += 128) {
          const int rr = first + idx / 16, ch = idx % 16;
          *reinterpret_cast<uint4 *>(vt + sw128(rr, ch, kTcHalf)) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_async_shared();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // ---- epilogue: O / l, bf16, into the ragged output
    if (!mbar_wait(o_done, (nblk - 1) & 1, abort_flag)) {
      report(a.dev_err, MSA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
    tc_fence_after();
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    const size_t orow = static_cast<size_t>(t0 + tl) * a.H_q + g * a.G + r % a.G;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t v[32];
      tmem_ld32(lane_addr + kColO + c * 32, v);
      tmem_wait_ld();
      if (valid) {
        uint4 *dst = reinterpret_cast<uint4 *>(a.out + orow * kHeadDim + c * 32);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          dst[q4] = make_uint4(
              pack_bf16x2(__uint_as_float(v[8 * q4 + 0]) * inv, __uint_as_float(v[8 * q4 + 1]) * inv),
              pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * inv, __uint_as_float(v[8 * q4 + 3]) * inv),
              pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * inv, __uint_as_float(v[8 * q4 + 5]) * inv),
              pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * inv, __uint_as_float(v[8 * q4 + 7]) * inv));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kTcCols);
}

}  // namespace

bool attention_tc_supported(int G, int qt) { return qt * G <= kTcRows && qt <= 32; }

cudaError_t launch_attention_tc(const CUtensorMap &kmap, const CUtensorMap &vmap,
                                const AttnArgs &a, cudaStream_t s) {
  const size_t smem = tc_smem_bytes();
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(&attn_tc_kernel),
                                    static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(a.batch * a.tiles, a.H_kv);
  return launch_pdl(attn_tc_kernel, grid, dim3(kTcThreads), smem, s, kmap, vmap, a);
}

}  // namespace msa
