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
//   warp 0     K producer: TMA loads of each block's K page tile (128-byte swizzle) into a
//              3-stage ring, freed as soon as the block's S is computed
//   warp 2     V producer: the V page tiles into a 2-stage ring, freed by the block's P V
//   warp 1     TMEM owner and MMA issuer (one thread): S = Q K^T (M = N = 128, K = 16 x 8) and
//              O += P V with P read from TMEM where the softmax left it (over its S) and V as
//              an N-major shared-memory operand; tcgen05.commit signals each
//   warps 4-11 softmax, two warpgroups taking alternate blocks (even / odd), each with its own
//              S buffer, O accumulator and running max and sum: one query row per thread (its
//              TMEM lane), one pass over the row's 128 scores held in registers (masked max,
//              exp2, P as bf16 back into TMEM over its S; the row sum adds the same rounded
//              P that the P V MMA reads, so that numerator and denominator weigh every
//              position alike).  The first warpgroup (producers, MMA
//              issuer, one idle warp) hands registers to the softmax warpgroups (setmaxnreg).
//              The groups never wait for each other inside the loop, so one group's
//              exponentials overlap the other's loads and maxima.  A group's
//              running max only moves when a block's max exceeds it by more than 2^8 (then its
//              O is rescaled in TMEM); in between P = 2^(s - m) stays <= 2^8, well inside bf16
//              and fp32 range.  Zeroes the rows of a last page past the sequence end in V
//              (0 * NaN is NaN).  Epilogue: the two groups' (m, l, O) merged by log-sum-exp,
//              O / l -> bf16, each group writing 64 of the 128 dims.
//
// TMEM columns: S/P of group 0 [0, 128) and group 1 [128, 256) (P of a block in the first 64
// columns of its S), O of group 0 [256, 384) and group 1 [384, 512).
#include <math.h>

#include "attn_common.cuh"

namespace msa {

namespace {

constexpr int kTcRows = 128;                     // MMA M: query rows of the tile
constexpr uint32_t kTcTile = 32768;              // one (page, head) bf16 tile
constexpr uint32_t kTcHalf = 16384;              // one swizzled [128][128 B] box
constexpr uint32_t kTc8Tile = 16384;             // one (page, head) e4m3 tile
constexpr int k8Stages = 2;                       // e4m3 staging tiles per operand (FP8 KV)
template <bool F8>
constexpr int k_stages() { return F8 ? 2 : 3; }   // K ring (f16 tiles for FP8 KV)
constexpr int kVStages = 2;
constexpr uint32_t kTcQBytes = 2 * kTcHalf;      // Q: 128 rows x 128 dims bf16
constexpr uint32_t kTcCols = 512;                // TMEM columns allocated
constexpr uint32_t kColO = 256;                  // + 128 per group
constexpr int kSoftWarps = 8;
constexpr int kSoftThreads = 32 * kSoftWarps;
constexpr int kVWarp = 2;
constexpr int kTcThreads = 32 * (4 + kSoftWarps);  // warpgroup 0: roles; 1 and 2: softmax
// Registers per thread after the split: the kernel is launched with kRegsLaunch per thread
// (384 threads, 65536 registers), warpgroup 0 gives up to kRegsRoles and the two softmax
// warpgroups take kRegsSoftmax; the split never asks for more than the launch holds (an
// increase waits until the registers are free, so a larger one would wait forever).
constexpr int kRegsLaunch = 168, kRegsRoles = 56, kRegsSoftmax = 224;
static_assert(128 * kRegsRoles + 256 * kRegsSoftmax <= kTcThreads * kRegsLaunch,
              "register split must fit in the launch's registers");
constexpr float kLazyLog2 = 8.f;                 // rescale only when the max grows by > 2^8

// FP8 KV adds the e4m3 staging tiles and keeps the epilogue's reduction buffers in the K
// staging (free by then); 225 KiB.
template <bool F8>
constexpr size_t tc_smem_bytes() {
  return 1024 + (k_stages<F8>() + kVStages) * kTcTile + (F8 ? 2 * k8Stages * kTc8Tile : 0) +
         kTcQBytes +
         (2 * k_stages<F8>() + 2 * kVStages + (F8 ? 4 * k8Stages : 0) + 2 * 3 + 1) *
             sizeof(uint64_t) +
         (F8 ? 0 : 2 * 2 * kTcRows * sizeof(float)) + 64;
}
static_assert(tc_smem_bytes<true>() <= 232448 && tc_smem_bytes<false>() <= 232448,
              "shared memory per CTA");

// S = Q K^T: A = Q (K-major, 128 rows), B = K tile (K-major, 128 positions), K = 128 dims.
// O += P V: A = P (TMEM), B = V tile (N-major: 128 dims contiguous in two 64-dim boxes 16 KiB
// apart; 8-position groups 1 KiB apart).
template <bool F8>
constexpr uint32_t idesc_qk() { return F8 ? umma_idesc_f16(128, 128, false) : umma_idesc_bf16(128, 128, false); }
template <bool F8>
constexpr uint32_t idesc_pv() { return F8 ? umma_idesc_f16(128, 128, true) : umma_idesc_bf16(128, 128, true); }

// Q rows (tok * G + head) as f16 in the MMA's K-major swizzled layout, dims in their natural
// order (the FP8-KV tiles: f16 operands; a q value outside f16's range is rounded as cvt does).
__device__ __forceinline__ void stage_q_f16(uint8_t *qs, const uint16_t *q, int t0, int rows,
                                            int G, int H_q, int g, int tid, int nthreads) {
  constexpr uint32_t sub = kTcRows * 128;
  for (int idx = tid; idx < kTcRows * 16; idx += nthreads) {
    const int r = idx >> 4, c = idx & 15;  // 8 dims (one 16-byte chunk) of row r
    uint4 o = make_uint4(0, 0, 0, 0);
    if (r < rows) {
      const int t = t0 + r / G, h = g * G + r % G;
      const uint4 x = *reinterpret_cast<const uint4 *>(
          q + (static_cast<size_t>(t) * H_q + h) * kHeadDim + c * 8);
      const float2 f0 = bf16x2_to_float2(x.x), f1 = bf16x2_to_float2(x.y);
      const float2 f2 = bf16x2_to_float2(x.z), f3 = bf16x2_to_float2(x.w);
      o = make_uint4(pack_f16x2(f0.x, f0.y), pack_f16x2(f1.x, f1.y), pack_f16x2(f2.x, f2.y),
                     pack_f16x2(f3.x, f3.y));
    }
    *reinterpret_cast<uint4 *>(qs + sw128(r, c, sub)) = o;
  }
}

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int kstep) {
  // 16 bf16 of K per step: steps 0-3 inside the first 64-column box, 4-7 in the second
  return umma_desc_sw128(base + (kstep >> 2) * kTcHalf + (kstep & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t nmajor_desc(uint32_t base, int kstep) {
  // 16 positions (rows) per step
  return umma_desc_sw128(base + kstep * 16 * 128, kTcHalf, 1024);
}
// TMEM column of P's 16-position K-slice `kstep` in group `w`'s S/P buffer
__device__ __forceinline__ uint32_t p_col(int w, int kstep) { return w * 128 + kstep * 8; }

template <bool F8>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const AttnArgs a) {
  constexpr int kKStages = k_stages<F8>();
  constexpr uint32_t kIdescQK = idesc_qk<F8>();
  constexpr uint32_t kIdescPV = idesc_pv<F8>();
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
  uint8_t *kst = smem;                                  // [3] K tiles
  uint8_t *vst = kst + kKStages * kTcTile;              // [2] V tiles
  uint8_t *k8st = vst + kVStages * kTcTile;             // FP8 KV: [2] e4m3 K tiles
  uint8_t *v8st = k8st + (F8 ? k8Stages * kTc8Tile : 0);  // FP8 KV: [2] e4m3 V tiles
  uint8_t *qs = v8st + (F8 ? k8Stages * kTc8Tile : 0);    // Q, K-major SW128
  uint64_t *k_full = reinterpret_cast<uint64_t *>(qs + kTcQBytes);
  uint64_t *k_empty = k_full + kKStages;
  uint64_t *v_full = k_empty + kKStages;
  uint64_t *v_empty = v_full + kVStages;
  uint64_t *k8_full = v_empty + kVStages;  // FP8 KV: staging tile landed / converted
  uint64_t *k8_empty = k8_full + (F8 ? k8Stages : 0);
  uint64_t *v8_full = k8_empty + (F8 ? k8Stages : 0);
  uint64_t *v8_empty = v8_full + (F8 ? k8Stages : 0);
  uint64_t *s_full = v8_empty + (F8 ? k8Stages : 0);  // [2 groups] S of the group's block
  uint64_t *p_full = s_full + 2;          // [2 groups] P of the group's block written
  uint64_t *o_done = p_full + 2;          // [2 groups] the group's P V done
  uint64_t *mma_done = o_done + 2;
  // [2 groups][128] each, for the epilogue (FP8 KV: in the K staging, free by then)
  float *red_m = F8 ? reinterpret_cast<float *>(k8st) : reinterpret_cast<float *>(mma_done + 1);
  float *red_l = red_m + 2 * kTcRows;
  uint32_t *tmem_base_s =
      reinterpret_cast<uint32_t *>(F8 ? reinterpret_cast<uint8_t *>(mma_done + 1)
                                      : reinterpret_cast<uint8_t *>(red_l + 2 * kTcRows));
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_base_s + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    if (F8)
      for (int s = 0; s < k8Stages; ++s) {
        mbar_init(&k8_full[s], 1);
        mbar_init(&k8_empty[s], 1);
        mbar_init(&v8_full[s], 1);
        mbar_init(&v8_empty[s], 1);
      }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&s_full[w], 1);
      mbar_init(&p_full[w], kSoftWarps / 2);
      mbar_init(&o_done[w], 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_s, kTcCols);
    tmem_relinquish();
  }
  // Q rows (tok * G + head) into shared memory in the MMA's K-major swizzled layout
  if constexpr (F8)
    stage_q_f16(qs, a.q, t0, rows, a.G, a.H_q, g, threadIdx.x, blockDim.x);
  else
    stage_q<false, kTcRows>(qs, a.q, t0, rows, a.G, a.H_q, g, threadIdx.x, blockDim.x);
  fence_async_shared();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_base_s;

  if (warp < 4) {
  // warpgroup 0: the roles, on few registers (each branch keeps its own budget to the end)
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsRoles));
  if (F8 && warp == 0) {
    // ============================================================== e4m3 K and V producer
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&vmap);
    }
    bool dead = false;
    uint32_t issued8[2] = {0u, 0u};  // K and V tiles given to the staging rings (lane 0)
    for (int base = 0; base < nblk && !dead; base += 32) {
      int j = -1, page = -1;
      if (base + lane < nblk) {
        j = list[base + lane];
        if (j >= 0 && j < a.max_blocks) page = a.table[static_cast<size_t>(b) * a.max_pages + j];
      }
      const int cnt = min(32, nblk - base);
      for (int k = 0; k < cnt && !dead; ++k) {
        const int jj = __shfl_sync(0xffffffffu, j, k);
        const int pg = __shfl_sync(0xffffffffu, page, k);
        if (lane == 0) {
          const int i = base + k;
          const int s8 = i % k8Stages;
          const bool jok = jj >= 0 && jj < a.max_blocks;
          const bool ok = jok && pg >= 0 && pg < a.num_pages;
          if (!ok) report(a.dev_err, jok ? MSA_DEVERR_PAGE_ID : MSA_DEVERR_BLOCK_ID);
          for (int op = 0; op < 2 && !dead; ++op) {  // K, then V
            uint64_t *full8 = op ? v8_full : k8_full, *empty8 = op ? v8_empty : k8_empty;
            uint8_t *dst = (op ? v8st : k8st) + s8 * kTc8Tile;
            if (i >= k8Stages && !mbar_wait(&empty8[s8], ((i / k8Stages) - 1) & 1, abort_flag)) {
              report(a.dev_err, MSA_DEVERR_TIMEOUT);
              *abort_flag = 1;
              dead = true;
            } else if (ok) {
              mbar_arrive_expect_tx(&full8[s8], kTc8Tile);
              tma_load_3d(dst, op ? &vmap : &kmap, &full8[s8], 0, 0, pg * a.H_kv + g);
              ++issued8[op];
            } else {
              // an unusable page: zeros, so that its block adds nothing (scores masked too)
              uint4 *z = reinterpret_cast<uint4 *>(dst);
              for (uint32_t w = 0; w < kTc8Tile / 16; ++w) z[w] = make_uint4(0, 0, 0, 0);
              fence_async_shared();
              mbar_arrive(&full8[s8]);
              ++issued8[op];
            }
          }
        }
        dead = __shfl_sync(0xffffffffu, dead, 0);
      }
    }
    // every tile load issued has landed before this warp exits
    if (lane == 0 && !(drain_ring(k8_full, k8Stages, issued8[0]) &&
                       drain_ring(v8_full, k8Stages, issued8[1])))
      report(a.dev_err, MSA_DEVERR_TIMEOUT);
  } else if (F8 && (warp == 2 || warp == 3)) {
    // ============================================================== e4m3 -> f16 converters
    // warp 3 converts K tiles, warp 2 V tiles, from the staging ring into the f16 ring in the
    // layout a TMA load of a bf16 tile gives (two 128-byte-swizzled 64-dim boxes); one cvt per
    // two codes, exact.
    const bool is_k = warp == 3;
    uint8_t *stg = is_k ? k8st : v8st;
    uint64_t *full8 = is_k ? k8_full : v8_full, *empty8 = is_k ? k8_empty : v8_empty;
    uint8_t *ring = is_k ? kst : vst;
    uint64_t *full = is_k ? k_full : v_full, *empty = is_k ? k_empty : v_empty;
    const int nst = is_k ? kKStages : kVStages;
    for (int i = 0; i < nblk; ++i) {
      const int s8 = i % k8Stages, s = i % nst;
      bool ok = mbar_wait(&full8[s8], (i / k8Stages) & 1, abort_flag);
      if (ok && i >= nst) ok = mbar_wait(&empty[s], ((i / nst) - 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) {
          report(a.dev_err, MSA_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const uint8_t *src = stg + s8 * kTc8Tile;
      uint8_t *dst = ring + s * kTcTile;
#pragma unroll 4
      for (int k = 0; k < 32; ++k) {
        const int task = lane + 32 * k, r = task >> 3, c = task & 7;  // 16 codes: dims 16c ..
        const uint4 x = *reinterpret_cast<const uint4 *>(src + sw128(r, c, kTc8Tile));
        uint4 lo, hi;
        e4m3x4_to_f16x2x2(x.x, lo.x, lo.y);
        e4m3x4_to_f16x2x2(x.y, lo.z, lo.w);
        e4m3x4_to_f16x2x2(x.z, hi.x, hi.y);
        e4m3x4_to_f16x2x2(x.w, hi.z, hi.w);
        *reinterpret_cast<uint4 *>(dst + sw128(r, 2 * c, kTcHalf)) = lo;
        *reinterpret_cast<uint4 *>(dst + sw128(r, 2 * c + 1, kTcHalf)) = hi;
      }
      fence_async_shared();  // the f16 tile, before the MMA (async proxy) reads it
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&full[s]);
        mbar_arrive(&empty8[s8]);
      }
    }
  } else if (!F8 && (warp == 0 || warp == kVWarp)) {
    // ============================================================== K or V producer
    const bool is_k = warp == 0;
    const CUtensorMap *map = is_k ? &kmap : &vmap;
    const int nst = is_k ? kKStages : kVStages;
    uint8_t *ring = is_k ? kst : vst;
    uint64_t *full = is_k ? k_full : v_full;
    uint64_t *empty = is_k ? k_empty : v_empty;
    if (lane == 0) prefetch_tmap(map);
    bool dead = false;
    uint32_t issued = 0;  // tiles given to the ring (lane 0)
    for (int base = 0; base < nblk && !dead; base += 32) {
      int j = -1, page = -1;
      if (base + lane < nblk) {
        j = list[base + lane];
        if (j >= 0 && j < a.max_blocks) page = a.table[static_cast<size_t>(b) * a.max_pages + j];
      }
      const int cnt = min(32, nblk - base);
      for (int k = 0; k < cnt; ++k) {
        const int jj = __shfl_sync(0xffffffffu, j, k);
        const int pg = __shfl_sync(0xffffffffu, page, k);
        if (lane == 0) {
          const int i = base + k;
          const int s = i % nst;
          if (i >= nst && !mbar_wait(&empty[s], ((i / nst) - 1) & 1, abort_flag)) {
            report(a.dev_err, MSA_DEVERR_TIMEOUT);
            *abort_flag = 1;
            dead = true;
          } else {
            const bool jok = jj >= 0 && jj < a.max_blocks;
            const bool ok = jok && pg >= 0 && pg < a.num_pages;
            if (ok) {
              mbar_arrive_expect_tx(&full[s], kTcTile);
              const int c2 = pg * a.H_kv + g;
              tma_load_3d(ring + s * kTcTile, map, &full[s], 0, 0, c2);
              tma_load_3d(ring + s * kTcTile + kTcHalf, map, &full[s], 64, 0, c2);
            } else {
              // an unusable page: the tile is filled with zeros so that its block adds
              // nothing (its scores are masked as well)
              if (is_k) report(a.dev_err, jok ? MSA_DEVERR_PAGE_ID : MSA_DEVERR_BLOCK_ID);
              uint4 *z = reinterpret_cast<uint4 *>(ring + s * kTcTile);
              for (uint32_t w = 0; w < kTcTile / 16; ++w) z[w] = make_uint4(0, 0, 0, 0);
              fence_async_shared();
              mbar_arrive(&full[s]);
            }
            ++issued;
          }
        }
        dead = __shfl_sync(0xffffffffu, dead, 0);
        if (dead) break;
      }
    }
    // every tile load issued has landed before this warp exits
    if (lane == 0 && !drain_ring(full, nst, issued)) report(a.dev_err, MSA_DEVERR_TIMEOUT);
  } else if (warp == 1) {
    // ============================================================== MMA issuer
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(qs);
      auto fail = [&]() {
        report(a.dev_err, MSA_DEVERR_TIMEOUT);
        *abort_flag = 1;
      };
      // S of block i into group (i & 1)'s buffer
      auto qk = [&](int i) -> bool {
        const int s = i % kKStages;
        if (!mbar_wait(&k_full[s], (i / kKStages) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(kst + s * kTcTile);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          umma_bf16_ss(tbase + (i & 1) * 128, kmajor_desc(q_addr, ks), kmajor_desc(k_addr, ks),
                       kIdescQK, ks > 0 ? 1u : 0u);
        umma_commit(&s_full[i & 1]);
        umma_commit(&k_empty[s]);
        return true;
      };
      // Event loop: the P V of the next block once its P (and V) is there, and the QK^T of the
      // next block once the P V that read its group's buffer is done, each in block order, so
      // that a QK^T never waits behind a P V that is not ready.  Every barrier's phases are
      // polled in order.  (Issuing per group out of block order measured slower: the groups
      // drift apart and the shared K ring serialises them anyway.)
      bool alive = qk(0) && (nblk < 2 || qk(1));
      int next_pv = 0, next_qk = 2;
      uint64_t t_idle = 0;
      uint32_t idle = 0;
      while (alive && next_pv < nblk) {
        bool progress = false;
        {
          const int i = next_pv, w = i & 1;
          if (mbar_try_wait(&p_full[w], (i >> 1) & 1) &&
              mbar_try_wait(&v_full[i % kVStages], (i / kVStages) & 1)) {
            tc_fence_after();
            const uint32_t v_addr = smem_u32(vst + (i % kVStages) * kTcTile);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
              umma_bf16_ts(tbase + kColO + w * 128, tbase + p_col(w, ks),
                           nmajor_desc(v_addr, ks), kIdescPV, (i >= 2 || ks > 0) ? 1u : 0u);
            umma_commit(&o_done[w]);
            umma_commit(&v_empty[i % kVStages]);
            ++next_pv;
            progress = true;
          }
        }
        if (next_qk < nblk && next_qk - 2 < next_pv) {
          const int i = next_qk, w = i & 1;
          // the group's previous P V read P from the buffer this S overwrites
          if (mbar_try_wait(&o_done[w], ((i >> 1) - 1) & 1) &&
              mbar_try_wait(&k_full[i % kKStages], (i / kKStages) & 1)) {
            alive = qk(i);
            ++next_qk;
            progress = true;
          }
        }
        if (progress) {
          idle = 0;
        } else if ((++idle & 255) == 1) {
          const uint64_t now = global_timer_ns();
          if (idle == 1) t_idle = now;
          if (*abort_flag || now - t_idle > kWaitTimeoutNs) alive = false;
        }
      }
      if (!alive) fail();
      // every tcgen05 operation of this thread done before the TMEM is released (waited for
      // even after an abort: bounded in time only)
      umma_commit(mma_done);
      if (!mbar_wait(mma_done, 0, nullptr)) report(a.dev_err, MSA_DEVERR_TIMEOUT);
    }
    __syncwarp();
  }
  // warp 3: no role of its own (its registers went to the softmax warpgroups)
  } else {
    // ============================================================== softmax warpgroups
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    const int w = (warp - 4) >> 2;       // this group takes blocks w, w + 2, w + 4, ...
    const int quarter = warp & 3;        // TMEM lanes 32 * quarter .. + 31
    const int r = quarter * 32 + lane;   // this thread's query row
    const int gt = (warp - 4 - 4 * w) * 32 + lane;  // 0 .. 127 within the group
    const uint32_t lane_addr = tbase + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t s_addr = lane_addr + w * 128;
    const uint32_t o_addr = lane_addr + kColO + w * 128;
    const int tl = r / a.G;
    const bool valid = r < rows;
    const int prow = valid ? cl + tok0 + tl : -1;
    const uint32_t tbit = valid ? (1u << tl) : 0u;
    float m_run = -INFINITY, l_run = 0.f;
    // The block's id, token mask and page validity come from the plan and the page table
    // through a two-deep register pipeline, so that no load is waited for in the block that
    // issues it: the list entries of this group's block after next, and the page of its next.
    const int32_t *trow = a.table + static_cast<size_t>(b) * a.max_pages;
    auto list_at = [&](int i, int &j, uint32_t &msk) {
      j = i < nblk ? list[i] : -1;
      msk = i < nblk ? masks[i] : 0u;
    };
    auto page_of = [&](int j) { return (j >= 0 && j < a.max_blocks) ? trow[j] : -1; };
    int j_n, j_nn;
    uint32_t msk_n, msk_nn;
    list_at(w, j_n, msk_n);
    list_at(w + 2, j_nn, msk_nn);
    int pg_n = page_of(j_n);
    for (int i = w; i < nblk; i += 2) {
      const int j = j_n;
      const uint32_t msk = msk_n;
      const bool ok = pg_n >= 0 && pg_n < a.num_pages;
      j_n = j_nn;
      msk_n = msk_nn;
      pg_n = page_of(j_n);
      list_at(i + 4, j_nn, msk_nn);
      const bool live = mbar_wait(&s_full[w], (i >> 1) & 1, abort_flag);
      if (!live) {
        report(a.dev_err, MSA_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
      tc_fence_after();
      const bool use = live && ok && (msk & tbit);
      const int pos0 = j * kBlock;
      const int lim = prow - pos0;               // position e is visible iff e <= lim
      // Per warp, one of three paths (lanes of a warp are 32 / G tokens that selected
      // different blocks, so a per-lane choice would run both code paths):
      //   none   no row of the warp uses the block: P = 0, nothing else;
      //   plain  every row either does not use it or sees all 128 positions: no per-position
      //          mask (a row that does not use the block gets scale 0 and offset -inf, and its
      //          scores are finite: some row of the warp sees the whole block, so it lies below
      //          the sequence end);
      //   masked the diagonal blocks.
      const bool any_use = __any_sync(0xffffffffu, use);
      const bool plain = __all_sync(0xffffffffu, !use || lim >= kBlock - 1);
      // After its first block a row's unmasked blocks take their exponentials against the
      // running max straight away: with the lazy rescale the block max matters only when it
      // exceeds the running max by more than 2^8, which the block's sum then shows (a term
      // above 2^8, or an infinite one); only then is the max computed and the block taken again.
      // (BF16 KV only: the FP8 kernel's conversion warps leave no registers for it.)
      const bool fast = !F8 && plain && __all_sync(0xffffffffu, !use || m_run > -INFINITY);
      uint32_t v[128];  // the row's 128 scores
      if (any_use) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(s_addr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(v + 32 * c));
        tmem_wait_ld();
      }
      float alpha = 1.f;
      float lblk = 0.f;  // the block's sum of P
#pragma unroll 1
      for (int pass = fast ? 0 : 1; pass < 2; ++pass) {
        if (pass == 1) {
          if (fast) tmem_wait_st();  // the fast pass's P, before it is written again
          float m8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) m8[k] = -INFINITY;
          if (any_use) {
            // row max (independent chains; three-input max where no position is masked)
            if (plain) {
#pragma unroll
              for (int e = 0; e < 128; e += 8)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  m8[k] = fmax3(m8[k], __uint_as_float(v[e + 2 * k]),
                                __uint_as_float(v[e + 2 * k + 1]));
            } else {
#pragma unroll
              for (int e = 0; e < 128; ++e)
                if (use && e <= lim) m8[e & 7] = fmaxf(m8[e & 7], __uint_as_float(v[e]));
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) m8[k] = fmaxf(m8[k], m8[k + 4]);
          }
          const float mrow = fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3]));
          const float mb = use ? mrow * a.scale_log2 : -INFINITY;
          const float m_cand = fmaxf(m_run, mb);
          if (m_cand > m_run + kLazyLog2) {  // also the first visible block (m_run = -inf)
            alpha = fast_exp2(m_run - m_cand);
            m_run = m_cand;
          }
        }
        // x = s * sc + nb: P = 2^(scale log2e S - m) where the row uses the block, else 0
        const float sc = use ? a.scale_log2 : 0.f;
        const float nb = use ? -m_run : -INFINITY;
        float ps4[4] = {0.f, 0.f, 0.f, 0.f};
        float2 ps2[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
        if (!any_use) {
          uint32_t z[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) z[e] = 0u;
          tmem_st32(s_addr, z);
          tmem_st32(s_addr + 32, z);
        } else {
          // P as bf16 into TMEM over the first 64 columns of S (the scores were read already)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t pk[32];
            if (plain) {  // pairs on the packed fp32x2 pipe: one FMA and one add per pair
#pragma unroll
              for (int e = 0; e < 64; e += 2) {
                const float2 x = fma2(make_float2(__uint_as_float(v[64 * h + e]),
                                                  __uint_as_float(v[64 * h + e + 1])),
                                      make_float2(sc, sc), make_float2(nb, nb));
                if constexpr (F8) {  // f16 P; its rounding (2^-11) is left out of the sum
                  const float e0 = fast_exp2(x.x), e1 = fast_exp2(x.y);
                  pk[e >> 1] = pack_f16x2(e0, e1);
                  ps2[(e >> 1) & 3] = add2(ps2[(e >> 1) & 3], make_float2(e0, e1));
                } else {
                  const uint32_t pb = pack_bf16x2(fast_exp2(x.x), fast_exp2(x.y));
                  pk[e >> 1] = pb;
                  ps2[(e >> 1) & 3] = add2(ps2[(e >> 1) & 3], bf16x2_to_float2(pb));
                }
              }
            } else {
#pragma unroll
              for (int e = 0; e < 64; e += 2) {
                const int pe = 64 * h + e;
                const float x0 = (use && pe <= lim) ? fmaf(__uint_as_float(v[pe]), sc, nb)
                                                    : -INFINITY;
                const float x1 = (use && pe + 1 <= lim)
                                     ? fmaf(__uint_as_float(v[pe + 1]), sc, nb)
                                     : -INFINITY;
                const float e0 = fast_exp2(x0), e1 = fast_exp2(x1);
                const uint32_t pb = F8 ? pack_f16x2(e0, e1) : pack_bf16x2(e0, e1);
                pk[e >> 1] = pb;
                const float2 pf = F8 ? make_float2(e0, e1) : bf16x2_to_float2(pb);
                ps4[(e >> 1) & 3] += pf.x + pf.y;
              }
            }
            tmem_st32(s_addr + 32 * h, pk);
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) ps4[k] += ps2[k].x + ps2[k].y;
        lblk = (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
        // every term <= 2^8 on the fast pass, or the rows concerned take the block again
        if (pass == 0 && !__any_sync(0xffffffffu, use && !(lblk <= 256.f))) break;
      }
      l_run = l_run * alpha + lblk;
      // this group's previous P V (done before this block's S was written; waited here so
      // that every phase is observed in order) before its O is rescaled
      if (i >= 2 && !mbar_wait(&o_done[w], ((i >> 1) - 1) & 1, abort_flag)) {
        report(a.dev_err, MSA_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
      tc_fence_after();
      if (i >= 2 && __any_sync(0xffffffffu, alpha < 1.f)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(o_addr + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 r = mul2(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])),
                                  make_float2(alpha, alpha));
            o[e] = __float_as_uint(r.x);
            o[e + 1] = __float_as_uint(r.y);
          }
          tmem_st32(o_addr + c * 32, o);
        }
      }
      tmem_wait_st();
      // positions past the sequence end in a last page: V rows there become zeros.  The V
      // tile of block i has landed, or is the next phase of its barrier to complete: V(i + 2)
      // waits for this block's P V, and V(i - 2) was read by a P V already waited for.
      if (pos0 + kBlock > L && live && ok) {
        const int first = max(L - pos0, 0);
        if (!mbar_wait(&v_full[i % kVStages], (i / kVStages) & 1, abort_flag)) {
          report(a.dev_err, MSA_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
        uint8_t *vt = vst + (i % kVStages) * kTcTile;
        for (int idx = gt; idx < (kBlock - first) * 16; idx += 128) {
          const int rr = first + idx / 16, ch = idx % 16;
          *reinterpret_cast<uint4 *>(vt + sw128(rr, ch, kTcHalf)) = make_uint4(0, 0, 0, 0);
        }
        fence_async_shared();  // the zeros, before the P V reads the tile
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[w]);
    }
    // ---- epilogue: the two groups merged by log-sum-exp, O / l, bf16 (group w: dims 64 w ..)
    const int nw = (nblk - w + 1) / 2;  // blocks this group took
    if (nw > 0 && !mbar_wait(&o_done[w], (nw - 1) & 1, abort_flag)) {
      report(a.dev_err, MSA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
    tc_fence_after();
    red_m[w * kTcRows + r] = m_run;
    red_l[w * kTcRows + r] = l_run;
    named_bar_sync(1, kSoftThreads);
    const float m0 = red_m[r], m1 = red_m[kTcRows + r];
    const float m = fmaxf(m0, m1);
    // a group with no block (nblk == 1) never wrote its O: its weight must be exactly 0
    const float f0 = m0 == -INFINITY ? 0.f : fast_exp2(m0 - m);
    const float f1 = (nblk < 2 || m1 == -INFINITY) ? 0.f : fast_exp2(m1 - m);
    const float l_tot = red_l[r] * f0 + red_l[kTcRows + r] * f1;
    const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
    const float g0 = f0 * inv, g1 = f1 * inv;
    const size_t orow = static_cast<size_t>(t0 + tl) * a.H_q + g * a.G + r % a.G;
    const uint32_t o0 = lane_addr + kColO + 64 * w, o1 = o0 + 128;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint32_t x0[32], x1[32];
      tmem_ld32(o0 + c * 32, x0);
      tmem_ld32(o1 + c * 32, x1);
      tmem_wait_ld();
      float y[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        // a zero weight contributes nothing, whatever the (possibly unwritten) O holds
        const float a0 = g0 != 0.f ? __uint_as_float(x0[e]) * g0 : 0.f;
        const float a1 = g1 != 0.f ? __uint_as_float(x1[e]) * g1 : 0.f;
        y[e] = a0 + a1;
      }
      if (valid) {
        uint4 *dst = reinterpret_cast<uint4 *>(a.out + orow * kHeadDim + 64 * w + c * 32);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          dst[q4] = make_uint4(pack_bf16x2(y[8 * q4 + 0], y[8 * q4 + 1]),
                               pack_bf16x2(y[8 * q4 + 2], y[8 * q4 + 3]),
                               pack_bf16x2(y[8 * q4 + 4], y[8 * q4 + 5]),
                               pack_bf16x2(y[8 * q4 + 6], y[8 * q4 + 7]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kTcCols);
}

template <bool F8>
cudaError_t launch_tc(const CUtensorMap &kmap, const CUtensorMap &vmap, const AttnArgs &a,
                      cudaStream_t s) {
  // The register split is only valid for a launch with exactly kRegsLaunch registers per
  // thread (a larger split than the launch holds would wait forever): checked once per device.
  static int checked[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!checked[dev]) {
    cudaFuncAttributes fa;
    cudaError_t e =
        cudaFuncGetAttributes(&fa, reinterpret_cast<const void *>(&attn_tc_kernel<F8>));
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kRegsLaunch || fa.maxThreadsPerBlock < kTcThreads)
      return cudaErrorInvalidConfiguration;
    checked[dev] = 1;
  }
  const size_t smem = tc_smem_bytes<F8>();
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(&attn_tc_kernel<F8>),
                                    static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(a.batch * a.tiles, a.H_kv);
  return launch_pdl(attn_tc_kernel<F8>, grid, dim3(kTcThreads), smem, s, kmap, vmap, a);
}

}  // namespace

bool attention_tc_supported(int G, int qt) { return qt * G <= kTcRows && qt <= 32; }

cudaError_t launch_attention_tc(const CUtensorMap &kmap, const CUtensorMap &vmap,
                                const AttnArgs &a, bool fp8, cudaStream_t s) {
  return fp8 ? launch_tc<true>(kmap, vmap, a, s) : launch_tc<false>(kmap, vmap, a, s);
}

}  // namespace msa
