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
//   warp 10    V producer: the V page tiles into a 2-stage ring, freed by the block's P V
//   warp 1     TMEM owner and MMA issuer (one thread): S = Q K^T into one of three TMEM S
//              buffers (M = N = 128, K = 16 x 8); O += P V with P read from TMEM where the
//              softmax left it (over its S) and V as an N-major shared-memory operand;
//              tcgen05.commit signals each
//   warps 2-9  softmax, two warpgroups: thread (row r, half h) owns positions 64 h .. 64 h + 63
//              of row r (its TMEM lane); one pass over S: masked partial max, the row max
//              through shared memory, exp2 in place, P as bf16 back into TMEM over the S it
//              came from.  The running max m only moves when a block's max exceeds it by more
//              than 2^8 (then O is rescaled in TMEM once the previous P V is done); in between
//              P = 2^(s - m) stays <= 2^8, well inside bf16 and fp32 range.  Zeroes
//              the rows of a last page past the sequence end in V (0 * NaN is NaN); epilogue
//              O / l -> bf16, each half writing its 64 dims.
//
// TMEM columns: S/P buffers [0, 128), [128, 256), [256, 384); O [384, 512).  P of buffer b
// holds positions 0-63 in columns 128 b + [0, 32) and 64-127 in 128 b + [64, 96).
#include <math.h>

#include "attn_common.cuh"

namespace msa {

namespace {

constexpr int kTcRows = 128;                     // MMA M: query rows of the tile
constexpr uint32_t kTcTile = 32768;              // one (page, head) bf16 tile
constexpr uint32_t kTcHalf = 16384;              // one swizzled [128][128 B] box
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr uint32_t kTcQBytes = 2 * kTcHalf;      // Q: 128 rows x 128 dims bf16
constexpr uint32_t kTcCols = 512;                // TMEM columns allocated
constexpr int kSBufs = 3;
constexpr uint32_t kColO = 384;
constexpr int kSoftWarps = 8;
constexpr int kSoftThreads = 32 * kSoftWarps;
constexpr int kVWarp = 2 + kSoftWarps;
constexpr int kTcThreads = 32 * (3 + kSoftWarps);
constexpr float kLazyLog2 = 8.f;                 // rescale only when the max grows by > 2^8

constexpr size_t tc_smem_bytes() {
  return 1024 + (kKStages + kVStages) * kTcTile + kTcQBytes +
         (2 * kKStages + 2 * kVStages + 2 * kSBufs + 3) * sizeof(uint64_t) +
         (2 * 2 * kTcRows + 2 * kTcRows) * sizeof(float) + 64;
}

// S = Q K^T: A = Q (K-major, 128 rows), B = K tile (K-major, 128 positions), K = 128 dims.
// O += P V: A = P (TMEM), B = V tile (N-major: 128 dims contiguous in two 64-dim boxes 16 KiB
// apart; 8-position groups 1 KiB apart).
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
// TMEM column of P's 16-position K-slice `kstep` in S/P buffer `buf`
__device__ __forceinline__ uint32_t p_col(int buf, int kstep) {
  return buf * 128 + (kstep >> 2) * 64 + (kstep & 3) * 8;
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
  uint8_t *kst = smem;                                  // [3] K tiles
  uint8_t *vst = kst + kKStages * kTcTile;              // [2] V tiles
  uint8_t *qs = vst + kVStages * kTcTile;               // Q, K-major SW128
  uint64_t *k_full = reinterpret_cast<uint64_t *>(qs + kTcQBytes);
  uint64_t *k_empty = k_full + kKStages;
  uint64_t *v_full = k_empty + kKStages;
  uint64_t *v_empty = v_full + kVStages;
  uint64_t *s_full = v_empty + kVStages;  // [3] S of the buffer written
  uint64_t *s_free = s_full + kSBufs;     // [3] the P V that read the buffer's P is done
  uint64_t *p_full = s_free + kSBufs;
  uint64_t *o_done = p_full + 1;
  uint64_t *mma_done = o_done + 1;
  float *red_m = reinterpret_cast<float *>(mma_done + 1);  // [2 parity][2 halves][128]
  float *red_l = red_m + 2 * 2 * kTcRows;                  // [2 halves][128]
  uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(red_l + 2 * kTcRows);
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
    for (int s = 0; s < kSBufs; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 1);
    }
    mbar_init(p_full, kSoftWarps);
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

  if (warp == 0 || warp == kVWarp) {
    // ============================================================== K or V producer
    const bool is_k = warp == 0;
    const CUtensorMap *map = is_k ? &kmap : &vmap;
    const int nst = is_k ? kKStages : kVStages;
    uint8_t *ring = is_k ? kst : vst;
    uint64_t *full = is_k ? k_full : v_full;
    uint64_t *empty = is_k ? k_empty : v_empty;
    if (lane == 0) prefetch_tmap(map);
    bool dead = false;
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
          }
        }
        dead = __shfl_sync(0xffffffffu, dead, 0);
        if (dead) break;
      }
    }
  } else if (warp == 1) {
    // ============================================================== MMA issuer
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(qs);
      auto pv = [&](int jb) {
        if (!mbar_wait(p_full, jb & 1, abort_flag) ||
            !mbar_wait(&v_full[jb % kVStages], (jb / kVStages) & 1, abort_flag)) {
          report(a.dev_err, MSA_DEVERR_TIMEOUT);
          *abort_flag = 1;
          return;
        }
        tc_fence_after();
        const int pb = jb % kSBufs;
        const uint32_t v_addr = smem_u32(vst + (jb % kVStages) * kTcTile);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          umma_bf16_ts(tbase + kColO, tbase + p_col(pb, ks), nmajor_desc(v_addr, ks), kIdescPV,
                       (jb > 0 || ks > 0) ? 1u : 0u);
        umma_commit(&s_free[pb]);
        umma_commit(&v_empty[jb % kVStages]);
        umma_commit(o_done);
      };
      for (int i = 0; i < nblk && !*abort_flag; ++i) {
        const int s = i % kKStages, sb = i % kSBufs;
        if (!mbar_wait(&k_full[s], (i / kKStages) & 1, abort_flag) ||
            (i >= kSBufs && !mbar_wait(&s_free[sb], ((i / kSBufs) - 1) & 1, abort_flag))) {
          report(a.dev_err, MSA_DEVERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(kst + s * kTcTile);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          umma_bf16_ss(tbase + sb * 128, kmajor_desc(q_addr, ks), kmajor_desc(k_addr, ks),
                       kIdescQK, ks > 0 ? 1u : 0u);
        umma_commit(&s_full[sb]);
        umma_commit(&k_empty[s]);
        if (i >= 1) pv(i - 1);
      }
      if (!*abort_flag) pv(nblk - 1);
      // every tcgen05 operation of this thread done before the TMEM is released
      umma_commit(mma_done);
      if (!mbar_wait(mma_done, 0, abort_flag)) report(a.dev_err, MSA_DEVERR_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ============================================================== softmax warpgroups
    const int half = (warp - 2) >> 2;    // positions / dims 64 half .. 64 half + 63
    const int quarter = warp & 3;        // TMEM lanes 32 * quarter .. + 31
    const int r = quarter * 32 + lane;   // this thread's query row
    const int st = (warp - 2) * 32 + lane;  // 0 .. 255
    const uint32_t lane_addr = tbase + (static_cast<uint32_t>(quarter * 32) << 16);
    const int tl = r / a.G;
    const bool valid = r < rows;
    const int prow = valid ? cl + tok0 + tl : -1;
    const uint32_t tbit = valid ? (1u << tl) : 0u;
    float m_run = -INFINITY, l_run = 0.f;
    // the block's id, token mask and page validity, read one block ahead from the plan
    auto block_meta = [&](int i, int &j, uint32_t &msk, bool &ok) {
      j = -1, msk = 0u, ok = false;
      if (i < nblk) {
        j = list[i];
        msk = masks[i];
        if (j >= 0 && j < a.max_blocks) {
          const int pg = a.table[static_cast<size_t>(b) * a.max_pages + j];
          ok = pg >= 0 && pg < a.num_pages;
        }
      }
    };
    int nj;
    uint32_t nmsk;
    bool nok;
    block_meta(0, nj, nmsk, nok);
    for (int i = 0; i < nblk; ++i) {
      const int sb = i % kSBufs;
      const int j = nj;
      const uint32_t msk = nmsk;
      const bool ok = nok;
      block_meta(i + 1, nj, nmsk, nok);
      const bool live = mbar_wait(&s_full[sb], (i / kSBufs) & 1, abort_flag);
      if (!live) {
        report(a.dev_err, MSA_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
      tc_fence_after();
      const bool use = live && ok && (msk & tbit);
      const int pos0 = j * kBlock + 64 * half;   // this thread's first position
      const int lim = prow - pos0;               // element e is visible iff e <= lim
      const bool full = use && lim >= 63;
      const uint32_t s_addr = lane_addr + sb * 128 + 64 * half;
      uint32_t v[64];
      tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(v));
      tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      tmem_wait_ld();
      // masked max over this half (eight independent chains), then the row's max through
      // shared memory
      float mx = -INFINITY;
      {
        float m8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) m8[k] = -INFINITY;
        if (full) {
#pragma unroll
          for (int e = 0; e < 64; ++e) m8[e & 7] = fmaxf(m8[e & 7], __uint_as_float(v[e]));
        } else if (use) {
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (e <= lim) m8[e & 7] = fmaxf(m8[e & 7], __uint_as_float(v[e]));
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) m8[k] = fmaxf(m8[k], m8[k + 4]);
        mx = fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3]));
      }
      float *rm = red_m + (i & 1) * 2 * kTcRows;
      rm[half * kTcRows + r] = mx;
      named_bar_sync(1, kSoftThreads);
      const float mb = fmaxf(mx, rm[(half ^ 1) * kTcRows + r]) * a.scale_log2;
      const float m_cand = fmaxf(m_run, mb);
      float alpha = 1.f;
      if (m_cand > m_run + kLazyLog2) {  // also the first visible block (m_run = -inf)
        alpha = fast_exp2(m_run - m_cand);
        m_run = m_cand;
      }
      const float nbase = m_run == -INFINITY ? 0.f : -m_run;
      // P = 2^(scale log2e S - m) as bf16 into TMEM over this half's S (four sum chains)
      float ps4[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[32];
      if (full) {
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const float e0 = fast_exp2(fmaf(__uint_as_float(v[e]), a.scale_log2, nbase));
          const float e1 = fast_exp2(fmaf(__uint_as_float(v[e + 1]), a.scale_log2, nbase));
          ps4[(e >> 1) & 3] += e0 + e1;
          pk[e >> 1] = pack_bf16x2(e0, e1);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const float x0 = (use && e <= lim) ? fmaf(__uint_as_float(v[e]), a.scale_log2, nbase)
                                             : -INFINITY;
          const float x1 = (use && e + 1 <= lim)
                               ? fmaf(__uint_as_float(v[e + 1]), a.scale_log2, nbase)
                               : -INFINITY;
          const float e0 = fast_exp2(x0), e1 = fast_exp2(x1);
          ps4[(e >> 1) & 3] += e0 + e1;
          pk[e >> 1] = pack_bf16x2(e0, e1);
        }
      }
      const float psum = (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
      tmem_st32(s_addr, pk);
      l_run = l_run * alpha + psum;
      // the previous P V must be done before O is rescaled (and, every block, so that the
      // o_done phases are waited in order)
      if (i >= 1 && !mbar_wait(o_done, (i - 1) & 1, abort_flag)) {
        report(a.dev_err, MSA_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
      tc_fence_after();
      if (i >= 1 && __any_sync(0xffffffffu, alpha < 1.f)) {
        const uint32_t o_addr = lane_addr + kColO + 64 * half;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t o[32];
          tmem_ld32(o_addr + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(o_addr + c * 32, o);
        }
      }
      tmem_wait_st();
      // positions past the sequence end in a last page: V rows there become zeros.  The V
      // tile of block i has landed, or is the next phase of its barrier to complete: V(i + 2)
      // waits for this block's P V, and V(i - 2) was read by a P V already waited for.
      const int bpos = j * kBlock;
      if (bpos + kBlock > L && live && ok) {
        const int first = max(L - bpos, 0);
        if (!mbar_wait(&v_full[i % kVStages], (i / kVStages) & 1, abort_flag)) {
          report(a.dev_err, MSA_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
        uint8_t *vt = vst + (i % kVStages) * kTcTile;
        for (int idx = st; idx < (kBlock - first) * 16; idx += kSoftThreads) {
          const int rr = first + idx / 16, ch = idx % 16;
          *reinterpret_cast<uint4 *>(vt + sw128(rr, ch, kTcHalf)) = make_uint4(0, 0, 0, 0);
        }
        fence_async_shared();  // the zeros, before the P V reads the tile
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // ---- epilogue: O / l, bf16, into the ragged output (each half: its 64 dims)
    if (!mbar_wait(o_done, (nblk - 1) & 1, abort_flag)) {
      report(a.dev_err, MSA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
    tc_fence_after();
    red_l[half * kTcRows + r] = l_run;
    named_bar_sync(1, kSoftThreads);
    const float l_tot = red_l[r] + red_l[kTcRows + r];
    const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
    const size_t orow = static_cast<size_t>(t0 + tl) * a.H_q + g * a.G + r % a.G;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint32_t v[32];
      tmem_ld32(lane_addr + kColO + 64 * half + c * 32, v);
      tmem_wait_ld();
      if (valid) {
        uint4 *dst = reinterpret_cast<uint4 *>(a.out + orow * kHeadDim + 64 * half + c * 32);
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
