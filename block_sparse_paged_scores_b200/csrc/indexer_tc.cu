// indexer_tc.cu — stage 1 for prefill on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// ferrox-core "Module block_sparse", "Four rules": a block's score is the MAX over its
// positions of the raw dot product q_idx . k_idx (no softmax scale), one index head per KV
// head.  With many new tokens per sequence the scores of a query tile against every visible
// page are a dense contraction, so they run on tcgen05: M = 128 rows (tile tokens x the
// index-query heads that read one index-K head), N = 128 positions of a page, K = 128 dims.
//
//   warp 0    producer: TMA loads of the tile's visible index-K pages (128-byte swizzle)
//             into a 4-stage ring
//   warp 1    TMEM owner and MMA issuer (one thread): S = Q_idx K_page^T into one of two TMEM
//             buffers; tcgen05.commit signals the scores
//   warps 2-5 one row per thread (its TMEM lane): the max of the row over the page's
//             positions up to the row's query position, written as the block's score; they
//             release the page's stage and S buffer once read.
#include <math.h>

#include "attn_common.cuh"

namespace msa {

namespace {

constexpr int kIxRows = 128;
constexpr uint32_t kIxTile = 32768;  // one (page, head) bf16 tile
constexpr uint32_t kIxHalf = 16384;  // one swizzled [128][128 B] box
constexpr int kIxStages = 4;
constexpr uint32_t kIxQBytes = 2 * kIxHalf;
constexpr uint32_t kIxCols = 256;  // two 128-column S buffers
constexpr int kIxThreads = 6 * 32;
constexpr uint32_t kIdescS = umma_idesc_bf16(128, 128, false);

constexpr size_t ix_smem_bytes() {
  return 1024 + kIxStages * kIxTile + kIxQBytes +
         (2 * kIxStages + 2 + 2 + 1) * sizeof(uint64_t) + kIxStages * sizeof(int) + 64;
}

__device__ __forceinline__ uint64_t ix_kdesc(uint32_t base, int kstep) {
  return umma_desc_sw128(base + (kstep >> 2) * kIxHalf + (kstep & 3) * 32, 16, 1024);
}

__global__ void __launch_bounds__(kIxThreads, 1)
    index_scores_tc_kernel(const __grid_constant__ CUtensorMap kmap, const IndexerArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x / a.tiles, tile = blockIdx.x % a.tiles;
  const int hk = blockIdx.y;
  const bool reporter = threadIdx.x == 0 && tile == 0 && hk == 0;

  const int row0 = a.row_off[b];
  int q_len = a.row_off[b + 1] - row0;
  if (q_len < 0 || q_len > a.max_q_len) {
    if (reporter) report(a.dev_err, MSA_DEVERR_LENGTHS);
    q_len = q_len < 0 ? 0 : a.max_q_len;
  }
  const int tok0 = tile * a.qt;
  if (tok0 >= q_len) return;
  const int ntok = min(a.qt, q_len - tok0);
  const int Hg = a.H_kv / a.H_idxk;
  const int rows = ntok * Hg;
  int cl = a.cache_len[b];
  if (cl < 0) {
    if (reporter) report(a.dev_err, MSA_DEVERR_LENGTHS);
    cl = 0;
  }
  int nb_last = (cl + tok0 + ntok - 1) / kBlock + 1;
  if (nb_last > a.max_blocks) {
    if (reporter) report(a.dev_err, MSA_DEVERR_LENGTHS);
    nb_last = a.max_blocks;
  }
  // blocks no token of the tile can see score -inf
  for (int idx = threadIdx.x; idx < rows * (a.max_blocks - nb_last); idx += blockDim.x) {
    const int nf = a.max_blocks - nb_last;
    const int r = idx / nf, j = nb_last + idx % nf;
    const int t = row0 + tok0 + r / Hg, g = hk + (r % Hg) * a.H_idxk;
    a.scores[(static_cast<size_t>(t) * a.H_kv + g) * a.max_blocks + j] = -INFINITY;
  }
  const int npages = nb_last;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;
  uint8_t *qs = stages + kIxStages * kIxTile;
  uint64_t *st_full = reinterpret_cast<uint64_t *>(qs + kIxQBytes);
  uint64_t *st_empty = st_full + kIxStages;
  uint64_t *s_full = st_empty + kIxStages;  // [2]
  uint64_t *s_free = s_full + 2;            // [2]
  uint64_t *mma_done = s_free + 2;
  int *st_ok = reinterpret_cast<int *>(mma_done + 1);
  uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(st_ok + kIxStages);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_base_s + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kIxStages; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 4);  // released by the row-max warps, after the MMA read it
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_s, kIxCols);
    tmem_relinquish();
  }
  // Q_idx rows r = tok * Hg + gi (index-query head hk + gi * H_idxk), K-major 128-byte swizzle
  for (int idx = threadIdx.x; idx < kIxRows * 16; idx += blockDim.x) {
    const int r = idx >> 4, chunk = idx & 15;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < rows) {
      const int t = row0 + tok0 + r / Hg, g = hk + (r % Hg) * a.H_idxk;
      v = reinterpret_cast<const uint4 *>(a.q_idx + (static_cast<size_t>(t) * a.H_kv + g) *
                                                        kHeadDim)[chunk];
    }
    *reinterpret_cast<uint4 *>(qs + sw128(r, chunk, kIxHalf)) = v;
  }
  fence_async_shared();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_base_s;

  if (warp == 0) {
    // ============================================================== producer
    if (lane == 0) prefetch_tmap(&kmap);
    bool dead = false;
    uint32_t issued = 0;  // pages given to the ring (lane 0)
    for (int base = 0; base < npages && !dead; base += 32) {
      const int pg_l = base + lane < npages
                           ? a.table[static_cast<size_t>(b) * a.max_pages + base + lane]
                           : -1;
      const int cnt = min(32, npages - base);
      for (int k = 0; k < cnt; ++k) {
        const int page = __shfl_sync(0xffffffffu, pg_l, k);
        if (lane == 0) {
          const int i = base + k;
          const int s = i % kIxStages;
          if (i >= kIxStages &&
              !mbar_wait(&st_empty[s], ((i / kIxStages) - 1) & 1, abort_flag)) {
            report(a.dev_err, MSA_DEVERR_TIMEOUT);
            *abort_flag = 1;
            dead = true;
          } else {
            const bool ok = page >= 0 && page < a.num_pages;
            st_ok[s] = ok;
            if (ok) {
              mbar_arrive_expect_tx(&st_full[s], kIxTile);
              const int c2 = page * a.H_idxk + hk;
              tma_load_3d(stages + s * kIxTile, &kmap, &st_full[s], 0, 0, c2);
              tma_load_3d(stages + s * kIxTile + kIxHalf, &kmap, &st_full[s], 64, 0, c2);
            } else {
              report(a.dev_err, MSA_DEVERR_PAGE_ID);
              mbar_arrive(&st_full[s]);
            }
            ++issued;
          }
        }
        dead = __shfl_sync(0xffffffffu, dead, 0);
        if (dead) break;
      }
    }
    // every tile load issued has landed before this warp exits
    if (lane == 0 && !drain_ring(st_full, kIxStages, issued))
      report(a.dev_err, MSA_DEVERR_TIMEOUT);
  } else if (warp == 1) {
    // ============================================================== MMA issuer
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(qs);
      for (int i = 0; i < npages && !*abort_flag; ++i) {
        const int s = i % kIxStages, sb = i & 1;
        if (!mbar_wait(&st_full[s], (i / kIxStages) & 1, abort_flag) ||
            (i >= 2 && !mbar_wait(&s_free[sb], ((i >> 1) - 1) & 1, abort_flag))) {
          report(a.dev_err, MSA_DEVERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(stages + s * kIxTile);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          umma_bf16_ss(tbase + sb * 128, ix_kdesc(q_addr, ks), ix_kdesc(k_addr, ks), kIdescS,
                       ks > 0 ? 1u : 0u);
        umma_commit(&s_full[sb]);
      }
      // every MMA done before the TMEM is released (even after an abort: bounded in time only)
      umma_commit(mma_done);
      if (!mbar_wait(mma_done, 0, nullptr)) report(a.dev_err, MSA_DEVERR_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ============================================================== row-max warps
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = tbase + (static_cast<uint32_t>(quarter * 32) << 16);
    const bool valid = r < rows;
    const int tl = r / Hg;
    const int prow = valid ? cl + tok0 + tl : -1;
    float *srow = valid ? a.scores + (static_cast<size_t>(row0 + tok0 + tl) * a.H_kv + hk +
                                      (r % Hg) * a.H_idxk) * a.max_blocks
                        : nullptr;
    for (int i = 0; i < npages; ++i) {
      const int s = i % kIxStages, sb = i & 1;
      const bool live = mbar_wait(&st_full[s], (i / kIxStages) & 1, abort_flag) &&
                        mbar_wait(&s_full[sb], (i >> 1) & 1, abort_flag);
      if (!live) {
        report(a.dev_err, MSA_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
      tc_fence_after();
      const bool use = live && st_ok[s];
      const int pos0 = i * kBlock;
      float mx = -INFINITY;
      uint32_t v[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_addr + sb * 128 + c * 32, v[c]);
      tmem_wait_ld();
      if (use && pos0 + kBlock - 1 <= prow) {
        // the whole page is visible to this row: four independent three-input max chains
        float m4[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          m4[c] = fmaxf(__uint_as_float(v[c][0]), __uint_as_float(v[c][1]));
#pragma unroll
          for (int e = 2; e < 32; e += 2)
            m4[c] = fmax3(m4[c], __uint_as_float(v[c][e]), __uint_as_float(v[c][e + 1]));
        }
        mx = fmax3(fmaxf(m4[0], m4[1]), m4[2], m4[3]);
      } else if (use) {  // the diagonal page: positions up to the row's own
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (pos0 + c * 32 + e <= prow) mx = fmaxf(mx, __uint_as_float(v[c][e]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&s_free[sb]);
        mbar_arrive(&st_empty[s]);  // the MMA finished with the page before S was signalled
      }
      if (valid) srow[i] = mx;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kIxCols);
}


// ---- the speculative route: positions as M
//
// With a few draft tokens per sequence a unit has at most 32 rows (tokens x the index-query
// heads of one index-K head), too few for M, and the row-major form above would be three
// quarters padding.  Here the operands are swapped: S^T = K_page Q_idx^T with M = the page's
// 128 positions, N = the unit's rows padded to NR = 32 (the route takes units of more than 16
// rows), K = 128 dims, so the MMAs work on little or no padding.  Each thread of the four epilogue warps holds one position (its TMEM lane) and the
// NR row values of it; the max over the page's positions is one warp reduction per row on
// order-preserving keys, then a max of the four warps' results through shared memory.  The
// grid is the warp-MMA kernel's: one CTA per (chunk of pages, unit), a unit's chunks launched
// together.
//
//   warp 0    producer: TMA loads of the chunk's pages into a kPosStages ring
//   warp 1    TMEM owner and MMA issuer (one thread): S^T into one of two NR-column buffers;
//             the commit frees the page's stage and signals the scores
//   warps 2-5 one position each: keys of the visible positions, the per-row warp max, and (one
//             warp per page, in turn) the block's scores
constexpr int kPosStages = 3;
constexpr uint32_t kPosCols = 64;  // two S^T buffers at columns 0 and 32

template <int NR>
constexpr size_t pos_smem_bytes() {
  return 1024 + kPosStages * kIxTile + 2 * NR * 128 +
         (2 * kPosStages + 2 + 2 + 1) * sizeof(uint64_t) + 2 * 4 * 32 * sizeof(uint32_t) + 64;
}

// the inverse of score_key
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

template <int NR>
__global__ void __launch_bounds__(kIxThreads)
    index_scores_pos_kernel(const __grid_constant__ CUtensorMap kmap, const IndexerArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cx = blockIdx.x % a.chunks;
  const int unit = blockIdx.x / a.chunks;  // (b * tiles + tile) * H_idxk + hk
  const int hk = unit % a.H_idxk, bt = unit / a.H_idxk;
  const int b = bt / a.tiles, tile = bt % a.tiles;
  const bool reporter = threadIdx.x == 0 && cx == 0 && tile == 0 && hk == 0;

  const int row0 = a.row_off[b];
  int q_len = a.row_off[b + 1] - row0;
  if (q_len < 0 || q_len > a.max_q_len) {
    if (reporter) report(a.dev_err, MSA_DEVERR_LENGTHS);
    q_len = q_len < 0 ? 0 : a.max_q_len;
  }
  const int tok0 = tile * a.qt;
  if (tok0 >= q_len) return;
  const int ntok = min(a.qt, q_len - tok0);
  const int Hg = a.H_kv / a.H_idxk;
  const int rows = min(ntok * Hg, NR);
  int cl = a.cache_len[b];
  if (cl < 0) {
    if (reporter) report(a.dev_err, MSA_DEVERR_LENGTHS);
    cl = 0;
  }
  int nb_last = (cl + tok0 + ntok - 1) / kBlock + 1;  // blocks visible to the tile's last token
  if (nb_last > a.max_blocks) {
    if (reporter) report(a.dev_err, MSA_DEVERR_LENGTHS);
    nb_last = a.max_blocks;
  }
  const int j0 = cx * a.chunk;
  const int j_end = min(j0 + a.chunk, a.max_blocks);
  const int j1 = min(j_end, nb_last);  // pages scored here: [j0, j1)
  {  // blocks of this chunk that no token of the tile can see score -inf
    const int f0 = max(j0, j1), nf = j_end - f0;
    for (int idx = threadIdx.x; idx < nf * rows; idx += blockDim.x) {
      const int r = idx / nf, j = f0 + idx % nf;
      const int t = row0 + tok0 + r / Hg, g = hk + (r % Hg) * a.H_idxk;
      a.scores[(static_cast<size_t>(t) * a.H_kv + g) * a.max_blocks + j] = -INFINITY;
    }
  }
  const int npages = j1 - j0;
  if (npages <= 0) return;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;
  uint8_t *qs = stages + kPosStages * kIxTile;  // [2 halves][NR rows][128 B], 1024-aligned
  uint64_t *st_full = reinterpret_cast<uint64_t *>(qs + 2 * NR * 128);
  uint64_t *st_empty = st_full + kPosStages;
  uint64_t *s_full = st_empty + kPosStages;  // [2]
  uint64_t *s_free = s_full + 2;             // [2]
  uint64_t *mma_done = s_free + 2;
  uint32_t *red = reinterpret_cast<uint32_t *>(mma_done + 1);  // [2][4 warps][32]
  uint32_t *tmem_base_s = red + 2 * 4 * 32;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_base_s + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPosStages; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 1);  // the MMA's commit: it has read the page
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);  // the epilogue warps, once their TMEM loads are done
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_s, kPosCols);
    tmem_relinquish();
  }
  // the rows' index queries (zeros past the unit's rows), K-major 128-byte swizzle
  const uint32_t qhalf = NR * 128;
  for (int idx = threadIdx.x; idx < NR * 16; idx += blockDim.x) {
    const int r = idx >> 4, chunk = idx & 15;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < rows) {
      const int t = row0 + tok0 + r / Hg, g = hk + (r % Hg) * a.H_idxk;
      v = reinterpret_cast<const uint4 *>(a.q_idx + (static_cast<size_t>(t) * a.H_kv + g) *
                                                        kHeadDim)[chunk];
    }
    *reinterpret_cast<uint4 *>(qs + sw128(r, chunk, qhalf)) = v;
  }
  fence_async_shared();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_base_s;
  const int32_t *trow = a.table + static_cast<size_t>(b) * a.max_pages + j0;

  if (warp == 0) {
    // ============================================================== producer
    if (lane == 0) prefetch_tmap(&kmap);
    bool dead = false;
    uint32_t issued = 0;  // pages given to the ring (lane 0)
    for (int base = 0; base < npages && !dead; base += 32) {
      const int pg_l = base + lane < npages ? trow[base + lane] : -1;
      const int cnt = min(32, npages - base);
      for (int k = 0; k < cnt; ++k) {
        const int page = __shfl_sync(0xffffffffu, pg_l, k);
        if (lane == 0) {
          const int i = base + k;
          const int s = i % kPosStages;
          if (i >= kPosStages &&
              !mbar_wait(&st_empty[s], ((i / kPosStages) - 1) & 1, abort_flag)) {
            report(a.dev_err, MSA_DEVERR_TIMEOUT);
            *abort_flag = 1;
            dead = true;
          } else {
            if (page >= 0 && page < a.num_pages) {
              mbar_arrive_expect_tx(&st_full[s], kIxTile);
              const int c2 = page * a.H_idxk + hk;
              tma_load_3d(stages + s * kIxTile, &kmap, &st_full[s], 0, 0, c2);
              tma_load_3d(stages + s * kIxTile + kIxHalf, &kmap, &st_full[s], 64, 0, c2);
            } else {  // the epilogue masks the page (it checks the page id itself)
              report(a.dev_err, MSA_DEVERR_PAGE_ID);
              mbar_arrive(&st_full[s]);
            }
            ++issued;
          }
        }
        dead = __shfl_sync(0xffffffffu, dead, 0);
        if (dead) break;
      }
    }
    // every tile load issued has landed before this warp exits
    if (lane == 0 && !drain_ring(st_full, kPosStages, issued))
      report(a.dev_err, MSA_DEVERR_TIMEOUT);
  } else if (warp == 1) {
    // ============================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(128, NR, false);
      const uint32_t q_addr = smem_u32(qs);
      for (int i = 0; i < npages && !*abort_flag; ++i) {
        const int s = i % kPosStages, sb = i & 1;
        if (!mbar_wait(&st_full[s], (i / kPosStages) & 1, abort_flag) ||
            (i >= 2 && !mbar_wait(&s_free[sb], ((i >> 1) - 1) & 1, abort_flag))) {
          report(a.dev_err, MSA_DEVERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(stages + s * kIxTile);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          umma_bf16_ss(tbase + sb * 32, ix_kdesc(k_addr, ks),
                       umma_desc_sw128(q_addr + (ks >> 2) * qhalf + (ks & 3) * 32, 16, 1024),
                       idesc, ks > 0 ? 1u : 0u);
        umma_commit(&s_full[sb]);
        umma_commit(&st_empty[s]);
      }
      // every MMA done before the TMEM is released (even after an abort: bounded in time only)
      umma_commit(mma_done);
      if (!mbar_wait(mma_done, 0, nullptr)) report(a.dev_err, MSA_DEVERR_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ============================================================== epilogue warps
    const int quarter = warp & 3;  // TMEM lanes (positions) 32 quarter .. + 31
    const int wq = warp - 2;
    const int p = quarter * 32 + lane;
    const uint32_t lane_addr = tbase + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t kNegInf = 0x007fffffu;  // score_key(-inf)
    const int prow0 = cl + tok0;           // the first token's position
    uint32_t okm = 0u;                     // pages base .. base + 31 with a usable page id
    for (int i = 0; i < npages; ++i) {
      const int sb = i & 1;
      if ((i & 31) == 0) {
        const int pg = i + lane < npages ? trow[i + lane] : -1;
        okm = __ballot_sync(0xffffffffu, pg >= 0 && pg < a.num_pages);
      }
      const bool live = mbar_wait(&s_full[sb], (i >> 1) & 1, abort_flag);
      if (!live) {
        report(a.dev_err, MSA_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32(lane_addr + sb * 32, v);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);
      const bool use = live && ((okm >> (i & 31)) & 1u);
      const int pos0 = (j0 + i) * kBlock;
      uint32_t key[NR];
      if (use && pos0 + kBlock - 1 <= prow0) {  // the whole page is visible to every row
#pragma unroll
        for (int c = 0; c < NR; ++c) key[c] = score_key(__uint_as_float(v[c]));
      } else {  // the diagonal page: positions up to each row's own token
#pragma unroll
        for (int c = 0; c < NR; ++c)
          key[c] = use && pos0 + p <= prow0 + c / Hg ? score_key(__uint_as_float(v[c])) : kNegInf;
      }
      uint32_t mine = kNegInf;  // lane c: row c's max over this warp's 32 positions
#pragma unroll
      for (int c = 0; c < NR; ++c) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, key[c]);
        if (lane == c) mine = m;
      }
      uint32_t *rb = red + sb * 4 * 32;
      rb[wq * 32 + lane] = mine;
      named_bar_sync(1, 4 * 32);
      if (wq == (i & 3) && lane < rows) {
        const uint32_t m = max(max(rb[lane], rb[32 + lane]), max(rb[64 + lane], rb[96 + lane]));
        const int t = row0 + tok0 + lane / Hg, g = hk + (lane % Hg) * a.H_idxk;
        a.scores[(static_cast<size_t>(t) * a.H_kv + g) * a.max_blocks + j0 + i] = key_score(m);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kPosCols);
}

}  // namespace

cudaError_t launch_index_scores_tc(const CUtensorMap &kidx_map, const IndexerArgs &a,
                                   cudaStream_t s) {
  const size_t smem = ix_smem_bytes();
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(&index_scores_tc_kernel),
                                    static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(a.batch * a.tiles, a.H_idxk);
  return launch_pdl(index_scores_tc_kernel, grid, dim3(kIxThreads), smem, s, kidx_map, a);
}


cudaError_t launch_index_scores_tc_pos(const CUtensorMap &kidx_map, const IndexerArgs &a,
                                       int chunks, cudaStream_t s) {
  auto go = [&](auto kernel, size_t smem) -> cudaError_t {
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(kernel),
                                      static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const dim3 grid(a.batch * a.tiles * a.H_idxk * chunks);
    return launch_pdl(kernel, grid, dim3(kIxThreads), smem, s, kidx_map, a);
  };
  if (a.qt * (a.H_kv / a.H_idxk) > 32) return cudaErrorInvalidValue;
  return go(&index_scores_pos_kernel<32>, pos_smem_bytes<32>());
}

}  // namespace msa
