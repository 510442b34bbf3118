// indexer.cu — stage 1: block scores of the index-K cache.
//
// ferrox-core "Module block_sparse", "Four rules": a block's score is the MAX over its
// positions of the raw dot product (no softmax scale), and one index head scores for one KV
// head.  Mojo module "msa": the index-K cache is BF16 with a single head (the build also
// accepts one index-K head per KV head).
//
// One CTA scores a chunk of pages of one sequence for a tile of its query tokens and all the
// index-query heads that read one index-K head (rows = tokens x heads, at most 32).  A
// producer warp streams the 32 KiB page tiles with TMA (128-byte swizzle) through a ring of
// shared-memory stages; four consumer warps each take 32 of the 128 positions, compute
// S = Q K^T with bf16 mma.sync (fp32 accumulation), mask positions after each row's query
// position, reduce the row max with warp shuffles and then across the four warps through
// shared memory, and write one fp32 score per (row, page).
//
// Scaled index-K caches (TensorRT-LLM "DeepSeekSparseAttentionConfig", indexer_k_dtype): fp8
// (e4m3 codes, one fp32 scale per token) and fp4 (e2m1 code pairs, one UE8M0 exponent per 32
// elements).  The codes stream by TMA like the bf16 tile and the token's 512 bytes of scales by
// one bulk copy on the same barrier.  The consumers turn two codes into an f16 pair with one
// cvt and run f16 mma.sync against q_idx turned into f16 once per CTA (each row prescaled by a
// power of two that keeps it below 2^15, undone exactly on its scores).  The 128 dims are
// visited in an order of the consumers' own (the same on both operands, so the dot product is
// unchanged) in which a thread reads one 32-bit word of its position's codes per k-step, and
// in which every k-step of the fp4 layout stays inside one 32-element exponent group: each
// group's partial product is then scaled by its exponent, and an fp8 row by its token's scale,
// before the max.
//
// With the selection fused in (decode and speculative routes), the CTAs of one (sequence,
// tile, index-K head) count themselves out on a device counter once their scores are written;
// the last one runs stage 2 for the unit's rows (select_row.cuh, reading the scores from L2) and
// puts the counter back to zero, so no separate selection launch is needed.
#include <math.h>

#include "select_row.cuh"

namespace msa {

namespace {

// Ring depth: two 32 KiB stages (three CTAs per SM) for CTAs with a short chunk of pages, three
// (two CTAs per SM) for long ones: the same bytes in flight per SM, but more pages in process at
// once wins on short chunks, a deeper ring on long streams.
constexpr int kLongChunk = 32;  // pages per CTA from which the deeper ring is used
constexpr int kConsumerWarps = 4;
constexpr int kThreads = 32 * (kConsumerWarps + 1);

// Index-K formats (IndexerArgs::idx_fmt), one (page, head) tile each: bf16 32 KiB; fp8 16 KiB
// of codes + 128 fp32 scales; fp4 8 KiB of code pairs (viewed as 64 rows of 128 bytes: tokens
// 2r and 2r + 1 in row r) + 128 x 4 exponent bytes.
template <int IF>
constexpr uint32_t tile_bytes() {
  return IF == kIdxBf16 ? 32768u : (IF == kIdxFp8 ? 16384u : 8192u);
}
template <int IF>
constexpr uint32_t scale_bytes() { return IF == kIdxBf16 ? 0u : 512u; }
// Ring depth of the scaled formats: 3 fp8 / 6 fp4 stages (about 50 KiB), so that four CTAs fit
// on an SM (their registers allow four): more consumer warps to hide the conversion chains'
// latency, about the same bytes in flight as the bf16 ring.
template <int ST, int IF>
constexpr int ring_stages() { return IF == kIdxBf16 ? ST : (IF == kIdxFp8 ? 3 : 6); }

template <int kStages, int IF>
constexpr size_t smem_bytes() {
  return 1024 /*alignment slack*/ + kStages * (tile_bytes<IF>() + scale_bytes<IF>()) +
         2 * kStages * sizeof(uint64_t) + kStages * sizeof(int) +
         2 * kConsumerWarps * 32 * sizeof(float) + 16;
}

// First of the four dims of k-step ks that lane j (lane % 4) holds, in the scaled formats'
// visiting order: fp8 dims 16 ks + 4 j .. + 3 (one word of codes); fp4 dims 32 g + 8 j + 4 h
// .. + 3 for ks = 2 g + h (half a word of code pairs, inside exponent group g).  The first
// two of the four are the MMA's k slots 2j, 2j + 1, the last two 2j + 8, 2j + 9.
template <int IF>
__device__ __forceinline__ int scaled_dim(int ks, int j) {
  return IF == kIdxFp8 ? 16 * ks + 4 * j : 32 * (ks >> 1) + 8 * j + 4 * (ks & 1);
}

// 2^(x - 127) of a UE8M0 byte (0xFF: NaN)
__device__ __forceinline__ float ue8m0_to_float(uint32_t x) {
  return x == 0xFFu ? __uint_as_float(0x7fc00000u)
                    : (x == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(x << 23));
}

// The consumer warps (threads 0..127) of every CTA of a unit call this once the CTA's scores
// are written; the last CTA to arrive selects for the unit's rows.
// With the top-k shared across draft tokens (a.share: the unit scored only the sequence's first
// new token), the last CTA selects for every new token of the sequence (q_len of them) from the
// first token's scores.
template <int KPL>
__device__ __forceinline__ void count_out_and_select(const IndexerArgs &a, int b, int tile,
                                                     int hk, int row0, int tok0, int ntok,
                                                     int cl, int q_len, volatile int *is_last) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  named_bar_sync(2, kConsumerWarps * 32);  // every thread's scores written
  if (threadIdx.x == 0) {
    int32_t *c = a.counters + (static_cast<size_t>(b) * a.tiles + tile) * a.H_idxk + hk;
    __threadfence();  // the CTA's scores (ordered before by the barrier), before the count
    const bool last = atomicAdd(c, 1) == a.chunks - 1;
    if (last) {
      __threadfence();  // every other CTA's scores, before this CTA reads them
      atomicExch(c, 0);
    }
    *is_last = last;
  }
  named_bar_sync(2, kConsumerWarps * 32);
  if (!*is_last) return;
  const int Hg = a.H_kv / a.H_idxk;
  const int n_out = a.share ? q_len : ntok;  // tokens selected for
  for (int r = warp; r < n_out * Hg; r += kConsumerWarps) {
    const int tl = r / Hg, g = hk + (r % Hg) * a.H_idxk;
    const size_t item = static_cast<size_t>(row0 + tok0 + tl) * a.H_kv + g;
    const size_t src = a.share ? static_cast<size_t>(row0) * a.H_kv + g : item;
    const int nb_out = min((cl + tok0 + tl) / kBlock + 1, a.max_blocks);
    const int nb = a.share ? min(cl / kBlock + 1, a.max_blocks) : nb_out;
    const int nsel =
        select_row<(KPL > 0 ? KPL : 0), true>(a.scores + src * a.max_blocks, nb, a.top_k,
                                              a.init_blocks, a.local_blocks, a.S,
                                              a.block_ids + item * a.S, a.dev_err, lane, nb_out);
    if (lane == 0) a.num_selected[item] = nsel;
  }
}

// The consumer warps of every CTA of a unit call this once the CTA's scores are written; the
// last CTA to arrive publishes the unit (the one-call decode step).
__device__ __forceinline__ void count_out_and_publish(const IndexerArgs &a, int b, int tile,
                                                      int hk) {
  named_bar_sync(2, kConsumerWarps * 32);  // every thread's scores written
  if (threadIdx.x == 0) {
    const size_t u = (static_cast<size_t>(b) * a.tiles + tile) * a.H_idxk + hk;
    __threadfence();  // the CTA's scores (ordered before by the barrier), before the count
    if (atomicAdd(a.counters + u, 1) == a.chunks - 1) {
      __threadfence();  // every other CTA's scores, before the flag
      atomicExch(a.counters + u, 0);
      const uint32_t step = static_cast<uint32_t>(ld_acquire_gpu(a.epoch));
      st_release_gpu(a.publish + u, static_cast<int>(step + 1u));  // wrapping
    }
  }
}

// KPL == -2: scores, then the unit published (count_out_and_publish); KPL == -1: scores only;
// KPL >= 0: selection fused, KPL keys per lane in registers (0: any
// number of blocks, read from L2 on every pass).
// With one 16-row tile the scaled formats are bounded to four CTAs per SM (registers <= 102
// per thread; two tiles would spill).
template <int MT, int KPL, int kStages, int IF>
__global__ void __launch_bounds__(kThreads, (IF != kIdxBf16 && MT == 1) ? 4 : 1)
    index_scores_kernel(const __grid_constant__ CUtensorMap kmap, const IndexerArgs a) {
  constexpr uint32_t kTileBytes = tile_bytes<IF>();
  constexpr uint32_t kScaleBytes = scale_bytes<IF>();
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // one CTA per (chunk, unit); a unit's chunks are launched together so that units finish one
  // after another (and, fused, select while later units are still scoring)
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
  const int Hg = a.H_kv / a.H_idxk;  // index-query heads per index-K head
  const int rows = ntok * Hg;
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

  // Blocks of this chunk that no token of the tile can see score -inf.
  {
    const int f0 = max(j0, j1), nf = j_end - f0;
    for (int idx = threadIdx.x; idx < nf * rows; idx += blockDim.x) {
      const int r = idx / nf, j = f0 + idx % nf;
      const int t = row0 + tok0 + r / Hg, g = hk + (r % Hg) * a.H_idxk;
      a.scores[(static_cast<size_t>(t) * a.H_kv + g) * a.max_blocks + j] = -INFINITY;
    }
  }
  const int npages = j1 - j0;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;
  uint8_t *scale_st = stages + kStages * kTileBytes;  // [kStages][kScaleBytes]
  uint64_t *full = reinterpret_cast<uint64_t *>(scale_st + kStages * kScaleBytes);
  uint64_t *empty = full + kStages;
  int *page_ok = reinterpret_cast<int *>(empty + kStages);
  float *red = reinterpret_cast<float *>(page_ok + kStages);  // [2][4 warps][32 rows]
  volatile int *abort_flag = reinterpret_cast<volatile int *>(red + 2 * kConsumerWarps * 32);
  volatile int *is_last = abort_flag + 1;

  if (npages <= 0) {
    if (KPL >= 0 || KPL == -2) {
      __syncthreads();  // every thread's -inf fills, before the count
      if (warp < kConsumerWarps) {
        if constexpr (KPL == -2)
          count_out_and_publish(a, b, tile, hk);
        else
          count_out_and_select<KPL>(a, b, tile, hk, row0, tok0, ntok, cl, q_len, is_last);
      }
    }
    return;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer: TMA page ring
    if (lane == 0) prefetch_tmap(&kmap);
    bool dead = false;
    uint32_t issued = 0;  // pages given to the ring (lane 0)
    // 32 page ids fetched at a time, one lane each, then issued by lane 0
    for (int base = 0; base < npages && !dead; base += 32) {
      const int pg_l = base + lane < npages
                           ? a.table[static_cast<size_t>(b) * a.max_pages + j0 + base + lane]
                           : -1;
      const int cnt = min(32, npages - base);
      for (int k = 0; k < cnt; ++k) {
        const int page = __shfl_sync(0xffffffffu, pg_l, k);
        if (lane == 0) {
          const int i = base + k;
          const int s = i % kStages;
          if (i >= kStages && !mbar_wait(&empty[s], ((i / kStages) - 1) & 1, abort_flag)) {
            report(a.dev_err, MSA_DEVERR_TIMEOUT);
            *abort_flag = 1;
            dead = true;
          } else {
            const bool ok = page >= 0 && page < a.num_pages;
            page_ok[s] = ok;
            if (ok) {
              mbar_arrive_expect_tx(&full[s], kTileBytes + kScaleBytes);
              const int c2 = page * a.H_idxk + hk;
              if constexpr (IF == kIdxBf16) {
                tma_load_3d(stages + s * kTileBytes, &kmap, &full[s], 0, 0, c2);
                tma_load_3d(stages + s * kTileBytes + kTileBytes / 2, &kmap, &full[s], 64, 0,
                            c2);
              } else {
                tma_load_3d(stages + s * kTileBytes, &kmap, &full[s], 0, 0, c2);
                bulk_load(scale_st + s * kScaleBytes,
                          static_cast<const uint8_t *>(a.k_idx_scale) +
                              static_cast<size_t>(c2) * kScaleBytes,
                          kScaleBytes, &full[s]);
              }
            } else {
              report(a.dev_err, MSA_DEVERR_PAGE_ID);
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
    if (lane == 0 && !drain_ring(full, kStages, issued)) report(a.dev_err, MSA_DEVERR_TIMEOUT);
    return;
  }

  // -------------------------------------------------------------- consumers
  // A fragments of Q (rows x 128) for m16n8k16: a0a1 = (row, k), a2a3 = (row + 8, k),
  // a4a5 = (row, k + 8), a6a7 = (row + 8, k + 8), k = 16 ks + 2 (lane % 4).
  // Scaled formats: the fragments hold f16 pairs of the dims scaled_dim() names, each row
  // multiplied by qscale = 2^-k (k >= 0, 1 unless the row holds |values| >= 2^15) and its
  // scores by 1 / qscale.
  uint32_t qa[MT][8][4];
  int prow[MT][2];
  float qinv[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int slot = 0; slot < 2; ++slot) {
      const int r = mt * 16 + (lane >> 2) + slot * 8;
      prow[mt][slot] = r < rows ? cl + tok0 + r / Hg : -1;
      qinv[mt][slot] = 1.f;
    }
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int r = mt * 16 + (lane >> 2) + (q4 & 1) * 8;
        const int k = IF == kIdxBf16 ? ks * 16 + (lane & 3) * 2 + (q4 >> 1) * 8
                                     : scaled_dim<IF>(ks, lane & 3) + (q4 >> 1) * 2;
        uint32_t v = 0;
        if (r < rows) {
          const int t = row0 + tok0 + r / Hg, g = hk + (r % Hg) * a.H_idxk;
          v = *reinterpret_cast<const uint32_t *>(
              a.q_idx + (static_cast<size_t>(t) * a.H_kv + g) * kHeadDim + k);
        }
        qa[mt][ks][q4] = v;
      }
    }
    if constexpr (IF != kIdxBf16) {
#pragma unroll
      for (int slot = 0; slot < 2; ++slot) {
        float m = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
#pragma unroll
          for (int hi = 0; hi < 2; ++hi) {
            const float2 f = bf16x2_to_float2(qa[mt][ks][slot + 2 * hi]);
            m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
          }
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        float qs = 1.f;
        if (m >= 32768.f) {  // 2^k with m * 2^-k < 2^15 (m < 2^(e + 1), e = its exponent)
          const int k = static_cast<int>((__float_as_uint(m) >> 23) & 0xff) - 127 - 14;
          qs = __uint_as_float(static_cast<uint32_t>(127 - k) << 23);
          qinv[mt][slot] = __uint_as_float(static_cast<uint32_t>(127 + k) << 23);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
#pragma unroll
          for (int hi = 0; hi < 2; ++hi) {
            const float2 f = bf16x2_to_float2(qa[mt][ks][slot + 2 * hi]);
            qa[mt][ks][slot + 2 * hi] = pack_f16x2(f.x * qs, f.y * qs);
          }
      }
    }
  }

  const int pbase = warp * 32;  // this warp's 32 positions of every page
  const int mi = lane >> 3, rr = lane & 7;
  for (int i = 0; i < npages; ++i) {
    const int s = i % kStages;
    const int j = j0 + i;
    bool live = mbar_wait(&full[s], (i / kStages) & 1, abort_flag);
    if (!live) {
      report(a.dev_err, MSA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
    const bool ok = live && page_ok[s];
    float acc[MT][4][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
    if (ok) {
      const uint32_t tile_addr = smem_u32(stages + s * kTileBytes);
      if constexpr (IF == kIdxBf16) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          uint32_t bf[4][2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int pos = pbase + h * 16 + (mi >> 1) * 8 + rr;
            const int chunk = ks * 2 + (mi & 1);
            ldsm_x4(tile_addr + sw128(pos, chunk, kTileBytes / 2), bf[2 * h][0], bf[2 * h][1],
                    bf[2 * h + 1][0], bf[2 * h + 1][1]);
          }
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
              mma_bf16(acc[mt][nt], qa[mt][ks], bf[nt][0], bf[nt][1]);
        }
      } else {
        const uint8_t *sc = scale_st + s * kScaleBytes;
        const uint8_t *tile = stages + s * kTileBytes;
        const int j4 = lane & 3;
        // the four n-tiles (8 positions each) are interleaved at every k-step so that their
        // accumulator chains run side by side
        if constexpr (IF == kIdxFp8) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            uint32_t w[4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
              w[nt] = *reinterpret_cast<const uint32_t *>(
                  tile + sw128(pbase + nt * 8 + (lane >> 2), ks, kTileBytes) + 4 * j4);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
              uint32_t b0, b1;
              e4m3x4_to_f16x2x2(w[nt], b0, b1);
#pragma unroll
              for (int mt = 0; mt < MT; ++mt) mma_f16(acc[mt][nt], qa[mt][ks], b0, b1);
            }
          }
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
            const float2 ts =
                *reinterpret_cast<const float2 *>(sc + 4 * (pbase + nt * 8 + 2 * j4));
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
              for (int e = 0; e < 4; ++e)
                acc[mt][nt][e] *= ((e & 1) ? ts.y : ts.x) * qinv[mt][e >> 1];
          }
        } else {
          // exponents of the two C columns of every n-tile: 4 bytes (groups) per position
          uint32_t ex[4][2];
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
            const uint2 e2 =
                *reinterpret_cast<const uint2 *>(sc + 4 * (pbase + nt * 8 + 2 * j4));
            ex[nt][0] = e2.x;
            ex[nt][1] = e2.y;
          }
          // NP n-tiles at a time (all four with one 16-row tile, two with two: registers)
          constexpr int NP = MT == 1 ? 4 : 2;
#pragma unroll
          for (int n0 = 0; n0 < 4; n0 += NP)
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
              uint32_t w[NP];
#pragma unroll
              for (int u = 0; u < NP; ++u) {
                const int pos = pbase + (n0 + u) * 8 + (lane >> 2);
                w[u] = *reinterpret_cast<const uint32_t *>(
                    tile + sw128(pos >> 1, 4 * (pos & 1) + gq, kTileBytes) + 4 * j4);
              }
              float cg[MT][NP][4];
#pragma unroll
              for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int u = 0; u < NP; ++u)
#pragma unroll
                  for (int e = 0; e < 4; ++e) cg[mt][u][e] = 0.f;
              uint32_t bf[NP][4];
#pragma unroll
              for (int u = 0; u < NP; ++u) e2m1x8_to_f16x2x4(w[u], bf[u]);
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int u = 0; u < NP; ++u)
#pragma unroll
                  for (int mt = 0; mt < MT; ++mt)
                    mma_f16(cg[mt][u], qa[mt][2 * gq + h], bf[u][2 * h], bf[u][2 * h + 1]);
#pragma unroll
              for (int u = 0; u < NP; ++u) {
                const int nt = n0 + u;
                const float e0 = ue8m0_to_float((ex[nt][0] >> (8 * gq)) & 0xffu);
                const float e1 = ue8m0_to_float((ex[nt][1] >> (8 * gq)) & 0xffu);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                  for (int e = 0; e < 4; ++e)
                    acc[mt][nt][e] = fmaf(cg[mt][u][e], (e & 1) ? e1 : e0, acc[mt][nt][e]);
              }
            }
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[mt][nt][e] *= qinv[mt][e >> 1];
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);

    // Row max over this warp's 32 positions (only positions <= the row's query position).
    float *rbuf = red + (i & 1) * kConsumerWarps * 32;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
      for (int slot = 0; slot < 2; ++slot) {
        float mx = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int pos = j * kBlock + pbase + nt * 8 + (lane & 3) * 2 + e;
            if (ok && pos <= prow[mt][slot]) mx = fmaxf(mx, acc[mt][nt][slot * 2 + e]);
          }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        if ((lane & 3) == 0) rbuf[warp * 32 + mt * 16 + (lane >> 2) + slot * 8] = mx;
      }
    }
    named_bar_sync(1, kConsumerWarps * 32);
    const int r = threadIdx.x;
    if (r < rows) {
      float m = rbuf[r];
#pragma unroll
      for (int w = 1; w < kConsumerWarps; ++w) m = fmaxf(m, rbuf[w * 32 + r]);
      const int t = row0 + tok0 + r / Hg, g = hk + (r % Hg) * a.H_idxk;
      a.scores[(static_cast<size_t>(t) * a.H_kv + g) * a.max_blocks + j] = m;
    }
  }
  if constexpr (KPL == -2)
    count_out_and_publish(a, b, tile, hk);
  else if constexpr (KPL >= 0)
    count_out_and_select<KPL>(a, b, tile, hk, row0, tok0, ntok, cl, q_len, is_last);
}

template <int MT, int KPL, int ST, int IF>
cudaError_t launch_one(const CUtensorMap &kidx_map, const IndexerArgs &a, int chunks,
                       cudaStream_t s) {
  constexpr int kStages = ring_stages<ST, IF>();
  const dim3 grid(a.batch * a.tiles * a.H_idxk * chunks);
  const size_t smem = smem_bytes<kStages, IF>();
  auto *kernel = &index_scores_kernel<MT, KPL, kStages, IF>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(kernel),
                                    static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(kernel, grid, dim3(kThreads), smem, s, kidx_map, a);
}

template <int MT, int KPL, int IF>
cudaError_t launch_st(const CUtensorMap &kidx_map, const IndexerArgs &a, int chunks,
                      cudaStream_t s) {
  return a.chunk >= kLongChunk ? launch_one<MT, KPL, 3, IF>(kidx_map, a, chunks, s)
                               : launch_one<MT, KPL, 2, IF>(kidx_map, a, chunks, s);
}

template <int MT, int IF>
cudaError_t launch_mt(const CUtensorMap &kidx_map, const IndexerArgs &a, int chunks,
                      cudaStream_t s) {
  if (!a.counters) return launch_st<MT, -1, IF>(kidx_map, a, chunks, s);
  if (a.publish) return launch_st<MT, -2, IF>(kidx_map, a, chunks, s);
  if (a.max_blocks <= 4 * 32) return launch_st<MT, 4, IF>(kidx_map, a, chunks, s);
  if (a.max_blocks <= 16 * 32) return launch_st<MT, 16, IF>(kidx_map, a, chunks, s);
  if (a.max_blocks <= 32 * 32) return launch_st<MT, 32, IF>(kidx_map, a, chunks, s);
  return launch_st<MT, 0, IF>(kidx_map, a, chunks, s);
}

template <int IF>
cudaError_t launch_if(const CUtensorMap &kidx_map, const IndexerArgs &a, int mt, int chunks,
                      cudaStream_t s) {
  return mt == 1 ? launch_mt<1, IF>(kidx_map, a, chunks, s)
                 : launch_mt<2, IF>(kidx_map, a, chunks, s);
}

}  // namespace

cudaError_t launch_index_scores(const CUtensorMap &kidx_map, const IndexerArgs &a, int mt,
                                int chunks, cudaStream_t s) {
  switch (a.idx_fmt) {
    case kIdxFp8: return launch_if<kIdxFp8>(kidx_map, a, mt, chunks, s);
    case kIdxFp4: return launch_if<kIdxFp4>(kidx_map, a, mt, chunks, s);
    default: return launch_if<kIdxBf16>(kidx_map, a, mt, chunks, s);
  }
}

}  // namespace msa
