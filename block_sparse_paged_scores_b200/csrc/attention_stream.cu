// attention_stream.cu — stage 3 for decode and speculative decode: a persistent kernel that
// streams the selected pages of every (sequence, KV head) through every SM at a steady rate.
//
// ferrox-core "Module block_sparse": the attention is an ordinary masked pass over the
// positions the selected blocks cover (ascending, causally clipped).  Mojo module "msa",
// "Three attention routes": decode needs no causal mask (the query is the last position of its
// sequence); the speculative route masks each draft token causally in-kernel (position =
// cache_lengths[b] + token index, block start = block id * 128); the selected blocks are split
// over SM-filling split-K partitions whose partials, keyed on the ragged global query row, are
// merged by a combine that writes the ragged output.  Main KV is BF16 or scale-free FP8 e4m3,
// accumulation FP32.
//
// Work list: item = (sequence, query tile, KV head); its `cap` slots are the selected block
// ids (decode: the selection itself, cap = S) or the tile's union of them (speculative:
// plan.cu, cap = tile tokens x S), of which the first U are real.  The items' slots laid end
// to end are cut into equal contiguous ranges of R slots, one per CTA (a split-K partition):
// every SM streams the same number of slots.  A CTA's range meets a few items; each meeting is
// a "segment", merged inside the CTA into one partial (normalised output and log-sum-exp) at
// split index `piece` = the CTA's rank among the CTAs that share the item; split indices no
// CTA fills are marked empty.  msa_splitk_combine's kernel merges the pieces.  With a single
// partition (every item inside one CTA) the kernel writes the bf16 output itself instead.
// On speculative tiles a row group (16 rows: two draft tokens) skips the math of a union block
// that neither of its tokens selected: their state would not change.
//
// Roles: one producer warp walks the items, marks empty partials, loads each non-empty
// segment's Q rows and metadata into a double-buffered Q slot and issues the TMA loads of the
// K and V page tiles (128-byte swizzle) into the consumers' rings, running ahead across
// segment boundaries.  Consumer warps touch no global memory but their partials: they run the
// per-block math of attn_common.cuh (each owns 16 rows and a share of every block's positions;
// FP8 with one row group splits into two teams taking alternate blocks), release the K slot
// after QK^T and the V slot after PV, and at the end of a segment fold their online-softmax
// states pairwise into one per row through shared memory.
#include <math.h>

#include <type_traits>

#include "attn_common.cuh"
#include "select_row.cuh"

namespace msa {

namespace {

// Consumer layout for RG 16-row groups: PQ warps split every block's positions and NT teams
// of RG * PQ warps take alternate blocks.  With a single row group every SM sub-partition
// gets two warps: BF16 splits each block eight ways; FP8 (whose K fragments come four n-tiles
// at a time) runs two teams of four.
template <bool FP8, int RG>
constexpr int stream_pq() {
  return RG == 1 ? (FP8 ? 4 : 8) : (RG == 2 ? 4 : 2);
}
template <bool FP8, int RG>
constexpr int stream_teams() {
  return RG == 1 && FP8 ? 2 : 1;
}
template <bool FP8, int RG>
constexpr int stream_consumer_warps() {
  return RG * stream_pq<FP8, RG>() * stream_teams<FP8, RG>();
}

// Every team has a ring of its own (a team consumes its ring strictly in order, which is what
// makes the phase-parity waits exact): 160 KiB of tiles per SM (128 KiB with four row groups,
// whose Q buffers and merge slices take the rest of the shared memory).
template <bool FP8, int RG>
struct StreamCfg {
  static constexpr uint32_t kTile = KvTile<FP8>::kBytes;
  static constexpr int kTeams = stream_teams<FP8, RG>();
  static constexpr int kRing = (RG == 4 ? (FP8 ? 8 : 4) : (FP8 ? 10 : 5)) / kTeams;
  static constexpr int kSlots = kTeams * kRing;
};

// What the producer hands the consumers with each non-empty segment's Q rows.
struct SegMeta {
  int valid;  // 0: no segment left
  int t0, rows, cl, tok0, g, L, v0, v1, piece;
};

// one warp's 16 rows (padded stride), then their m and l
template <bool FP8>
constexpr int slice_floats() {
  return 16 * MergeRow<FP8>::kStride + 32;
}

// Decode with the selection inside (SEL > 0): the selecting warps hand the producer each
// selected block with its page id, for the CTA's first kSelSlots work-list slots, and the
// number selected, for its first kSelItems items, through shared memory.  A CTA whose range is
// longer reads them back from global memory instead.
constexpr int kSelSlots = 1024;
constexpr int kSelItems = 128;

template <bool FP8, int RG, int SEL = -1>
constexpr size_t stream_smem_bytes() {
  using C = StreamCfg<FP8, RG>;
  constexpr int W = stream_pq<FP8, RG>() * stream_teams<FP8, RG>();  // warps per row group
  return 1024 + C::kSlots * C::kTile + 2 * (RG * 16 * 256) +            // tiles, 2 Q buffers
         RG * (W / 2) * slice_floats<FP8>() * sizeof(float) +           // merge slices
         (2 * C::kSlots + 4) * sizeof(uint64_t) + C::kSlots * 3 * sizeof(int) +
         2 * sizeof(SegMeta) + 16 +
         (SEL > 0 ? 16 + kSelSlots * sizeof(int2) + kSelItems * sizeof(int) : 0);
}

struct Item {
  int b, g, tok0, ntok, rows, t0, cl, L, U;
  const int32_t *list;
  const uint32_t *masks;
};

// u_known >= 0: the item's number selected, already known (the selection inside the kernel)
template <bool PLAN>
__device__ __forceinline__ Item load_item(const AttnArgs &a, int it, bool reporter,
                                          int u_known = -1) {
  Item m;
  const int y = it / a.H_kv;
  m.g = it % a.H_kv;
  m.b = y / a.tiles;
  const int tile = y % a.tiles;
  const int row0 = a.row_off[m.b];
  int q_len = a.row_off[m.b + 1] - row0;
  if (q_len < 0 || q_len > a.max_q_len) {
    if (reporter) report(a.dev_err, MSA_DEVERR_LENGTHS);
    q_len = q_len < 0 ? 0 : a.max_q_len;
  }
  m.tok0 = tile * a.qt;
  m.ntok = max(0, min(a.qt, q_len - m.tok0));
  m.rows = m.ntok * a.G;
  m.t0 = row0 + m.tok0;
  int cl = a.cache_len[m.b];
  if (cl < 0) {
    if (reporter) report(a.dev_err, MSA_DEVERR_LENGTHS);
    cl = 0;
  }
  m.cl = cl;
  m.L = cl + q_len;
  m.U = 0;
  m.list = nullptr;
  m.masks = nullptr;
  if (m.ntok > 0) {
    if (PLAN) {
      const size_t idx = static_cast<size_t>(it);
      m.list = a.plan_list + idx * a.cap;
      m.masks = a.plan_masks + idx * a.cap;
      m.U = min(max(a.plan_counts[idx], 0), a.cap);
    } else {
      const size_t sel = static_cast<size_t>(m.t0) * a.H_kv + m.g;
      m.list = a.block_ids + sel * a.S;
      int u = u_known >= 0 ? u_known : a.num_selected[sel];
      if (u < 0 || u > a.S) {
        if (reporter) report(a.dev_err, MSA_DEVERR_NUM_SELECTED);
        u = u < 0 ? 0 : a.S;
      }
      m.U = u;
    }
    if (m.U == 0 && reporter) report(a.dev_err, MSA_DEVERR_NUM_SELECTED);  // never empty
  }
  return m;
}

// Slots [v0, v1) of item `it` that fall in this CTA's range [r0, r1) and are real.
__device__ __forceinline__ void segment(const AttnArgs &a, int it, long long r0, long long r1,
                                        int U, int &v0, int &v1) {
  const long long base = static_cast<long long>(it) * a.cap;
  v0 = static_cast<int>(max(r0 - base, 0LL));
  const int s1 = static_cast<int>(min(r1 - base, static_cast<long long>(a.cap)));
  v1 = min(s1, U);
}

// SEL >= 0: decode with the selection in the kernel (select_row with SEL keys per lane in
// registers, 0: from memory); SEL < 0: the selection comes from an earlier launch.
// SWAP: decode items of at most 8 rows, on the swapped-operand math (WarpAttnSwap).
template <bool FP8, int RG, bool PLAN, int SEL, bool SWAP>
__global__ void __launch_bounds__(32 * (stream_consumer_warps<FP8, RG>() + 1))
    attn_stream_kernel(const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap, const AttnArgs a) {
  constexpr int PQ = stream_pq<FP8, RG>();
  constexpr int NT = stream_teams<FP8, RG>();
  constexpr int TEAM = RG * PQ;                           // warps of one team
  constexpr int W = NT * PQ;                              // warps sharing a row group
  constexpr int NCW = stream_consumer_warps<FP8, RG>();   // all consumer warps
  constexpr int NSLOT = StreamCfg<FP8, RG>::kSlots;       // all rings
  constexpr int NR = StreamCfg<FP8, RG>::kRing;           // slots of one team's ring
  constexpr uint32_t TILE = StreamCfg<FP8, RG>::kTile;
  constexpr int QR = RG * 16;                             // rows of a Q buffer
  constexpr uint32_t QSUB = QR * 128, QBUF = 2 * QSUB;
  static_assert(!SWAP || (RG == 1 && !PLAN), "swapped math: one decode row group");
  using WA = std::conditional_t<SWAP, WarpAttnSwap<FP8, PQ>, WarpAttn<FP8, PQ>>;
  constexpr int SLICE = slice_floats<FP8>();
  constexpr int MS = MergeRow<FP8>::kStride;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long total = static_cast<long long>(a.items) * a.cap;
  const long long r0 = static_cast<long long>(blockIdx.x) * a.R;
  const long long r1 = min(total, r0 + a.R);
  if (r0 >= r1) return;
  const int it_first = static_cast<int>(r0 / a.cap);
  const int it_last = static_cast<int>((r1 - 1) / a.cap);
  const size_t split_stride = static_cast<size_t>(a.total_q) * a.H_q;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *slots = smem;
  uint8_t *qbufs = slots + NSLOT * TILE;
  float *slices = reinterpret_cast<float *>(qbufs + 2 * QBUF);  // [RG][W/2][SLICE]
  uint64_t *sfull = reinterpret_cast<uint64_t *>(slices + RG * (W / 2) * SLICE);
  uint64_t *sempty = sfull + NSLOT;
  uint64_t *qfull = sempty + NSLOT;
  uint64_t *qempty = qfull + 2;
  int *slot_j = reinterpret_cast<int *>(qempty + 2);
  uint32_t *slot_mask = reinterpret_cast<uint32_t *>(slot_j + NSLOT);
  int *slot_ok = reinterpret_cast<int *>(slot_mask + NSLOT);
  SegMeta *meta = reinterpret_cast<SegMeta *>(slot_ok + NSLOT);  // [2], one per Q buffer
  volatile int *abort_flag = reinterpret_cast<volatile int *>(meta + 2);
  int2 *sel_pairs = reinterpret_cast<int2 *>(
      (reinterpret_cast<uintptr_t>(abort_flag + 4) + 15) & ~static_cast<uintptr_t>(15));
  int *sel_u = reinterpret_cast<int *>(sel_pairs + kSelSlots);  // used when SEL > 0
  const int n_items = it_last - it_first + 1;
  // the selection hands its result over in shared memory (see kSelSlots)
  const bool sel_smem = SEL > 0 && r1 - r0 <= kSelSlots && n_items <= kSelItems;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], TEAM);  // each tile is read by one team
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&qfull[q], 1);
      mbar_init(&qempty[q], NCW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // ---- producer state and helpers (warp NCW; declared here because, on decode with the
  // selection inside, the producer hands the first segment over while the others select)
  int q_staged = -1;  // item whose Q rows are in Q buffer 0 already
  bool dead = false;
  uint32_t nload0 = 0, nload1 = 0;  // tile loads issued into each team's ring
  int n = 0;                        // non-empty segments handed over
  int seg_k = 0;                    // blocks of the current segment issued so far
  // waits (lane 0) until the consumers are done with Q buffer n & 1; false on timeout
  auto claim_qbuf = [&](int n_) -> bool {
    bool ok = true;
    if (lane == 0 && n_ >= 2) ok = mbar_wait(&qempty[n_ & 1], ((n_ >> 1) - 1) & 1, abort_flag);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok && lane == 0) {
      report(a.dev_err, MSA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
    return ok;
  };
  // hands segment n's Q rows (staged already when q_ready) and metadata to the consumers
  auto hand_segment = [&](const Item &m, int v0, int v1, int piece, bool q_ready) -> bool {
    if (!claim_qbuf(n)) return false;
    const int buf = n & 1;
    if (!q_ready)
      stage_q<FP8, QR>(qbufs + buf * QBUF, a.q, m.t0, m.rows, a.G, a.H_q, m.g, lane, 32);
    if (lane == 0) {
      SegMeta md;
      md.valid = 1;
      md.t0 = m.t0;
      md.rows = m.rows;
      md.cl = m.cl;
      md.tok0 = m.tok0;
      md.g = m.g;
      md.L = m.L;
      md.v0 = v0;
      md.v1 = v1;
      md.piece = piece;
      meta[buf] = md;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&qfull[buf]);
    ++n;
    seg_k = 0;
    return true;
  };
  // lane 0: K and V tile loads of block jj (page pg, token mask mm) of KV head g into the
  // ring of the team that reads the segment's seg_k-th block; false on timeout
  auto issue_block = [&](int jj, int pg, uint32_t mm, int g) -> bool {
    const bool jok = jj >= 0 && jj < a.max_blocks;
    const bool ok = jok && pg >= 0 && pg < a.num_pages;
    if (!ok) report(a.dev_err, jok ? MSA_DEVERR_PAGE_ID : MSA_DEVERR_BLOCK_ID);
    const int c2 = pg * a.H_kv + g;
    const int tm = seg_k % NT;  // the team that reads this block
    ++seg_k;
#pragma unroll
    for (int kv = 0; kv < 2; ++kv) {
      const uint32_t nl = tm ? nload1 : nload0;
      const int s = tm * NR + static_cast<int>(nl % NR);
      if (nl >= static_cast<uint32_t>(NR) &&
          !mbar_wait(&sempty[s], ((nl / NR) - 1) & 1, abort_flag)) {
        report(a.dev_err, MSA_DEVERR_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
      slot_j[s] = jj;
      slot_mask[s] = mm;
      slot_ok[s] = ok;
      if (ok) {
        const CUtensorMap *mp = kv ? &vmap : &kmap;
        uint8_t *dst = slots + s * TILE;
        mbar_arrive_expect_tx(&sfull[s], TILE);
        tma_load_3d(dst, mp, &sfull[s], 0, 0, c2);
        if (!FP8) tma_load_3d(dst + TILE / 2, mp, &sfull[s], 64, 0, c2);
      } else {
        mbar_arrive(&sfull[s]);
      }
      if (tm)
        nload1 = nl + 1;
      else
        nload0 = nl + 1;
    }
    return true;
  };
  int pre_it = -1, pre_u = 0;  // item whose segment was handed over before the selection

  if (warp == NCW && lane == 0) {  // kernel parameters: no earlier kernel writes them
    prefetch_tmap(&kmap);
    prefetch_tmap(&vmap);
  }
  // With the flags of the one-call decode step the scores are waited for row by row below;
  // nothing else this kernel reads comes from the launch before it.
  const bool flagged = SEL >= 0 && a.ready != nullptr;
  if (!flagged) pdl_wait();  // block ids, counts and the plan (or the scores): earlier kernels
  pdl_launch_dependents();
  const int ready_value =  // the step counter + 1 (wrapping)
      flagged ? static_cast<int>(static_cast<uint32_t>(ld_acquire_gpu(a.epoch)) + 1u) : 0;

  if constexpr (SEL > 0) {
    // The producer hands the first segment (Q rows and metadata) to the consumers before the
    // selection is known: the number of blocks selected follows from the sequence length
    // alone (the forced blocks and min(top_k, candidates)), and so does the segment.  After
    // the selection it only issues the tile loads, in the list's order.
    if (warp == NCW && sel_smem) {
      const Item m0 = load_item<false>(a, it_first, false, 0);
      if (m0.ntok > 0) {
        int nb = m0.cl / kBlock + 1;
        if (nb > a.max_blocks) nb = a.max_blocks;  // reported by the selecting warp
        const int init_e = min(a.init_blocks, nb);
        const int local_lo = max(init_e, nb - a.local_blocks);
        const int u =
            min(init_e + (nb - local_lo) + min(max(a.top_k, 0), local_lo - init_e), a.S);
        int v0, v1;
        segment(a, it_first, r0, r1, u, v0, v1);
        const long long base = static_cast<long long>(it_first) * a.cap;
        const int piece = static_cast<int>(blockIdx.x - base / a.R);
        if (v1 > v0 && hand_segment(m0, v0, v1, piece, false)) {
          q_staged = it_first;
          pre_it = it_first;
          pre_u = u;
        }
      }
    }
  }

  // Decode with the selection inside: every warp of the CTA selects rows of the CTA's items
  // (one query row per item; block_sparse_select as in select.cu), before any of them is
  // streamed.  Items shared with a neighbouring CTA are selected by both, with identical
  // results.  The loads that do not depend on one another are issued together, in one memory
  // round trip: each selecting warp's row metadata, the scores of the row where the sequence's
  // first query row lies when every sequence has the same number of rows (read again from the
  // right row otherwise), and the page ids of its first item's blocks (held one per lane and
  // block, so that the lane that takes a block also knows its page); the producer's first Q
  // rows while the others select.
  constexpr int KS = SEL > 0 ? SEL : 1;
  if constexpr (SEL >= 0) {
    const int rows_per_seq = a.total_q / max(a.batch, 1);
    for (int k = warp; k < n_items; k += NCW + 1) {
      const int it = it_first + k;
      const int g = it % a.H_kv, b = it / a.H_kv;  // one query tile per sequence
      const bool keep = sel_smem && k == warp;    // hand the result over in shared memory
      // page id of block 32 i + lane, loaded with the scores when a lane holds up to 16 blocks
      // (more would spill registers: the producer then looks the pages up itself)
      constexpr bool kPagesInRegs = KS <= 16;
      uint32_t sel_page[kPagesInRegs ? KS : 1];
      float sc[KS];           // score of block 32 i + lane (SEL > 0)
      const int guess = b * rows_per_seq;
      auto load_scores = [&](int row) {
        const float *sr = a.scores + (static_cast<size_t>(row) * a.H_kv + g) * a.max_blocks;
#pragma unroll
        for (int i = 0; i < KS; ++i) {
          const int j = 32 * i + lane;
          sc[i] = j < a.max_blocks ? sr[j] : -INFINITY;
        }
      };
      if constexpr (SEL > 0) {
        if (!flagged) load_scores(guess);
      }
      if (kPagesInRegs && keep) {
#pragma unroll
        for (int i = 0; i < KS; ++i) {
          const int j = 32 * i + lane;
          sel_page[i] =
              j < a.max_blocks ? a.table[static_cast<size_t>(b) * a.max_pages + j] : 0xffffffffu;
        }
      }
      const int row0 = a.row_off[b];
      if (a.row_off[b + 1] - row0 <= 0) {  // no query row
        if (sel_smem && lane == 0) sel_u[k] = -1;
        continue;
      }
      int nb = max(a.cache_len[b], 0) / kBlock + 1;
      if (nb > a.max_blocks) {
        if (lane == 0) report(a.dev_err, MSA_DEVERR_LENGTHS);
        nb = a.max_blocks;
      }
      if (flagged) {
        // this row's index unit published by the indexer launch: every lane acquires the flag
        // itself before reading the scores
        const int32_t *f = a.ready + static_cast<size_t>(b) * a.H_idxk + g % a.H_idxk;
        const uint64_t t0 = global_timer_ns();
        bool timed_out = false;
        while (!__all_sync(0xffffffffu, ld_acquire_gpu(f) == ready_value)) {
          if (global_timer_ns() - t0 > kWaitTimeoutNs) {
            timed_out = true;
            break;
          }
          __nanosleep(128);
        }
        if (timed_out && lane == 0) {
          report(a.dev_err, MSA_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
        if constexpr (SEL > 0) load_scores(row0);
      } else if constexpr (SEL > 0) {
        if (row0 != guess) load_scores(row0);
      }
      const size_t sel = static_cast<size_t>(row0) * a.H_kv + g;
      const long long slot0 = static_cast<long long>(it) * a.cap - r0;
      // the selected blocks of this CTA's range, with their pages, into shared memory
      struct Emit {
        const uint32_t *page;  // this lane's sel_page
        int2 *pairs;
        long long slot0, n;
        bool keep;
        __device__ __forceinline__ void put(int pos, int j, int pg) const {
          const long long slot = slot0 + pos;
          if (keep && slot >= 0 && slot < n) pairs[slot] = make_int2(j, pg);
        }
        __device__ __forceinline__ void taken(int pos, int j, int i) const {
          put(pos, j, kPagesInRegs ? static_cast<int>(page[i < KS ? i : 0]) : -1);
        }
        __device__ __forceinline__ void gathered(int pos, int j, int i, int src,
                                                 bool valid) const {
          int pg = -1;
          if constexpr (kPagesInRegs) {  // pass i's page of lane src, one shuffle per pass
#pragma unroll
            for (int t = 0; t < KS; ++t) {
              const int v = __shfl_sync(0xffffffffu, static_cast<int>(page[t]), src);
              if (t == i) pg = v;
            }
          }
          if (valid) put(pos, j, pg);
        }
      };
      const Emit emit{sel_page, sel_pairs, slot0, r1 - r0, keep};
      auto score = [&](int i) { return sc[i < KS ? i : 0]; };
      const int nsel = select_row_from<(SEL > 0 ? SEL : 0), false>(
          score, a.scores + sel * a.max_blocks, nb, a.top_k, a.init_blocks, a.local_blocks, a.S,
          a.sel_ids + sel * a.S, a.dev_err, lane, 0, emit);
      if (lane == 0) {
        a.sel_counts[sel] = nsel;
        if (sel_smem) sel_u[k] = keep ? nsel : -1;
      }
    }
    if (warp == NCW && NCW >= n_items && pre_it < 0) {  // the producer selected nothing: its first Q rows
      const Item m0 = load_item<false>(a, it_first, false, 0);
      if (m0.ntok > 0) {
        stage_q<FP8, QR>(qbufs, a.q, m0.t0, m0.rows, a.G, a.H_q, m0.g, lane, 32);
        q_staged = it_first;
      }
    }
    __syncthreads();  // the producer reads the selection back
  }

  if (warp == NCW) {
    // ============================================================== producer warp
    for (int it = it_first; it <= it_last && !dead; ++it) {
      // >= 0: the item's selection is in sel_pairs / sel_u
      const int u_sm = sel_smem ? sel_u[it - it_first] : -1;
      const Item m = load_item<PLAN>(a, it, lane == 0, u_sm);
      if (m.ntok == 0) continue;  // a tile past its sequence's end: no rows
      int v0, v1;
      segment(a, it, r0, r1, m.U, v0, v1);
      const long long base = static_cast<long long>(it) * a.cap;
      const int piece = static_cast<int>(blockIdx.x - base / a.R);
      const bool last_cta = (base + a.cap - 1) / a.R == blockIdx.x;
      // split indices of this item's rows that stay empty: this CTA's own when it has no real
      // block of the item, and, from the item's last CTA, those past it
      const int p_lo = v1 > v0 ? piece + 1 : piece;
      const int p_hi = last_cta ? a.P : piece + 1;
      for (int idx = lane; idx < m.rows * max(p_hi - p_lo, 0); idx += 32) {
        const int r = idx % m.rows, p2 = p_lo + idx / m.rows;
        const size_t orr = static_cast<size_t>(m.t0 + r / a.G) * a.H_q + m.g * a.G + r % a.G;
        if (a.direct) {  // a row that saw nothing: zeros, as the combine would give
          uint4 *dst = reinterpret_cast<uint4 *>(a.out + orr * kHeadDim);
          for (int c = 0; c < kHeadDim / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
        } else {
          a.part_lse[static_cast<size_t>(p2) * split_stride + orr] = -INFINITY;
        }
      }
      if (v1 <= v0) continue;

      // ---- Q rows and metadata of this segment (handed over already for pre_it)
      const bool pre = it == pre_it;
      if (pre && m.U != pre_u && lane == 0) report(a.dev_err, MSA_DEVERR_NUM_SELECTED);
      if (!pre && !hand_segment(m, v0, v1, piece, n == 0 && it == q_staged)) {
        dead = true;
        break;
      }

      // ---- K and V tiles.  The warp resolves 32 blocks' page ids at a time (one lane
      // each) so that lane 0 never waits on a dependent lookup between two TMAs.
      for (int bbase = v0; bbase < v1 && !dead; bbase += 32) {
        const int e = bbase + lane;
        int j = -1, page = -1;
        uint32_t msk = 0u;
        if (e < v1) {
          if (u_sm >= 0) {  // e lies in this CTA's range: its slot was written
            const int2 pr = sel_pairs[static_cast<long long>(it) * a.cap + e - r0];
            j = pr.x;
            page = pr.y;
            msk = 0xffffffffu;
            if (page < 0 && j >= 0 && j < a.max_blocks)  // not resolved by the selecting warp
              page = a.table[static_cast<size_t>(m.b) * a.max_pages + j];
          } else {
            j = m.list[e];
            msk = PLAN ? m.masks[e] : 0xffffffffu;
            if (j >= 0 && j < a.max_blocks)
              page = a.table[static_cast<size_t>(m.b) * a.max_pages + j];
          }
        }
        const int cnt = min(32, v1 - bbase);
        for (int i = 0; i < cnt; ++i) {
          const int jj = __shfl_sync(0xffffffffu, j, i);
          const int pg = __shfl_sync(0xffffffffu, page, i);
          const uint32_t mm = __shfl_sync(0xffffffffu, msk, i);
          if (lane == 0 && !issue_block(jj, pg, mm, m.g)) dead = true;
          dead = __shfl_sync(0xffffffffu, dead, 0);
          if (dead) break;
        }
      }
    }
    // ---- no segment left
    if (!dead && claim_qbuf(n) && lane == 0) {
      meta[n & 1].valid = 0;
      mbar_arrive(&qfull[n & 1]);
    }
    // one-call decode step: every flag this CTA waits for was seen (the selection is done);
    // the last CTA to get here advances the epoch for the next step
    if (flagged && lane == 0) {
      if (atomicAdd(a.step_done, 1) == static_cast<int>(gridDim.x) - 1) {
        atomicExch(a.step_done, 0);
        st_release_gpu(a.epoch, ready_value);
      }
    }
    // every tile load it issued (lane 0 did) has landed before this warp exits
    if (lane == 0) {
      const bool landed =
          drain_ring(sfull, NR, nload0) && (NT < 2 || drain_ring(sfull + NR, NR, nload1));
      if (!landed) report(a.dev_err, MSA_DEVERR_TIMEOUT);
    }
    return;
  }

  // ================================================================ consumer warps
  const int team = warp / TEAM, rg = (warp % TEAM) / PQ, pq = warp % PQ;
  const int rank = team * PQ + pq;  // rank among the W warps of this row group
  const int nct = 32 * NCW;
  float *my_slices = slices + rg * (W / 2) * SLICE;
  WA wa;
  uint32_t nload = 0;  // loads this warp's team has consumed from its ring
  for (int n = 0;; ++n) {
    const int buf = n & 1;
    if (!mbar_wait(&qfull[buf], (n >> 1) & 1, abort_flag)) {
      report(a.dev_err, MSA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
    named_bar_sync(1, nct);  // every consumer takes the same decision below
    if (*abort_flag) break;
    const SegMeta md = meta[buf];
    if (!md.valid) break;
    int prow[2];
    uint32_t tbit[2];
#pragma unroll
    for (int slot = 0; slot < 2; ++slot) {
      const int r = SWAP ? 2 * (lane & 3) + slot : rg * 16 + (lane >> 2) + slot * 8;
      const int tl = r / a.G;
      prow[slot] = r < md.rows ? md.cl + md.tok0 + tl : -1;
      tbit[slot] = r < md.rows ? (1u << tl) : 0u;
    }
    // the tokens of this warp's row group: a block none of them selected leaves its rows'
    // state unchanged, so its math is skipped (speculative tiles walk their tokens' union)
    const uint32_t rg_bits = __reduce_or_sync(0xffffffffu, tbit[0] | tbit[1]);
    const uint32_t qs_addr = smem_u32(qbufs + buf * QBUF);
    wa.reset();
    if constexpr (SWAP) wa.load_q(qs_addr, QSUB, lane);
    for (int e = md.v0 + team; e < md.v1; e += NT) {
      const uint32_t nk = nload;  // this team's K tile; V is nk + 1
      int s = team * NR + static_cast<int>(nk % NR);
      bool live = mbar_wait(&sfull[s], (nk / NR) & 1, abort_flag);
      const int j = slot_j[s];
      const uint32_t msk = slot_mask[s];
      const bool ok = live && slot_ok[s] && (msk & rg_bits) != 0;
      if (ok) wa.qk(qs_addr, QSUB, rg * 16, smem_u32(slots + s * TILE), pq, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sempty[s]);
      if (ok) wa.softmax(j, pq, lane, prow, tbit, msk, a.scale_log2);
      s = team * NR + static_cast<int>((nk + 1) % NR);
      live = mbar_wait(&sfull[s], ((nk + 1) / NR) & 1, abort_flag) && live;
      if (ok && live) wa.pv(smem_u32(slots + s * TILE), j, pq, lane, md.L);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sempty[s]);
      nload = nk + 2;
      if (!live) {
        report(a.dev_err, MSA_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&qempty[buf]);

    // ---- fold the W warp states of every row into rank 0: a pairwise log-sum-exp tree
    // through shared-memory slices, in a fixed order (reproducible sums)
    wa.finish_rows();
#pragma unroll
    for (int step = W / 2; step >= 1; step >>= 1) {
      if constexpr (SWAP) {
        if (rank >= step && rank < 2 * step)
          wa.store_rows(my_slices + (rank - step) * SLICE, {1.f, 1.f}, lane);
        named_bar_sync(1, nct);
        if (rank < step) wa.merge_rows(my_slices + rank * SLICE, lane);
        named_bar_sync(1, nct);
      } else {
        if (rank >= step && rank < 2 * step) {
          float *sl = my_slices + (rank - step) * SLICE;
#pragma unroll
          for (int slot = 0; slot < 2; ++slot) {
            const int r16 = (lane >> 2) + slot * 8;
            wa.store_row(sl, r16, slot, 1.f, lane, false);
            if ((lane & 3) == 0) {
              sl[16 * MS + r16] = wa.m_run[slot];
              sl[16 * MS + 16 + r16] = wa.l_run[slot];
            }
          }
        }
        named_bar_sync(1, nct);
        if (rank < step) {
          const float *sl = my_slices + rank * SLICE;
#pragma unroll
          for (int slot = 0; slot < 2; ++slot) {
            const int r16 = (lane >> 2) + slot * 8;
            wa.merge_row(sl, r16, slot, sl[16 * MS + r16], sl[16 * MS + 16 + r16], lane);
          }
        }
        named_bar_sync(1, nct);
      }
    }
    // ---- rank 0 writes this segment's partial: normalised output and log-sum-exp
    if constexpr (SWAP) {
      // through its own slice (rank 0 read it last), so that the rows leave in whole 16-byte
      // pieces
      if (rank == 0) {
        float *sl = my_slices;
        const float f[2] = {wa.l_run[0] > 0.f ? 1.f / wa.l_run[0] : 0.f,
                            wa.l_run[1] > 0.f ? 1.f / wa.l_run[1] : 0.f};
        wa.store_rows(sl, f, lane);
        __syncwarp();
        for (int idx = lane; idx < md.rows * 32; idx += 32) {
          const int r = idx >> 5, c4 = idx & 31;
          const size_t orr =
              static_cast<size_t>(md.t0 + r / a.G) * a.H_q + md.g * a.G + r % a.G;
          const float4 v = *reinterpret_cast<const float4 *>(sl + r * MS + 4 * c4);
          if (a.direct) {
            *reinterpret_cast<uint2 *>(a.out + orr * kHeadDim + 4 * c4) =
                make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
          } else {
            const size_t pr = static_cast<size_t>(md.piece) * split_stride + orr;
            *reinterpret_cast<float4 *>(a.part_o + pr * kHeadDim + 4 * c4) = v;
          }
        }
        if (!a.direct && lane < 4) {
#pragma unroll
          for (int slot = 0; slot < 2; ++slot) {
            const int r = 2 * lane + slot;
            if (r >= md.rows) continue;
            const size_t orr =
                static_cast<size_t>(md.t0 + r / a.G) * a.H_q + md.g * a.G + r % a.G;
            const float l = wa.l_run[slot];
            a.part_lse[static_cast<size_t>(md.piece) * split_stride + orr] =
                l > 0.f ? (wa.m_run[slot] + __log2f(l)) * kLn2 : -INFINITY;
          }
        }
      }
    } else {
      if (rank == 0) {
#pragma unroll
        for (int slot = 0; slot < 2; ++slot) {
          const int r = rg * 16 + (lane >> 2) + slot * 8;
          if (r >= md.rows) continue;
          const size_t orr =
              static_cast<size_t>(md.t0 + r / a.G) * a.H_q + md.g * a.G + r % a.G;
          const float l = wa.l_run[slot];
          if (a.direct) {
            wa.store_bf16(a.out + orr * kHeadDim, slot, l > 0.f ? 1.f / l : 0.f, lane);
            continue;
          }
          const size_t pr = static_cast<size_t>(md.piece) * split_stride + orr;
          wa.store_global(a.part_o + pr * kHeadDim, slot, l > 0.f ? 1.f / l : 0.f, lane);
          if ((lane & 3) == 0)
            a.part_lse[pr] = l > 0.f ? (wa.m_run[slot] + __log2f(l)) * kLn2 : -INFINITY;
        }
      }
    }
  }
}

template <bool FP8, int RG, bool PLAN, int SEL, bool SWAP = false>
cudaError_t launch_stream_one(const CUtensorMap &kmap, const CUtensorMap &vmap,
                              const AttnArgs &a, int grid, cudaStream_t s) {
  constexpr size_t smem = stream_smem_bytes<FP8, RG, SEL>();
  static_assert(smem <= 227 * 1024, "shared memory of one CTA");
  auto fn = &attn_stream_kernel<FP8, RG, PLAN, SEL, SWAP>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(fn), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(fn, dim3(grid), dim3(32 * (stream_consumer_warps<FP8, RG>() + 1)), smem, s,
                    kmap, vmap, a);
}

template <bool FP8, bool PLAN>
cudaError_t launch_stream_rg(const CUtensorMap &kmap, const CUtensorMap &vmap, const AttnArgs &a,
                             int rg, int grid, cudaStream_t s) {
  switch (rg) {
    case 1:
      if (!PLAN && a.G <= 8)
        return launch_stream_one<FP8, 1, false, -1, true>(kmap, vmap, a, grid, s);
      return launch_stream_one<FP8, 1, PLAN, -1>(kmap, vmap, a, grid, s);
    case 2: return launch_stream_one<FP8, 2, PLAN, -1>(kmap, vmap, a, grid, s);
    case 3: return launch_stream_one<FP8, 3, PLAN, -1>(kmap, vmap, a, grid, s);
    default: return launch_stream_one<FP8, 4, PLAN, -1>(kmap, vmap, a, grid, s);
  }
}

// decode with the selection inside: one row group, keys per lane chosen by the row length
template <bool FP8, bool SWAP>
cudaError_t launch_stream_sel_math(const CUtensorMap &kmap, const CUtensorMap &vmap,
                                   const AttnArgs &a, int grid, cudaStream_t s) {
  if (a.max_blocks <= 4 * 32)
    return launch_stream_one<FP8, 1, false, 4, SWAP>(kmap, vmap, a, grid, s);
  if (a.max_blocks <= 16 * 32)
    return launch_stream_one<FP8, 1, false, 16, SWAP>(kmap, vmap, a, grid, s);
  if (a.max_blocks <= 32 * 32)
    return launch_stream_one<FP8, 1, false, 32, SWAP>(kmap, vmap, a, grid, s);
  return launch_stream_one<FP8, 1, false, 0, SWAP>(kmap, vmap, a, grid, s);
}
template <bool FP8>
cudaError_t launch_stream_sel(const CUtensorMap &kmap, const CUtensorMap &vmap, const AttnArgs &a,
                              int grid, cudaStream_t s) {
  return a.G <= 8 ? launch_stream_sel_math<FP8, true>(kmap, vmap, a, grid, s)
                  : launch_stream_sel_math<FP8, false>(kmap, vmap, a, grid, s);
}

}  // namespace

cudaError_t launch_attention_stream(const CUtensorMap &kmap, const CUtensorMap &vmap,
                                    const AttnArgs &a, bool fp8, int rg, bool plan, int grid,
                                    cudaStream_t s) {
  if (a.sel_ids) {  // decode (rg == 1, no plan) with the selection inside
    if (plan || rg != 1) return cudaErrorInvalidValue;
    return fp8 ? launch_stream_sel<true>(kmap, vmap, a, grid, s)
               : launch_stream_sel<false>(kmap, vmap, a, grid, s);
  }
  if (fp8)
    return plan ? launch_stream_rg<true, true>(kmap, vmap, a, rg, grid, s)
                : launch_stream_rg<true, false>(kmap, vmap, a, rg, grid, s);
  return plan ? launch_stream_rg<false, true>(kmap, vmap, a, rg, grid, s)
              : launch_stream_rg<false, false>(kmap, vmap, a, rg, grid, s);
}

}  // namespace msa
