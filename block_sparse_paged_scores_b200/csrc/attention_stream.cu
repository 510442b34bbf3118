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
// split index `piece` = the CTA's rank among the CTAs that share the item.
// msa_splitk_combine's kernel merges the pieces.
//
// Roles: one producer warp loads each segment's Q rows into a double-buffered Q slot and
// issues the TMA loads of the K and V page tiles (128-byte swizzle) into a ring of tile slots,
// running ahead across segment boundaries.  Consumer warps run the per-block math of
// attn_common.cuh (each owns 16 rows and a share of every block's positions; with one row
// group, two teams take alternate blocks), release the K slot after QK^T and the V slot after
// PV, and at the end of a segment fold their online-softmax states into one per row through
// shared memory.
#include <math.h>

#include "attn_common.cuh"

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
// makes the phase-parity waits exact): 160 KiB of tiles per SM.
template <bool FP8, int RG>
struct StreamCfg {
  static constexpr uint32_t kTile = KvTile<FP8>::kBytes;
  static constexpr int kTeams = stream_teams<FP8, RG>();
  static constexpr int kRing = (FP8 ? 10 : 5) / kTeams;  // slots per team
  static constexpr int kSlots = kTeams * kRing;
};

template <bool FP8, int RG>
constexpr size_t stream_smem_bytes() {
  using C = StreamCfg<FP8, RG>;
  return 1024 + C::kSlots * C::kTile + 2 * kQBuf +
         RG * 16 * kHeadDim * sizeof(float) +                        // merge accumulator
         (2 * C::kSlots + 4) * sizeof(uint64_t) + C::kSlots * 3 * sizeof(int) +
         2 * stream_consumer_warps<FP8, RG>() * 16 * sizeof(float) +       // per-warp m, l
         2 * RG * 16 * sizeof(float) + 16;                           // per-row M, L
}

struct Item {
  int b, g, tok0, ntok, rows, t0, cl, L, U;
  const int32_t *list;
  const uint32_t *masks;
};

template <bool PLAN>
__device__ __forceinline__ Item load_item(const AttnArgs &a, int it, bool reporter) {
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
      int u = a.num_selected[sel];
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

template <bool FP8, int RG, bool PLAN>
__global__ void __launch_bounds__(32 * (stream_consumer_warps<FP8, RG>() + 1))
    attn_stream_kernel(const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap, const AttnArgs a) {
  constexpr int PQ = stream_pq<FP8, RG>();
  constexpr int NT = stream_teams<FP8, RG>();
  constexpr int TEAM = RG * PQ;                    // warps of one team
  constexpr int NCW = stream_consumer_warps<FP8, RG>();  // all consumer warps
  constexpr int NSLOT = StreamCfg<FP8, RG>::kSlots;  // all rings
  constexpr int NR = StreamCfg<FP8, RG>::kRing;      // slots of one team's ring
  constexpr uint32_t TILE = StreamCfg<FP8, RG>::kTile;
  using WA = WarpAttn<FP8, PQ>;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long total = static_cast<long long>(a.items) * a.cap;
  const long long r0 = static_cast<long long>(blockIdx.x) * a.R;
  const long long r1 = min(total, r0 + a.R);
  if (r0 >= r1) return;
  const int it_first = static_cast<int>(r0 / a.cap);
  const int it_last = static_cast<int>((r1 - 1) / a.cap);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *slots = smem;
  uint8_t *qbufs = slots + NSLOT * TILE;
  float *acc = reinterpret_cast<float *>(qbufs + 2 * kQBuf);  // [RG*16][128] merge buffer
  uint64_t *sfull = reinterpret_cast<uint64_t *>(acc + RG * 16 * kHeadDim);
  uint64_t *sempty = sfull + NSLOT;
  uint64_t *qfull = sempty + NSLOT;
  uint64_t *qempty = qfull + 2;
  int *slot_j = reinterpret_cast<int *>(qempty + 2);
  uint32_t *slot_mask = reinterpret_cast<uint32_t *>(slot_j + NSLOT);
  int *slot_ok = reinterpret_cast<int *>(slot_mask + NSLOT);
  float *mrg_m = reinterpret_cast<float *>(slot_ok + NSLOT);  // [NCW][16]
  float *mrg_l = mrg_m + NCW * 16;                              // [NCW][16]
  float *row_m = mrg_l + NCW * 16;                              // [RG*16]
  float *row_l = row_m + RG * 16;                               // [RG*16]
  volatile int *abort_flag = reinterpret_cast<volatile int *>(row_l + RG * 16);

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
  pdl_wait();  // block ids, selection counts and the plan come from earlier kernels
  pdl_launch_dependents();

  if (warp == NCW) {
    // ============================================================== producer warp
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&vmap);
    }
    bool dead = false;
    // tile loads issued into each team's ring (two per block: K then V)
    uint32_t nload0 = 0, nload1 = 0;
    int n = 0;           // index of the current non-empty segment
    // first non-empty segment
    int it = it_first, v0 = 0, v1 = 0;
    Item cur;
    for (; it <= it_last; ++it) {
      cur = load_item<PLAN>(a, it, lane == 0);
      segment(a, it, r0, r1, cur.U, v0, v1);
      if (v1 > v0) break;
    }
    if (it <= it_last) {
      stage_q<FP8>(qbufs, a.q, cur.t0, cur.rows, a.G, a.H_q, cur.g, lane, 32);
      __syncwarp();
      if (lane == 0) mbar_arrive(&qfull[0]);
    }
    while (it <= it_last && !dead) {
      // ---- K and V tiles of segment n.  The warp resolves 32 blocks' page ids at a time
      // (one lane each) so that lane 0 never waits on a dependent lookup between two TMAs.
      for (int base = v0; base < v1 && !dead; base += 32) {
        const int e = base + lane;
        int j = -1, page = -1;
        uint32_t msk = 0u;
        if (e < v1) {
          j = cur.list[e];
          msk = PLAN ? cur.masks[e] : 0xffffffffu;
          if (j >= 0 && j < a.max_blocks)
            page = a.table[static_cast<size_t>(cur.b) * a.max_pages + j];
        }
        const int cnt = min(32, v1 - base);
        for (int i = 0; i < cnt; ++i) {
          const int jj = __shfl_sync(0xffffffffu, j, i);
          const int pg = __shfl_sync(0xffffffffu, page, i);
          const uint32_t mm = __shfl_sync(0xffffffffu, msk, i);
          if (lane == 0) {
            const bool jok = jj >= 0 && jj < a.max_blocks;
            const bool ok = jok && pg >= 0 && pg < a.num_pages;
            if (!ok) report(a.dev_err, jok ? MSA_DEVERR_PAGE_ID : MSA_DEVERR_BLOCK_ID);
            const int c2 = pg * a.H_kv + cur.g;
            const int tm = (base + i - v0) % NT;  // the team that reads this block
#pragma unroll
            for (int kv = 0; kv < 2; ++kv) {
              const uint32_t nl = tm ? nload1 : nload0;
              const int s = tm * NR + static_cast<int>(nl % NR);
              if (nl >= static_cast<uint32_t>(NR) &&
                  !mbar_wait(&sempty[s], ((nl / NR) - 1) & 1, abort_flag)) {
                report(a.dev_err, MSA_DEVERR_TIMEOUT);
                *abort_flag = 1;
                dead = true;
                break;
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
          }
          dead = __shfl_sync(0xffffffffu, dead, 0);
          if (dead) break;
        }
      }
      dead = __shfl_sync(0xffffffffu, dead, 0);
      if (dead) break;
      // ---- Q rows of the next non-empty segment into the other Q buffer
      int nit = it + 1, w0 = 0, w1 = 0;
      Item nxt;
      for (; nit <= it_last; ++nit) {
        nxt = load_item<PLAN>(a, nit, lane == 0);
        segment(a, nit, r0, r1, nxt.U, w0, w1);
        if (w1 > w0) break;
      }
      if (nit <= it_last) {
        const int buf = (n + 1) & 1;
        bool qok = true;  // lane 0 waits for the buffer, the warp follows it
        if (lane == 0 && n + 1 >= 2)
          qok = mbar_wait(&qempty[buf], (((n + 1) >> 1) - 1) & 1, abort_flag);
        qok = __shfl_sync(0xffffffffu, qok, 0);
        if (!qok) {
          if (lane == 0) {
            report(a.dev_err, MSA_DEVERR_TIMEOUT);
            *abort_flag = 1;
          }
          break;
        }
        stage_q<FP8>(qbufs + buf * kQBuf, a.q, nxt.t0, nxt.rows, a.G, a.H_q, nxt.g, lane, 32);
        __syncwarp();
        if (lane == 0) mbar_arrive(&qfull[buf]);
      }
      cur = nxt;
      it = nit;
      v0 = w0;
      v1 = w1;
      ++n;
    }
    return;
  }

  // ================================================================ consumer warps
  const int team = warp / TEAM, rg = (warp % TEAM) / PQ, pq = warp % PQ;
  const bool row_owner = team == 0 && pq == 0 && (lane & 3) == 0;  // one writer per row
  const int nct = 32 * NCW;
  WA wa;
  uint32_t nload = 0;  // loads this warp's team has consumed from its ring
  int n = 0;
  for (int it = it_first; it <= it_last; ++it) {
    const Item m = load_item<PLAN>(a, it, false);
    if (m.ntok == 0) continue;  // a tile past its sequence's end: no rows
    int v0, v1;
    segment(a, it, r0, r1, m.U, v0, v1);
    const long long base = static_cast<long long>(it) * a.cap;
    const int piece = static_cast<int>(blockIdx.x - base / a.R);
    const bool last_cta = (base + a.cap - 1) / a.R == blockIdx.x;
    const size_t split_stride = static_cast<size_t>(a.total_q) * a.H_q;
    // this thread's two rows
    int prow[2];
    uint32_t tbit[2];
    size_t orow[2];
    bool rvalid[2];
#pragma unroll
    for (int slot = 0; slot < 2; ++slot) {
      const int r = rg * 16 + (lane >> 2) + slot * 8;
      const int tl = r / a.G;
      rvalid[slot] = r < m.rows;
      prow[slot] = rvalid[slot] ? m.cl + m.tok0 + tl : -1;
      tbit[slot] = rvalid[slot] ? (1u << tl) : 0u;
      orow[slot] = rvalid[slot] ? static_cast<size_t>(m.t0 + tl) * a.H_q + m.g * a.G + r % a.G : 0;
    }

    if (v1 > v0) {
      const int buf = n & 1;
      const bool qlive = mbar_wait(&qfull[buf], (n >> 1) & 1, abort_flag);
      if (!qlive) {
        report(a.dev_err, MSA_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
      const uint32_t qs_addr = smem_u32(qbufs + buf * kQBuf);
      wa.reset();
      for (int e = v0 + team; e < v1; e += NT) {
        const uint32_t nk = nload;  // this team's K tile; V is nk + 1
        int s = team * NR + static_cast<int>(nk % NR);
        bool live = mbar_wait(&sfull[s], (nk / NR) & 1, abort_flag);
        const bool ok = live && qlive && slot_ok[s];
        const int j = slot_j[s];
        const uint32_t msk = slot_mask[s];
        if (ok) wa.qk(qs_addr, rg * 16, smem_u32(slots + s * TILE), pq, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[s]);
        if (ok) wa.softmax(j, pq, lane, prow, tbit, msk, a.scale_log2);
        s = team * NR + static_cast<int>((nk + 1) % NR);
        live = mbar_wait(&sfull[s], ((nk + 1) / NR) & 1, abort_flag) && live;
        if (ok && live) wa.pv(smem_u32(slots + s * TILE), j, pq, lane, m.L);
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
      ++n;

      // ---- fold the NT * PQ warp states of every row into one, through shared memory
      wa.finish_rows();
      if ((lane & 3) == 0) {
#pragma unroll
        for (int slot = 0; slot < 2; ++slot) {
          mrg_m[warp * 16 + (lane >> 2) + slot * 8] = wa.m_run[slot];
          mrg_l[warp * 16 + (lane >> 2) + slot * 8] = wa.l_run[slot];
        }
      }
      named_bar_sync(1, nct);
      float fac[2];
#pragma unroll
      for (int slot = 0; slot < 2; ++slot) {
        const int r16 = (lane >> 2) + slot * 8;
        float M = -INFINITY;
#pragma unroll
        for (int t2 = 0; t2 < NT; ++t2)
#pragma unroll
          for (int p2 = 0; p2 < PQ; ++p2)
            M = fmaxf(M, mrg_m[(t2 * TEAM + rg * PQ + p2) * 16 + r16]);
        float Ls = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int t2 = 0; t2 < NT; ++t2)
#pragma unroll
            for (int p2 = 0; p2 < PQ; ++p2) {
              const int w2 = t2 * TEAM + rg * PQ + p2;
              const float mw = mrg_m[w2 * 16 + r16];
              if (mw != -INFINITY) Ls += mrg_l[w2 * 16 + r16] * fast_exp2(mw - M);
            }
        }
        fac[slot] = wa.m_run[slot] == -INFINITY ? 0.f : fast_exp2(wa.m_run[slot] - M);
        if (row_owner) {
          row_m[rg * 16 + r16] = M;
          row_l[rg * 16 + r16] = Ls;
        }
      }
      // fixed-order accumulation (reproducible sums): in round k the warp of each row group
      // whose rank in the group is k adds its rescaled output; round 0 stores.
      const int rank = team * PQ + pq;
      for (int k = 0; k < NT * PQ; ++k) {
        if (rank == k) {
#pragma unroll
          for (int slot = 0; slot < 2; ++slot)
            wa.store_row(acc, rg * 16 + (lane >> 2) + slot * 8, slot, fac[slot], lane, k > 0);
        }
        named_bar_sync(1, nct);
      }
      // ---- write this segment's partial (all consumer threads)
      const int ctid = threadIdx.x;  // consumers are threads [0, nct)
      for (int idx = ctid; idx < RG * 16 * (kHeadDim / 4); idx += nct) {
        const int r = idx / (kHeadDim / 4), d4 = idx % (kHeadDim / 4);
        if (r >= m.rows) continue;
        const int tl = r / a.G;
        const size_t orr = static_cast<size_t>(m.t0 + tl) * a.H_q + m.g * a.G + r % a.G;
        const size_t pr = static_cast<size_t>(piece) * split_stride + orr;
        const float L = row_l[r];
        const float inv = L > 0.f ? 1.f / L : 0.f;
        const float4 v =
            *reinterpret_cast<const float4 *>(acc + r * kHeadDim + acc_col(r, 4 * d4));
        reinterpret_cast<float4 *>(a.part_o + pr * kHeadDim)[d4] =
            make_float4(v.x * inv, v.y * inv, v.z * inv, v.w * inv);
        if (d4 == 0) a.part_lse[pr] = L > 0.f ? (row_m[r] + __log2f(L)) * kLn2 : -INFINITY;
      }
    } else if (row_owner) {
      // a range that meets this item only in slots past its count: an empty partial
#pragma unroll
      for (int slot = 0; slot < 2; ++slot)
        if (rvalid[slot]) a.part_lse[static_cast<size_t>(piece) * split_stride + orow[slot]] = -INFINITY;
    }
    // the item's last CTA marks the split indices no CTA of this item owns
    if (last_cta && row_owner) {
      for (int p2 = piece + 1; p2 < a.P; ++p2)
#pragma unroll
        for (int slot = 0; slot < 2; ++slot)
          if (rvalid[slot])
            a.part_lse[static_cast<size_t>(p2) * split_stride + orow[slot]] = -INFINITY;
    }
  }
}

template <bool FP8, int RG, bool PLAN>
cudaError_t launch_stream_one(const CUtensorMap &kmap, const CUtensorMap &vmap,
                              const AttnArgs &a, int grid, cudaStream_t s) {
  const size_t smem = stream_smem_bytes<FP8, RG>();
  auto fn = &attn_stream_kernel<FP8, RG, PLAN>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(fn), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(fn, dim3(grid), dim3(32 * (stream_consumer_warps<FP8, RG>() + 1)), smem, s,
                    kmap, vmap, a);
}

template <bool FP8, bool PLAN>
cudaError_t launch_stream_rg(const CUtensorMap &kmap, const CUtensorMap &vmap, const AttnArgs &a,
                             int rg, int grid, cudaStream_t s) {
  switch (rg) {
    case 1: return launch_stream_one<FP8, 1, PLAN>(kmap, vmap, a, grid, s);
    case 2: return launch_stream_one<FP8, 2, PLAN>(kmap, vmap, a, grid, s);
    case 3: return launch_stream_one<FP8, 3, PLAN>(kmap, vmap, a, grid, s);
    default: return launch_stream_one<FP8, 4, PLAN>(kmap, vmap, a, grid, s);
  }
}

}  // namespace

cudaError_t launch_attention_stream(const CUtensorMap &kmap, const CUtensorMap &vmap,
                                    const AttnArgs &a, bool fp8, int rg, bool plan, int grid,
                                    cudaStream_t s) {
  if (fp8)
    return plan ? launch_stream_rg<true, true>(kmap, vmap, a, rg, grid, s)
                : launch_stream_rg<true, false>(kmap, vmap, a, rg, grid, s);
  return plan ? launch_stream_rg<false, true>(kmap, vmap, a, rg, grid, s)
              : launch_stream_rg<false, false>(kmap, vmap, a, rg, grid, s);
}

}  // namespace msa
