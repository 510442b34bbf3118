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
// a "segment" and each (segment, consumer warp) leaves one partial (normalised output and
// log-sum-exp) at split index piece * PQ + position-quarter, piece = the CTA's rank among the
// CTAs that share the item.  msa_splitk_combine's kernel merges them.
//
// Roles: one producer warp loads each segment's Q rows into a double-buffered Q slot and
// issues the TMA loads of the K and V page tiles (128-byte swizzle) into a ring of tile slots,
// running ahead across segment boundaries; 4 x RG consumer warps run the per-block math of
// attn_common.cuh, releasing the K slot after QK^T and the V slot after PV.
#include <math.h>

#include "attn_common.cuh"

namespace msa {

namespace {

template <bool FP8>
struct StreamCfg {
  static constexpr uint32_t kTile = KvTile<FP8>::kBytes;
  static constexpr int kSlots = FP8 ? 10 : 5;  // 160 KiB of tiles in flight per SM
};

template <bool FP8>
constexpr size_t stream_smem_bytes() {
  return 1024 + StreamCfg<FP8>::kSlots * StreamCfg<FP8>::kTile + 2 * kQBuf +
         (2 * StreamCfg<FP8>::kSlots + 4) * sizeof(uint64_t) +
         StreamCfg<FP8>::kSlots * 3 * sizeof(int) + 16;
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
__global__ void __launch_bounds__(32 * (RG * (RG <= 2 ? 4 : 2) + 1))
    attn_stream_kernel(const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap, const AttnArgs a) {
  constexpr int PQ = RG <= 2 ? 4 : 2;
  constexpr int NCW = RG * PQ;
  constexpr int NSLOT = StreamCfg<FP8>::kSlots;
  constexpr uint32_t TILE = StreamCfg<FP8>::kTile;
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
  uint64_t *sfull = reinterpret_cast<uint64_t *>(qbufs + 2 * kQBuf);
  uint64_t *sempty = sfull + NSLOT;
  uint64_t *qfull = sempty + NSLOT;
  uint64_t *qempty = qfull + 2;
  int *slot_j = reinterpret_cast<int *>(qempty + 2);
  uint32_t *slot_mask = reinterpret_cast<uint32_t *>(slot_j + NSLOT);
  int *slot_ok = reinterpret_cast<int *>(slot_mask + NSLOT);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(slot_ok + NSLOT);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], NCW);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&qfull[q], 1);
      mbar_init(&qempty[q], NCW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NCW) {
    // ============================================================== producer warp
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&vmap);
    }
    bool dead = false;
    uint32_t nload = 0;  // tile loads issued (two per block: K then V)
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
      // ---- K and V tiles of segment n
      if (lane == 0) {
        for (int e = v0; e < v1 && !dead; ++e) {
          const int j = cur.list[e];
          const uint32_t msk = PLAN ? cur.masks[e] : 0xffffffffu;
          const bool jok = j >= 0 && j < a.max_blocks;
          const int page = jok ? a.table[static_cast<size_t>(cur.b) * a.max_pages + j] : -1;
          const bool ok = jok && page >= 0 && page < a.num_pages;
          if (!ok) report(a.dev_err, jok ? MSA_DEVERR_PAGE_ID : MSA_DEVERR_BLOCK_ID);
          const int c2 = page * a.H_kv + cur.g;
#pragma unroll
          for (int kv = 0; kv < 2; ++kv) {
            const int s = static_cast<int>(nload % NSLOT);
            if (nload >= static_cast<uint32_t>(NSLOT) &&
                !mbar_wait(&sempty[s], ((nload / NSLOT) - 1) & 1, abort_flag)) {
              report(a.dev_err, MSA_DEVERR_TIMEOUT);
              *abort_flag = 1;
              dead = true;
              break;
            }
            slot_j[s] = j;
            slot_mask[s] = msk;
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
            ++nload;
          }
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
  const int rg = warp / PQ, pq = warp % PQ;
  WA wa;
  uint32_t nload = 0;
  int n = 0;
  for (int it = it_first; it <= it_last; ++it) {
    const Item m = load_item<PLAN>(a, it, false);
    if (m.ntok == 0) continue;  // a tile past its sequence's end: no rows
    int v0, v1;
    segment(a, it, r0, r1, m.U, v0, v1);
    const long long base = static_cast<long long>(it) * a.cap;
    const int piece = static_cast<int>(blockIdx.x - base / a.R);
    const bool last_cta = (base + a.cap - 1) / a.R == blockIdx.x;
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
    const size_t split_stride = static_cast<size_t>(a.total_q) * a.H_q;

    if (v1 > v0) {
      const int buf = n & 1;
      const bool qlive = mbar_wait(&qfull[buf], (n >> 1) & 1, abort_flag);
      if (!qlive) {
        report(a.dev_err, MSA_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
      const uint32_t qs_addr = smem_u32(qbufs + buf * kQBuf);
      wa.reset();
      for (int e = v0; e < v1; ++e) {
        // K tile
        int s = static_cast<int>(nload % NSLOT);
        bool live = mbar_wait(&sfull[s], (nload / NSLOT) & 1, abort_flag);
        const bool ok = live && qlive && slot_ok[s];
        const int j = slot_j[s];
        const uint32_t msk = slot_mask[s];
        if (ok) wa.qk(qs_addr, rg * 16, smem_u32(slots + s * TILE), pq, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[s]);
        ++nload;
        if (ok) wa.softmax(j, pq, lane, prow, tbit, msk, a.scale_log2);
        // V tile
        s = static_cast<int>(nload % NSLOT);
        live = mbar_wait(&sfull[s], (nload / NSLOT) & 1, abort_flag) && live;
        if (ok && live) wa.pv(smem_u32(slots + s * TILE), j, pq, lane, m.L);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[s]);
        ++nload;
        if (!live) {
          report(a.dev_err, MSA_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&qempty[buf]);
      ++n;
      wa.finish_rows();
      // partial of this (segment, warp): normalised output and natural log-sum-exp
      const size_t split = static_cast<size_t>(piece) * PQ + pq;
#pragma unroll
      for (int slot = 0; slot < 2; ++slot) {
        if (!rvalid[slot]) continue;
        const float l = wa.l_run[slot];
        const size_t prow_i = split * split_stride + orow[slot];
        if (l > 0.f) {
          wa.store_row(a.part_o + prow_i * kHeadDim, slot, 1.f / l, lane);
          if ((lane & 3) == 0) a.part_lse[prow_i] = (wa.m_run[slot] + __log2f(l)) * kLn2;
        } else if ((lane & 3) == 0) {
          a.part_lse[prow_i] = -INFINITY;
        }
      }
    } else {
      // a range that meets this item only in slots past its count: an empty partial
#pragma unroll
      for (int slot = 0; slot < 2; ++slot)
        if (rvalid[slot] && (lane & 3) == 0)
          a.part_lse[(static_cast<size_t>(piece) * PQ + pq) * split_stride + orow[slot]] =
              -INFINITY;
    }
    // the item's last CTA marks the split indices no CTA of this item owns
    if (last_cta) {
      for (int p2 = piece + 1; p2 < a.P; ++p2)
#pragma unroll
        for (int slot = 0; slot < 2; ++slot)
          if (rvalid[slot] && (lane & 3) == 0)
            a.part_lse[(static_cast<size_t>(p2) * PQ + pq) * split_stride + orow[slot]] =
                -INFINITY;
    }
  }
}

template <bool FP8, int RG, bool PLAN>
cudaError_t launch_stream_one(const CUtensorMap &kmap, const CUtensorMap &vmap,
                              const AttnArgs &a, int grid, cudaStream_t s) {
  const size_t smem = stream_smem_bytes<FP8>();
  auto fn = &attn_stream_kernel<FP8, RG, PLAN>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(fn), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  fn<<<grid, 32 * (RG * (RG <= 2 ? 4 : 2) + 1), smem, s>>>(kmap, vmap, a);
  return cudaGetLastError();
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

int attn_position_splits(int rg) { return rg <= 2 ? 4 : 2; }

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
