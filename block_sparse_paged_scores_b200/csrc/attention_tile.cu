// attention_tile.cu — stage 3 for prefill: one CTA per (sequence, query tile, KV head).
//
// ferrox-core "Module block_sparse": the attention is an ordinary masked pass over the
// positions the selected blocks cover (ascending, causally clipped).  Mojo module "msa",
// "Three attention routes": above 8 new tokens per sequence the step is a prefill driven by a
// device-built CSR of the selected blocks; each token's causal diagonal is cache_lengths[b] +
// its index.
//
// The CTA walks its tile's union of selected blocks (plan.cu) once; every token keeps only the
// blocks it selected itself (a per-entry token mask) and the positions up to its own.  A
// producer warp streams the K and V page tiles by TMA through a 3-stage ring; 4 x RG consumer
// warps (RG row groups of 16 rows, PQ position splits of every block) run the per-block math
// of attn_common.cuh, merge their online-softmax states through shared memory at the end and
// write the bf16 output.
#include <math.h>

#include "attn_common.cuh"

namespace msa {

namespace {

template <bool FP8>
struct TileCfg {
  static constexpr uint32_t kTile = KvTile<FP8>::kBytes;
  static constexpr int kStages = FP8 ? 6 : 3;
  static constexpr uint32_t kStage = 2 * kTile;  // K + V
};

template <int RG>
constexpr int tile_pq() {
  return RG <= 2 ? 4 : 2;
}

template <bool FP8, int RG>
constexpr size_t tile_smem_bytes() {
  return 1024 + TileCfg<FP8>::kStages * TileCfg<FP8>::kStage + kQBuf +
         TileCfg<FP8>::kStages * (2 * sizeof(uint64_t) + 3 * sizeof(int)) +
         2 * RG * 4 * 16 * sizeof(float) + 16;
}

template <bool FP8, int RG>
__global__ void __launch_bounds__(32 * (RG * tile_pq<RG>() + 1))
    attn_tile_kernel(const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap, const AttnArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  using C = TileCfg<FP8>;
  constexpr int PQ = tile_pq<RG>();
  constexpr int NCW = RG * PQ, NCT = 32 * NCW, NS = C::kStages;
  constexpr uint32_t TILE = C::kTile, STAGE = C::kStage;
  using WA = WarpAttn<FP8, PQ>;

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
  uint8_t *stages = smem;
  uint8_t *qs = stages + NS * STAGE;
  uint64_t *full = reinterpret_cast<uint64_t *>(qs + kQBuf);
  uint64_t *empty = full + NS;
  int *st_j = reinterpret_cast<int *>(empty + NS);
  uint32_t *st_mask = reinterpret_cast<uint32_t *>(st_j + NS);
  int *st_ok = reinterpret_cast<int *>(st_mask + NS);
  float *mrg_m = reinterpret_cast<float *>(st_ok + NS);  // [NCW][16]
  float *mrg_l = mrg_m + RG * 4 * 16;                      // [NCW][16]
  volatile int *abort_flag = reinterpret_cast<volatile int *>(mrg_l + RG * 4 * 16);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  stage_q<FP8, kQRows>(qs, a.q, t0, rows, a.G, a.H_q, g, threadIdx.x, blockDim.x);
  __syncthreads();

  if (warp == NCW) {
    // -------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&vmap);
    }
    bool dead = false;
    uint32_t issued = 0;  // stages given K and V (lane 0)
    // 32 blocks' page ids resolved at a time, one lane each, then issued by lane 0
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
          const int s = i % NS;
          if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1, abort_flag)) {
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
              mbar_arrive_expect_tx(&full[s], 2 * TILE);
              const int c2 = pg * a.H_kv + g;
              uint8_t *kd = stages + s * STAGE, *vd = kd + TILE;
              if (FP8) {
                tma_load_3d(kd, &kmap, &full[s], 0, 0, c2);
                tma_load_3d(vd, &vmap, &full[s], 0, 0, c2);
              } else {
                tma_load_3d(kd, &kmap, &full[s], 0, 0, c2);
                tma_load_3d(kd + TILE / 2, &kmap, &full[s], 64, 0, c2);
                tma_load_3d(vd, &vmap, &full[s], 0, 0, c2);
                tma_load_3d(vd + TILE / 2, &vmap, &full[s], 64, 0, c2);
              }
            } else {
              report(a.dev_err, jok ? MSA_DEVERR_PAGE_ID : MSA_DEVERR_BLOCK_ID);
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
    if (lane == 0 && !drain_ring(full, NS, issued)) report(a.dev_err, MSA_DEVERR_TIMEOUT);
    return;
  }

  // ---------------------------------------------------------------- consumers
  const int rg = warp / PQ, pq = warp % PQ;
  int prow[2];
  uint32_t tbit[2];
#pragma unroll
  for (int slot = 0; slot < 2; ++slot) {
    const int r = rg * 16 + (lane >> 2) + slot * 8;
    const int tl = r / a.G;
    prow[slot] = r < rows ? cl + tok0 + tl : -1;
    tbit[slot] = r < rows ? (1u << tl) : 0u;
  }
  const uint32_t qs_addr = smem_u32(qs);
  WA wa;
  wa.reset();
  for (int i = 0; i < nblk; ++i) {
    const int s = i % NS;
    const bool live = mbar_wait(&full[s], (i / NS) & 1, abort_flag);
    if (!live) {
      report(a.dev_err, MSA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
    if (live && st_ok[s]) {
      const int j = st_j[s];
      const uint32_t kt = smem_u32(stages + s * STAGE);
      wa.qk(qs_addr, kQSub, rg * 16, kt, pq, lane);
      wa.softmax(j, pq, lane, prow, tbit, st_mask[s], a.scale_log2);
      wa.pv(kt + TILE, j, pq, lane, L);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // ---------------------------------------------------------------- merge the PQ position
  // splits of every row group through shared memory, normalise, write bf16
  wa.finish_rows();
  named_bar_sync(1, NCT);  // every consumer is done with the stages
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  float *mo = reinterpret_cast<float *>(stages);  // [NCW][16][padded 128]
  constexpr int MS = MergeRow<FP8>::kStride;
  if ((lane & 3) == 0) {
#pragma unroll
    for (int slot = 0; slot < 2; ++slot) {
      mrg_m[warp * 16 + (lane >> 2) + slot * 8] = wa.m_run[slot];
      mrg_l[warp * 16 + (lane >> 2) + slot * 8] = wa.l_run[slot];
    }
  }
  named_bar_sync(1, NCT);
#pragma unroll
  for (int slot = 0; slot < 2; ++slot) {
    const int r16 = (lane >> 2) + slot * 8;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < PQ; ++w) M = fmaxf(M, mrg_m[(rg * PQ + w) * 16 + r16]);
    float Ls = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < PQ; ++w) {
        const float mw = mrg_m[(rg * PQ + w) * 16 + r16];
        if (mw != -INFINITY) Ls += mrg_l[(rg * PQ + w) * 16 + r16] * fast_exp2(mw - M);
      }
    }
    const float f =
        (Ls > 0.f && wa.m_run[slot] != -INFINITY) ? fast_exp2(wa.m_run[slot] - M) / Ls : 0.f;
    wa.store_row(mo + static_cast<size_t>(warp) * 16 * MS, r16, slot, f, lane, false);
  }
  named_bar_sync(1, NCT);
  for (int idx = threadIdx.x; idx < RG * 16 * (kHeadDim / 4); idx += NCT) {
    const int r = idx / (kHeadDim / 4), d4 = idx % (kHeadDim / 4);
    if (r >= rows) continue;
    const int rgr = r >> 4, r16 = r & 15;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < PQ; ++w) {
      const float4 v = *reinterpret_cast<const float4 *>(
          mo + (static_cast<size_t>(rgr * PQ + w) * 16 + r16) * MS + 4 * d4);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    const size_t orow = static_cast<size_t>(t0 + r / a.G) * a.H_q + g * a.G + r % a.G;
    uint2 packed;
    packed.x = pack_bf16x2(acc.x, acc.y);
    packed.y = pack_bf16x2(acc.z, acc.w);
    reinterpret_cast<uint2 *>(a.out + orow * kHeadDim)[d4] = packed;
  }
}

template <bool FP8, int RG>
cudaError_t launch_tile_one(const CUtensorMap &kmap, const CUtensorMap &vmap, const AttnArgs &a,
                            cudaStream_t s) {
  const size_t smem = tile_smem_bytes<FP8, RG>();
  auto fn = &attn_tile_kernel<FP8, RG>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(fn), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(a.batch * a.tiles, a.H_kv);
  return launch_pdl(fn, grid, dim3(32 * (RG * tile_pq<RG>() + 1)), smem, s, kmap, vmap, a);
}

template <bool FP8>
cudaError_t launch_tile_rg(const CUtensorMap &kmap, const CUtensorMap &vmap, const AttnArgs &a,
                           int rg, cudaStream_t s) {
  switch (rg) {
    case 1: return launch_tile_one<FP8, 1>(kmap, vmap, a, s);
    case 2: return launch_tile_one<FP8, 2>(kmap, vmap, a, s);
    case 3: return launch_tile_one<FP8, 3>(kmap, vmap, a, s);
    default: return launch_tile_one<FP8, 4>(kmap, vmap, a, s);
  }
}

}  // namespace

cudaError_t launch_attention_tiles(const CUtensorMap &kmap, const CUtensorMap &vmap,
                                   const AttnArgs &a, bool fp8, int rg, cudaStream_t s) {
  return fp8 ? launch_tile_rg<true>(kmap, vmap, a, rg, s)
             : launch_tile_rg<false>(kmap, vmap, a, rg, s);
}

}  // namespace msa
