// attention.cu — stage 3: softmax attention over the selected pages of the paged KV cache.
//
// ferrox-core "Module block_sparse": the attention is an ordinary masked pass over the
// positions the selected blocks cover (positions_of_blocks: ascending, causally clipped).
// Mojo module "msa", "Three attention routes": decode needs no causal mask (the query sits at
// the end of its sequence), the speculative route masks each draft token causally in-kernel
// with position cache_lengths[b] + token index and block start = block id * 128, split-K
// partials are keyed on the ragged global query row; the main KV is BF16 or scale-free FP8
// e4m3 and everything accumulates in FP32.
//
// Work item = (sequence, query tile, KV head, split-K partition).  Its rows are the tile's
// tokens x the KV head's GQA group (at most 64).  The item walks its slice of the ascending
// list of blocks to read: the selection itself for decode, or the tile's union (plan.cu) with
// a per-token mask for the other routes, so each page crosses HBM once per tile.
//
// Warp roles: one producer warp issues TMA loads of the K and V page tiles (128-byte swizzle)
// into a ring of shared-memory stages; 4 x RG consumer warps each own 16 rows and 32 of the
// 128 positions of every block and keep their own online-softmax state (flash-decoding inside
// the CTA), merged once at the end.  QK^T and PV run on mma.sync m16n8k16 with FP32
// accumulators; BF16 KV uses bf16 operands, FP8 KV is converted to f16 in registers (exact)
// and runs f16 operands (q rounded to f16, P in f16).
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace msa {

namespace {

constexpr int kQRows = 64;
constexpr uint32_t kQSub = kQRows * 128;  // one 64-column (bf16/f16) sub-tile of Q
constexpr float kLn2 = 0.69314718055994530942f;

template <bool FP8>
struct KvCfg {
  static constexpr uint32_t kTile = FP8 ? 16384u : 32768u;  // one (page, head) tile
  static constexpr int kStages = FP8 ? 6 : 3;
  static constexpr uint32_t kStage = 2 * kTile;  // K + V
};

template <bool FP8, int RG>
constexpr size_t attn_smem_bytes() {
  return 1024 + KvCfg<FP8>::kStages * KvCfg<FP8>::kStage + 2 * kQSub +
         KvCfg<FP8>::kStages * (2 * sizeof(uint64_t) + 3 * sizeof(int)) +
         2 * RG * 4 * 16 * sizeof(float) + RG * 16 * sizeof(float) + 16;
}

template <bool FP8, int RG, bool PLAN>
__global__ void __launch_bounds__(32 * (RG * (RG <= 2 ? 4 : 2) + 1))
    attn_kernel(const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap, const AttnArgs a) {
  using C = KvCfg<FP8>;
  constexpr int PQ = RG <= 2 ? 4 : 2;     // position splits of every block
  constexpr int PW = kBlock / PQ;          // positions per consumer warp
  constexpr int NTW = PW / 8, KSW = PW / 16;
  constexpr int NCW = RG * PQ, NCT = 32 * NCW, NS = C::kStages;
  constexpr uint32_t TILE = C::kTile, STAGE = C::kStage;
  constexpr uint32_t KSUB = FP8 ? TILE : TILE / 2;  // bytes of one swizzled [128][128 B] sub-tile

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.z, g = blockIdx.y;
  const int b = blockIdx.x / a.tiles, tile = blockIdx.x % a.tiles;
  const bool reporter = threadIdx.x == 0 && split == 0 && g == 0 && tile == 0;

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
  const int L = cl + q_len;  // KV length of the sequence, new tokens included

  const int32_t *list;
  const uint32_t *masks = nullptr;
  int U;
  if (PLAN) {
    const size_t item = static_cast<size_t>(blockIdx.x) * a.H_kv + g;
    list = a.plan_list + item * a.cap;
    masks = a.plan_masks + item * a.cap;
    U = min(max(a.plan_counts[item], 0), a.cap);
  } else {
    const size_t sel = static_cast<size_t>(t0) * a.H_kv + g;
    list = a.block_ids + sel * a.S;
    U = a.num_selected[sel];
    if (U < 0 || U > a.S) {
      if (threadIdx.x == 0 && split == 0) report(a.dev_err, MSA_DEVERR_NUM_SELECTED);
      U = U < 0 ? 0 : a.S;
    }
  }
  const int lo = static_cast<int>(static_cast<long long>(split) * U / a.splits);
  const int hi = static_cast<int>(static_cast<long long>(split + 1) * U / a.splits);
  const int nblk = hi - lo;

  if (nblk <= 0) {  // this partition covers no block
    if (U == 0 && threadIdx.x == 0 && split == 0) report(a.dev_err, MSA_DEVERR_NUM_SELECTED);
    for (int idx = threadIdx.x; idx < rows * (kHeadDim / 4); idx += blockDim.x) {
      const int r = idx / (kHeadDim / 4), d4 = idx % (kHeadDim / 4);
      const int t = t0 + r / a.G, h = g * a.G + r % a.G;
      const size_t orow = static_cast<size_t>(t) * a.H_q + h;
      if (a.splits > 1) {
        const size_t prow = static_cast<size_t>(split) * a.total_q * a.H_q + orow;
        reinterpret_cast<float4 *>(a.part_o + prow * kHeadDim)[d4] = make_float4(0, 0, 0, 0);
        if (d4 == 0) a.part_lse[prow] = -INFINITY;
      } else {
        reinterpret_cast<uint2 *>(a.out + orow * kHeadDim)[d4] = make_uint2(0, 0);
      }
    }
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;
  uint8_t *qs = stages + NS * STAGE;
  uint64_t *full = reinterpret_cast<uint64_t *>(qs + 2 * kQSub);
  uint64_t *empty = full + NS;
  int *st_j = reinterpret_cast<int *>(empty + NS);
  uint32_t *st_mask = reinterpret_cast<uint32_t *>(st_j + NS);
  int *st_ok = reinterpret_cast<int *>(st_mask + NS);
  float *mrg_m = reinterpret_cast<float *>(st_ok + NS);  // [NCW][16]
  float *mrg_l = mrg_m + RG * 4 * 16;                      // [NCW][16]
  float *row_lse = mrg_l + RG * 4 * 16;                    // [RG*16]
  volatile int *abort_flag = reinterpret_cast<volatile int *>(row_lse + RG * 16);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Stage Q (rows x 128) into shared memory, swizzled like the TMA tiles.  For FP8 KV the
  // values become f16 and, inside every 16-dim group, slot 2c+e holds dim 4c+e and slot
  // 2c+8+e holds dim 4c+2+e (c < 4, e < 2): the order in which a plain ldmatrix of an e4m3
  // K tile hands the dims to the MMA, so that both operands agree on k.
  for (int idx = threadIdx.x; idx < kQRows * 8; idx += blockDim.x) {
    const int r = idx >> 3, grp = idx & 7;
    uint4 lo4 = make_uint4(0, 0, 0, 0), hi4 = make_uint4(0, 0, 0, 0);
    if (r < rows) {
      const int t = t0 + r / a.G, h = g * a.G + r % a.G;
      const uint4 *src = reinterpret_cast<const uint4 *>(
          a.q + (static_cast<size_t>(t) * a.H_q + h) * kHeadDim + grp * 16);
      const uint4 x0 = src[0], x1 = src[1];
      if (!FP8) {
        lo4 = x0;
        hi4 = x1;
      } else {
        const uint32_t wv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        float f[16];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          f[2 * k] = __uint_as_float(wv[k] << 16);
          f[2 * k + 1] = __uint_as_float(wv[k] & 0xffff0000u);
        }
        uint32_t o8[8];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          o8[c] = pack_f16x2(f[4 * c], f[4 * c + 1]);
          o8[4 + c] = pack_f16x2(f[4 * c + 2], f[4 * c + 3]);
        }
        lo4 = make_uint4(o8[0], o8[1], o8[2], o8[3]);
        hi4 = make_uint4(o8[4], o8[5], o8[6], o8[7]);
      }
    }
    *reinterpret_cast<uint4 *>(qs + sw128(r, 2 * grp, kQSub)) = lo4;
    *reinterpret_cast<uint4 *>(qs + sw128(r, 2 * grp + 1, kQSub)) = hi4;
  }
  __syncthreads();

  if (warp == NCW) {
    // -------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&vmap);
      for (int i = 0; i < nblk; ++i) {
        const int s = i % NS;
        if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1, abort_flag)) {
          report(a.dev_err, MSA_DEVERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        const int j = list[lo + i];
        const uint32_t m = PLAN ? masks[lo + i] : 0xffffffffu;
        const bool jok = j >= 0 && j < a.max_blocks;
        const int page = jok ? a.table[static_cast<size_t>(b) * a.max_pages + j] : -1;
        const bool ok = jok && page >= 0 && page < a.num_pages;
        st_j[s] = j;
        st_mask[s] = m;
        st_ok[s] = ok;
        if (ok) {
          mbar_arrive_expect_tx(&full[s], 2 * TILE);
          const int c2 = page * a.H_kv + g;
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
      }
    }
    return;
  }

  // ---------------------------------------------------------------- consumers
  const int rg = warp / PQ, pq = warp % PQ;
  const int mi = lane >> 3, rr = lane & 7, c4 = lane & 3;
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

  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

  for (int i = 0; i < nblk; ++i) {
    const int s = i % NS;
    const bool live = mbar_wait(&full[s], (i / NS) & 1, abort_flag);
    if (!live) {
      report(a.dev_err, MSA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
    if (live && st_ok[s]) {
      const int j = st_j[s];
      const uint32_t msk = st_mask[s];
      const uint32_t kt = smem_u32(stages + s * STAGE), vt = kt + TILE;

      // S = Q K^T over this warp's PW positions
      float sc[NTW][4];
#pragma unroll
      for (int n = 0; n < NTW; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[n][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t qa[4];
        ldsm_x4(qs_addr + sw128(rg * 16 + (mi & 1) * 8 + rr, 2 * ks + (mi >> 1), kQSub), qa[0],
                qa[1], qa[2], qa[3]);
        if (FP8) {
#pragma unroll
          for (int h = 0; h < NTW / 4; ++h) {
            uint32_t kr[4];
            ldsm_x4(kt + sw128(pq * PW + h * 32 + mi * 8 + rr, ks, KSUB), kr[0], kr[1], kr[2],
                    kr[3]);
#pragma unroll
            for (int n = 0; n < 4; ++n)
              mma_f16(sc[4 * h + n], qa, e4m3x2_to_f16x2(static_cast<uint16_t>(kr[n] & 0xffffu)),
                      e4m3x2_to_f16x2(static_cast<uint16_t>(kr[n] >> 16)));
          }
        } else {
          uint32_t bf[NTW][2];
#pragma unroll
          for (int h = 0; h < NTW / 2; ++h)
            ldsm_x4(kt + sw128(pq * PW + h * 16 + (mi >> 1) * 8 + rr, 2 * ks + (mi & 1), KSUB),
                    bf[2 * h][0], bf[2 * h][1], bf[2 * h + 1][0], bf[2 * h + 1][1]);
#pragma unroll
          for (int n = 0; n < NTW; ++n) mma_bf16(sc[n], qa, bf[n][0], bf[n][1]);
        }
      }

      // mask (causal per token + the token's own selection) and online softmax, log2 domain
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int n = 0; n < NTW; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int slot = e >> 1;
          const int pos = j * kBlock + pq * PW + n * 8 + 2 * c4 + (e & 1);
          const bool vis = pos <= prow[slot] && (msk & tbit[slot]);
          const float x = vis ? sc[n][e] * a.scale_log2 : -INFINITY;
          sc[n][e] = x;
          mx[slot] = fmaxf(mx[slot], x);
        }
      float alpha[2], base[2];
#pragma unroll
      for (int slot = 0; slot < 2; ++slot) {
        mx[slot] = fmaxf(mx[slot], __shfl_xor_sync(0xffffffffu, mx[slot], 1));
        mx[slot] = fmaxf(mx[slot], __shfl_xor_sync(0xffffffffu, mx[slot], 2));
        const float m_new = fmaxf(m_run[slot], mx[slot]);
        base[slot] = m_new == -INFINITY ? 0.f : m_new;
        alpha[slot] = fast_exp2(m_run[slot] - base[slot]);
        m_run[slot] = m_new;
        l_run[slot] *= alpha[slot];
      }
#pragma unroll
      for (int n = 0; n < NTW; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float pv = fast_exp2(sc[n][e] - base[e >> 1]);
          sc[n][e] = pv;
          l_run[e >> 1] += pv;
        }
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        o[n][0] *= alpha[0];
        o[n][1] *= alpha[0];
        o[n][2] *= alpha[1];
        o[n][3] *= alpha[1];
      }
      // P as the A operand (rows x PW positions = KSW k-steps)
      uint32_t pa[KSW][4];
#pragma unroll
      for (int kk = 0; kk < KSW; ++kk) {
        if (FP8) {
          pa[kk][0] = pack_f16x2(sc[2 * kk][0], sc[2 * kk][1]);
          pa[kk][1] = pack_f16x2(sc[2 * kk][2], sc[2 * kk][3]);
          pa[kk][2] = pack_f16x2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
          pa[kk][3] = pack_f16x2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
        } else {
          pa[kk][0] = pack_bf16x2(sc[2 * kk][0], sc[2 * kk][1]);
          pa[kk][1] = pack_bf16x2(sc[2 * kk][2], sc[2 * kk][3]);
          pa[kk][2] = pack_bf16x2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
          pa[kk][3] = pack_bf16x2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
        }
      }
      // O += P V.  Positions >= L of the sequence's last page hold whatever the pool has
      // there; their P is 0, but 0 * NaN is NaN, so those V values are zeroed first.
      const bool tail = j * kBlock + kBlock > L;
#pragma unroll
      for (int kk = 0; kk < KSW; ++kk) {
        const int p0 = j * kBlock + pq * PW + kk * 16 + 2 * c4;
        const uint32_t keep0 = (p0 < L ? 0x0000ffffu : 0u) | (p0 + 1 < L ? 0xffff0000u : 0u);
        const uint32_t keep1 = (p0 + 8 < L ? 0x0000ffffu : 0u) | (p0 + 9 < L ? 0xffff0000u : 0u);
        const int vrow = pq * PW + kk * 16 + (mi & 1) * 8 + rr;
        if (FP8) {
#pragma unroll
          for (int cp = 0; cp < 4; ++cp) {
            uint32_t r[4];
            ldsm_x4_t(vt + sw128(vrow, 2 * cp + (mi >> 1), KSUB), r[0], r[1], r[2], r[3]);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const uint32_t ra = r[2 * q], rb = r[2 * q + 1];
              uint32_t e0 = e4m3x2_to_f16x2(static_cast<uint16_t>(__byte_perm(ra, 0, 0x0020)));
              uint32_t e1 = e4m3x2_to_f16x2(static_cast<uint16_t>(__byte_perm(rb, 0, 0x0020)));
              uint32_t d0 = e4m3x2_to_f16x2(static_cast<uint16_t>(__byte_perm(ra, 0, 0x0031)));
              uint32_t d1 = e4m3x2_to_f16x2(static_cast<uint16_t>(__byte_perm(rb, 0, 0x0031)));
              if (tail) {
                e0 &= keep0;
                d0 &= keep0;
                e1 &= keep1;
                d1 &= keep1;
              }
              const int ch = 2 * cp + q;
              mma_f16(o[2 * ch], pa[kk], e0, e1);
              mma_f16(o[2 * ch + 1], pa[kk], d0, d1);
            }
          }
        } else {
#pragma unroll
          for (int dp = 0; dp < 8; ++dp) {
            uint32_t r[4];
            ldsm_x4_t(vt + sw128(vrow, 2 * dp + (mi >> 1), KSUB), r[0], r[1], r[2], r[3]);
            if (tail) {
              r[0] &= keep0;
              r[1] &= keep1;
              r[2] &= keep0;
              r[3] &= keep1;
            }
            mma_bf16(o[2 * dp], pa[kk], r[0], r[1]);
            mma_bf16(o[2 * dp + 1], pa[kk], r[2], r[3]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // ---------------------------------------------------------------- merge the PQ position
  // splits of every row group, normalise, write out (or the split-K partial)
#pragma unroll
  for (int slot = 0; slot < 2; ++slot) {
    l_run[slot] += __shfl_xor_sync(0xffffffffu, l_run[slot], 1);
    l_run[slot] += __shfl_xor_sync(0xffffffffu, l_run[slot], 2);
  }
  named_bar_sync(1, NCT);  // every consumer is done with the stages
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  float *mo = reinterpret_cast<float *>(stages);  // [NCW][16][128]
  if (c4 == 0) {
#pragma unroll
    for (int slot = 0; slot < 2; ++slot) {
      mrg_m[warp * 16 + (lane >> 2) + slot * 8] = m_run[slot];
      mrg_l[warp * 16 + (lane >> 2) + slot * 8] = l_run[slot];
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
    const float f = (Ls > 0.f && m_run[slot] != -INFINITY) ? fast_exp2(m_run[slot] - M) / Ls : 0.f;
    float *dst = mo + (static_cast<size_t>(warp) * 16 + r16) * kHeadDim;
    if (FP8) {
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        *reinterpret_cast<float4 *>(dst + ch * 16 + 4 * c4) =
            make_float4(o[2 * ch][2 * slot] * f, o[2 * ch + 1][2 * slot] * f,
                        o[2 * ch][2 * slot + 1] * f, o[2 * ch + 1][2 * slot + 1] * f);
    } else {
#pragma unroll
      for (int n = 0; n < 16; ++n)
        *reinterpret_cast<float2 *>(dst + n * 8 + 2 * c4) =
            make_float2(o[n][2 * slot] * f, o[n][2 * slot + 1] * f);
    }
    if (pq == 0 && c4 == 0)
      row_lse[rg * 16 + r16] = Ls > 0.f ? (M + __log2f(Ls)) * kLn2 : -INFINITY;
  }
  named_bar_sync(1, NCT);
  for (int idx = threadIdx.x; idx < RG * 16 * (kHeadDim / 4); idx += NCT) {
    const int r = idx / (kHeadDim / 4), d4 = idx % (kHeadDim / 4);
    if (r >= rows) continue;
    const int rgr = r >> 4, r16 = r & 15;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < PQ; ++w) {
      const float4 v =
          reinterpret_cast<const float4 *>(mo + (static_cast<size_t>(rgr * PQ + w) * 16 + r16) *
                                                    kHeadDim)[d4];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    const int t = t0 + r / a.G, h = g * a.G + r % a.G;
    const size_t orow = static_cast<size_t>(t) * a.H_q + h;
    if (a.splits > 1) {
      const size_t prow = static_cast<size_t>(split) * a.total_q * a.H_q + orow;
      reinterpret_cast<float4 *>(a.part_o + prow * kHeadDim)[d4] = acc;
      if (d4 == 0) a.part_lse[prow] = row_lse[r];
    } else {
      uint2 packed;
      packed.x = pack_bf16x2(acc.x, acc.y);
      packed.y = pack_bf16x2(acc.z, acc.w);
      reinterpret_cast<uint2 *>(a.out + orow * kHeadDim)[d4] = packed;
    }
  }
}

template <bool FP8, int RG, bool PLAN>
cudaError_t launch_one(const CUtensorMap &kmap, const CUtensorMap &vmap, const AttnArgs &a,
                       cudaStream_t s) {
  const size_t smem = attn_smem_bytes<FP8, RG>();
  auto fn = &attn_kernel<FP8, RG, PLAN>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(fn), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(a.batch * a.tiles, a.H_kv, a.splits);
  fn<<<grid, 32 * (RG * (RG <= 2 ? 4 : 2) + 1), smem, s>>>(kmap, vmap, a);
  return cudaGetLastError();
}

template <bool FP8, bool PLAN>
cudaError_t launch_rg(const CUtensorMap &kmap, const CUtensorMap &vmap, const AttnArgs &a, int rg,
                      cudaStream_t s) {
  switch (rg) {
    case 1: return launch_one<FP8, 1, PLAN>(kmap, vmap, a, s);
    case 2: return launch_one<FP8, 2, PLAN>(kmap, vmap, a, s);
    case 3: return launch_one<FP8, 3, PLAN>(kmap, vmap, a, s);
    default: return launch_one<FP8, 4, PLAN>(kmap, vmap, a, s);
  }
}

}  // namespace

cudaError_t launch_attention(const CUtensorMap &kmap, const CUtensorMap &vmap, const AttnArgs &a,
                             bool fp8, int rg, bool plan, cudaStream_t s) {
  if (fp8)
    return plan ? launch_rg<true, true>(kmap, vmap, a, rg, s)
                : launch_rg<true, false>(kmap, vmap, a, rg, s);
  return plan ? launch_rg<false, true>(kmap, vmap, a, rg, s)
              : launch_rg<false, false>(kmap, vmap, a, rg, s);
}

}  // namespace msa
