// attn_common.cuh — the per-block math of the sparse paged attention, shared by the
// persistent decode / speculative kernel (attention_stream.cu) and the tiled kernel used for
// prefill (attention_tile.cu).
//
// A consumer warp owns 16 query rows (one m16 MMA tile) and PW = 128 / PQ of the 128 positions
// of every block, and keeps its own online-softmax state over them.  Q sits in shared memory
// (swizzled like the TMA tiles), K and V page tiles arrive by TMA with the 128-byte swizzle.
// QK^T and PV run on mma.sync m16n8k16 with FP32 accumulators: bf16 operands for BF16 KV;
// for e4m3 KV the tiles are converted to f16 in registers (exact) and the MMAs take f16
// operands (q rounded to f16, P in f16).
#pragma once

#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace msa {

constexpr int kQRows = 64;                // rows of a Q buffer
constexpr uint32_t kQSub = kQRows * 128;  // one 64-column (bf16/f16) sub-tile of Q
constexpr uint32_t kQBuf = 2 * kQSub;     // one Q buffer
constexpr float kLn2 = 0.69314718055994530942f;

template <bool FP8>
struct KvTile {
  static constexpr uint32_t kBytes = FP8 ? 16384u : 32768u;  // one (page, head) tile
  static constexpr uint32_t kSub = 16384u;                    // one swizzled [128][128 B] box
};

// Stage rows [0, QR) of Q (rows r = tok * G + h_local of one work item) into a Q buffer of
// two swizzled [QR][128 B] sub-tiles (zeros past `rows`).  Threads `tid` of `nthreads` share
// the copy.  For e4m3 KV the values become f16 and, inside every 16-dim group, slot 2c+e holds
// dim 4c+e and slot 2c+8+e holds dim 4c+2+e (c < 4, e < 2): the order in which a plain
// ldmatrix of an e4m3 K tile hands the dims to the MMA, so that both operands agree on k.
template <bool FP8, int QR>
__device__ __forceinline__ void stage_q(uint8_t *qs, const uint16_t *q, int t0, int rows, int G,
                                        int H_q, int g, int tid, int nthreads) {
  constexpr uint32_t sub = QR * 128;
  for (int idx = tid; idx < QR * 8; idx += nthreads) {
    const int r = idx >> 3, grp = idx & 7;
    uint4 lo4 = make_uint4(0, 0, 0, 0), hi4 = make_uint4(0, 0, 0, 0);
    if (r < rows) {
      const int t = t0 + r / G, h = g * G + r % G;
      const uint4 *src = reinterpret_cast<const uint4 *>(
          q + (static_cast<size_t>(t) * H_q + h) * kHeadDim + grp * 16);
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
    *reinterpret_cast<uint4 *>(qs + sw128(r, 2 * grp, sub)) = lo4;
    *reinterpret_cast<uint4 *>(qs + sw128(r, 2 * grp + 1, sub)) = hi4;
  }
}

// Row stride (floats) of the fp32 merge buffers: padded so that the 8 rows a warp's lanes hold
// fall in different banks for the float2 (BF16 layout) and float4 (FP8 layout) accesses.
template <bool FP8>
struct MergeRow {
  static constexpr int kStride = kHeadDim + (FP8 ? 16 : 8);
};

template <bool FP8, int PQ>
struct WarpAttn {
  static constexpr int PW = kBlock / PQ;  // positions per warp
  static constexpr int NTW = PW / 8;      // n8 tiles of S per warp
  static constexpr int KSW = PW / 16;     // k16 steps of PV per warp

  float o[16][4];
  float m_run[2], l_run[2];  // rows lane/4 and lane/4 + 8 (log2 domain)
  float sc[NTW][4];

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int n = 0; n < 16; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
    m_run[0] = m_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.f;
  }

  // sc = Q K^T for the warp's 16 rows (row base qrow0 of a Q buffer whose sub-tiles are
  // qsub bytes) and PW positions.
  __device__ __forceinline__ void qk(uint32_t qs_addr, uint32_t qsub, int qrow0, uint32_t kt,
                                     int pq, int lane) {
    const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
    for (int n = 0; n < NTW; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[n][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t qa[4];
      ldsm_x4(qs_addr + sw128(qrow0 + (mi & 1) * 8 + rr, 2 * ks + (mi >> 1), qsub), qa[0], qa[1],
              qa[2], qa[3]);
      if (FP8) {
#pragma unroll
        for (int h = 0; h < NTW / 4; ++h) {
          uint32_t kr[4];
          ldsm_x4(kt + sw128(pq * PW + h * 32 + mi * 8 + rr, ks, KvTile<FP8>::kSub), kr[0], kr[1],
                  kr[2], kr[3]);
#pragma unroll
          for (int n = 0; n < 4; ++n)
            mma_f16(sc[4 * h + n], qa, e4m3x2_to_f16x2(static_cast<uint16_t>(kr[n] & 0xffffu)),
                    e4m3x2_to_f16x2(static_cast<uint16_t>(kr[n] >> 16)));
        }
      } else {
        uint32_t bf[NTW][2];
#pragma unroll
        for (int h = 0; h < NTW / 2; ++h)
          ldsm_x4(kt + sw128(pq * PW + h * 16 + (mi >> 1) * 8 + rr, 2 * ks + (mi & 1),
                             KvTile<FP8>::kSub),
                  bf[2 * h][0], bf[2 * h][1], bf[2 * h + 1][0], bf[2 * h + 1][1]);
#pragma unroll
        for (int n = 0; n < NTW; ++n) mma_bf16(sc[n], qa, bf[n][0], bf[n][1]);
      }
    }
  }

  // Mask (position <= the row's query position and the row's token selected the block),
  // online-softmax update in the log2 domain; sc becomes P.
  __device__ __forceinline__ void softmax(int j, int pq, int lane, const int (&prow)[2],
                                          const uint32_t (&tbit)[2], uint32_t msk,
                                          float scale_log2) {
    const int c4 = lane & 3;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < NTW; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int slot = e >> 1;
        const int pos = j * kBlock + pq * PW + n * 8 + 2 * c4 + (e & 1);
        const bool vis = pos <= prow[slot] && (msk & tbit[slot]);
        const float x = vis ? sc[n][e] * scale_log2 : -INFINITY;
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
  }

  // O += P V.  Positions >= L (the sequence length) of the last page hold whatever the pool
  // has there; their P is 0, but 0 * NaN is NaN, so those V values are zeroed first.
  __device__ __forceinline__ void pv(uint32_t vt, int j, int pq, int lane, int L) {
    const int mi = lane >> 3, rr = lane & 7, c4 = lane & 3;
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
          ldsm_x4_t(vt + sw128(vrow, 2 * cp + (mi >> 1), KvTile<FP8>::kSub), r[0], r[1], r[2],
                    r[3]);
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
          ldsm_x4_t(vt + sw128(vrow, 2 * dp + (mi >> 1), KvTile<FP8>::kSub), r[0], r[1], r[2],
                    r[3]);
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

  // After the last block: each row's sum of P, reduced over the quad that holds the row.
  __device__ __forceinline__ void finish_rows() {
#pragma unroll
    for (int slot = 0; slot < 2; ++slot) {
      l_run[slot] += __shfl_xor_sync(0xffffffffu, l_run[slot], 1);
      l_run[slot] += __shfl_xor_sync(0xffffffffu, l_run[slot], 2);
    }
  }

  // This thread's part of row slot `slot` times f, as fp32, into row `row` of a merge buffer
  // (rows MergeRow<FP8>::kStride floats apart; the FP8 path's dim permutation is undone
  // here).  With `add` the values are added to what the buffer holds.
  __device__ __forceinline__ void store_row(float *buf, int row, int slot, float f, int lane,
                                            bool add) const {
    const int c4 = lane & 3;
    float *dst = buf + row * MergeRow<FP8>::kStride;
    if (FP8) {
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        float4 *d = reinterpret_cast<float4 *>(dst + ch * 16 + 4 * c4);
        float4 v = make_float4(o[2 * ch][2 * slot] * f, o[2 * ch + 1][2 * slot] * f,
                               o[2 * ch][2 * slot + 1] * f, o[2 * ch + 1][2 * slot + 1] * f);
        if (add) {
          const float4 u = *d;
          v = make_float4(u.x + v.x, u.y + v.y, u.z + v.z, u.w + v.w);
        }
        *d = v;
      }
    } else {
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        float2 *d = reinterpret_cast<float2 *>(dst + n * 8 + 2 * c4);
        float2 v = make_float2(o[n][2 * slot] * f, o[n][2 * slot + 1] * f);
        if (add) {
          const float2 u = *d;
          v = make_float2(u.x + v.x, u.y + v.y);
        }
        *d = v;
      }
    }
  }

  // Fold the state another warp left in shared memory (its output row `row` of `buf`, laid
  // out by store_row, with max m2 and sum l2) into this thread's row slot `slot`.
  __device__ __forceinline__ void merge_row(const float *buf, int row, int slot, float m2,
                                            float l2, int lane) {
    const float m1 = m_run[slot];
    const float m = fmaxf(m1, m2);
    const float a1 = m1 == -INFINITY ? 0.f : fast_exp2(m1 - m);
    const float a2 = m2 == -INFINITY ? 0.f : fast_exp2(m2 - m);
    const int c4 = lane & 3;
    const float *src = buf + row * MergeRow<FP8>::kStride;
    if (FP8) {
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const float4 u = *reinterpret_cast<const float4 *>(src + ch * 16 + 4 * c4);
        o[2 * ch][2 * slot] = o[2 * ch][2 * slot] * a1 + u.x * a2;
        o[2 * ch + 1][2 * slot] = o[2 * ch + 1][2 * slot] * a1 + u.y * a2;
        o[2 * ch][2 * slot + 1] = o[2 * ch][2 * slot + 1] * a1 + u.z * a2;
        o[2 * ch + 1][2 * slot + 1] = o[2 * ch + 1][2 * slot + 1] * a1 + u.w * a2;
      }
    } else {
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        const float2 u = *reinterpret_cast<const float2 *>(src + n * 8 + 2 * c4);
        o[n][2 * slot] = o[n][2 * slot] * a1 + u.x * a2;
        o[n][2 * slot + 1] = o[n][2 * slot + 1] * a1 + u.y * a2;
      }
    }
    l_run[slot] = l_run[slot] * a1 + l2 * a2;
    m_run[slot] = m;
  }

  // This thread's part of row slot `slot` times f, as bf16 in natural dim order, into a
  // 128-dim row of global memory.
  __device__ __forceinline__ void store_bf16(uint16_t *dst, int slot, float f, int lane) const {
    const int c4 = lane & 3;
    if (FP8) {
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        *reinterpret_cast<uint2 *>(dst + ch * 16 + 4 * c4) =
            make_uint2(pack_bf16x2(o[2 * ch][2 * slot] * f, o[2 * ch + 1][2 * slot] * f),
                       pack_bf16x2(o[2 * ch][2 * slot + 1] * f, o[2 * ch + 1][2 * slot + 1] * f));
    } else {
#pragma unroll
      for (int n = 0; n < 16; ++n)
        *reinterpret_cast<uint32_t *>(dst + n * 8 + 2 * c4) =
            pack_bf16x2(o[n][2 * slot] * f, o[n][2 * slot + 1] * f);
    }
  }
  // This thread's part of row slot `slot` times f, as fp32 in natural dim order, into a
  // 128-dim row of global memory.
  __device__ __forceinline__ void store_global(float *dst, int slot, float f, int lane) const {
    const int c4 = lane & 3;
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
  }
};


// ---- decode math with the operands swapped (at most 8 query rows)
//
// A decode item has one query token, so its rows are the G <= 8 heads of one KV head and an
// m16 tile of query rows is at least half padding.  Here the MMAs run transposed: S^T = K Q^T
// takes 16 of the block's positions as M and the query rows as N (n8), and O^T += V^T P^T takes
// 16 head dims as M, the rows as N and the positions as K, so no MMA computes padding and the
// softmax touches half the values.  P^T moves from the C layout of S^T to the B layout of the
// P V MMA through movmatrix (an 8x8 transpose in registers).  Lane (g, c) = (lane / 4,
// lane % 4) holds query rows 2c and 2c + 1; its online-softmax state covers its own positions
// (the max is reduced over the eight lanes of the same c, the sum at finish_rows).
// For e4m3 KV the K rows arrive in the same per-16-dim order as stage_q gives Q, and the V^T
// tiles of 32 dims split into an even-dim and an odd-dim m16 tile (dim_lo / dim_hi say which
// dims a lane's accumulators hold).
template <bool FP8, int PQ>
struct WarpAttnSwap {
  static constexpr int PW = kBlock / PQ;  // positions per warp
  static constexpr int MT = PW / 16;      // m16 tiles of S^T per warp

  float o[8][4];  // O^T tile t: [s] = (dim_lo(t), row 2c + s), [2 + s] = (dim_hi(t), row 2c + s)
  float m_run[2], l_run[2];  // rows 2c and 2c + 1 (log2 domain)
  float st[MT][4];           // S^T, then P^T: [s] = (position g, row 2c + s), [2 + s] = (g + 8, .)
  uint32_t qb[8][2];         // Q^T B fragments of the eight k16 steps

  __device__ static __forceinline__ int dim_lo(int t, int g) {
    return FP8 ? 32 * (t >> 1) + 2 * g + (t & 1) : 16 * t + g;
  }
  __device__ static __forceinline__ int dim_hi(int t, int g) {
    return dim_lo(t, g) + (FP8 ? 16 : 8);
  }

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int t = 0; t < 8; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[t][e] = 0.f;
    m_run[0] = m_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.f;
  }

  // Q rows 0..7 of a Q buffer (sub-tiles qsub bytes apart) as the B operand of every k step.
  __device__ __forceinline__ void load_q(uint32_t qs_addr, uint32_t qsub, int lane) {
    const int r = lane & 7, hi = (lane >> 3) & 1;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
      ldsm_x2(qs_addr + sw128(r, 2 * ks + hi, qsub), qb[ks][0], qb[ks][1]);
  }

  // st = K Q^T over the warp's PW positions (the Q arguments are those of WarpAttn::qk; the
  // fragments come from load_q).
  __device__ __forceinline__ void qk(uint32_t, uint32_t, int, uint32_t kt, int pq, int lane) {
    const int q = lane >> 3, r = lane & 7;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) st[mt][e] = 0.f;
      const int row = pq * PW + mt * 16 + (q & 1) * 8 + r;  // the position this lane addresses
      if (FP8) {
#pragma unroll
        for (int jd = 0; jd < 4; ++jd) {  // 32 dims (two k steps) per load
          uint32_t kr[4];
          ldsm_x4(kt + sw128(row, 2 * jd + (q >> 1), KvTile<FP8>::kSub), kr[0], kr[1], kr[2],
                  kr[3]);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t a[4] = {
                e4m3x2_to_f16x2(static_cast<uint16_t>(kr[2 * h] & 0xffffu)),
                e4m3x2_to_f16x2(static_cast<uint16_t>(kr[2 * h + 1] & 0xffffu)),
                e4m3x2_to_f16x2(static_cast<uint16_t>(kr[2 * h] >> 16)),
                e4m3x2_to_f16x2(static_cast<uint16_t>(kr[2 * h + 1] >> 16))};
            mma_f16(st[mt], a, qb[2 * jd + h][0], qb[2 * jd + h][1]);
          }
        }
      } else {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          uint32_t a[4];
          ldsm_x4(kt + sw128(row, 2 * ks + (q >> 1), KvTile<FP8>::kSub), a[0], a[1], a[2], a[3]);
          mma_bf16(st[mt], a, qb[ks][0], qb[ks][1]);
        }
      }
    }
  }

  // Mask (position <= the row's query position, the row's token selected the block) and the
  // online-softmax update in the log2 domain; st becomes P^T.
  __device__ __forceinline__ void softmax(int j, int pq, int lane, const int (&prow)[2],
                                          const uint32_t (&tbit)[2], uint32_t msk,
                                          float scale_log2) {
    const int g = lane >> 2;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int s = e & 1;
        const int pos = j * kBlock + pq * PW + mt * 16 + g + (e >> 1) * 8;
        const bool vis = pos <= prow[s] && (msk & tbit[s]);
        const float x = vis ? st[mt][e] * scale_log2 : -INFINITY;
        st[mt][e] = x;
        mx[s] = fmaxf(mx[s], x);
      }
    float alpha[2], base[2];
#pragma unroll
    for (int s = 0; s < 2; ++s) {
#pragma unroll
      for (int off = 4; off < 32; off <<= 1)
        mx[s] = fmaxf(mx[s], __shfl_xor_sync(0xffffffffu, mx[s], off));
      const float m_new = fmaxf(m_run[s], mx[s]);
      base[s] = m_new == -INFINITY ? 0.f : m_new;
      alpha[s] = fast_exp2(m_run[s] - base[s]);
      m_run[s] = m_new;
      l_run[s] *= alpha[s];
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float pv = fast_exp2(st[mt][e] - base[e & 1]);
        st[mt][e] = pv;
        l_run[e & 1] += pv;
      }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      o[t][0] *= alpha[0];
      o[t][1] *= alpha[1];
      o[t][2] *= alpha[0];
      o[t][3] *= alpha[1];
    }
  }

  // O^T += V^T P^T.  V values at positions >= L (the sequence length) are zeroed first (P is 0
  // there, but the pool may hold NaN).
  __device__ __forceinline__ void pv(uint32_t vt, int j, int pq, int lane, int L) {
    const int c = lane & 3, q = lane >> 3, r = lane & 7;
    const bool tail = j * kBlock + kBlock > L;
#pragma unroll
    for (int kk = 0; kk < MT; ++kk) {
      uint32_t x0, x1;
      if (FP8) {
        x0 = pack_f16x2(st[kk][0], st[kk][1]);
        x1 = pack_f16x2(st[kk][2], st[kk][3]);
      } else {
        x0 = pack_bf16x2(st[kk][0], st[kk][1]);
        x1 = pack_bf16x2(st[kk][2], st[kk][3]);
      }
      const uint32_t b0 = movmatrix_t(x0), b1 = movmatrix_t(x1);  // (positions 2c.., row g)
      const int p0 = j * kBlock + pq * PW + kk * 16 + 2 * c;
      const uint32_t keep0 = (p0 < L ? 0x0000ffffu : 0u) | (p0 + 1 < L ? 0xffff0000u : 0u);
      const uint32_t keep1 = (p0 + 8 < L ? 0x0000ffffu : 0u) | (p0 + 9 < L ? 0xffff0000u : 0u);
      const int vrow = pq * PW + kk * 16 + (q >> 1) * 8 + r;  // the position this lane addresses
      if (FP8) {
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {  // dims 32 qd .. 32 qd + 31
          uint32_t rr[4];
          ldsm_x4_t(vt + sw128(vrow, 2 * qd + (q & 1), KvTile<FP8>::kSub), rr[0], rr[1], rr[2],
                    rr[3]);
#pragma unroll
          for (int sd = 0; sd < 2; ++sd) {  // even, odd dims
            const uint32_t sel = sd ? 0x0031u : 0x0020u;
            uint32_t a[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              a[i] = e4m3x2_to_f16x2(static_cast<uint16_t>(__byte_perm(rr[i], 0, sel)));
            if (tail) {
              a[0] &= keep0;
              a[1] &= keep0;
              a[2] &= keep1;
              a[3] &= keep1;
            }
            mma_f16(o[2 * qd + sd], a, b0, b1);
          }
        }
      } else {
#pragma unroll
        for (int d = 0; d < 8; ++d) {  // dims 16 d .. 16 d + 15
          uint32_t a[4];
          ldsm_x4_t(vt + sw128(vrow, 2 * d + (q & 1), KvTile<FP8>::kSub), a[0], a[1], a[2],
                    a[3]);
          if (tail) {
            a[0] &= keep0;
            a[1] &= keep0;
            a[2] &= keep1;
            a[3] &= keep1;
          }
          mma_bf16(o[d], a, b0, b1);
        }
      }
    }
  }

  // After the last block: each row's sum of P over all of the warp's positions.
  __device__ __forceinline__ void finish_rows() {
#pragma unroll
    for (int s = 0; s < 2; ++s)
#pragma unroll
      for (int off = 4; off < 32; off <<= 1)
        l_run[s] += __shfl_xor_sync(0xffffffffu, l_run[s], off);
  }

  // Rows 2c and 2c + 1 times f[0] / f[1], as fp32 rows of buf (kStride floats apart, natural
  // dim order), and (from the lanes with g == 0) their m and l after the 16 rows.
  __device__ __forceinline__ void store_rows(float *buf, const float (&f)[2], int lane) const {
    constexpr int MS = MergeRow<FP8>::kStride;
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      float *row = buf + (2 * c + s) * MS;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        row[dim_lo(t, g)] = o[t][s] * f[s];
        row[dim_hi(t, g)] = o[t][2 + s] * f[s];
      }
      if (g == 0) {
        buf[16 * MS + 2 * c + s] = m_run[s];
        buf[16 * MS + 16 + 2 * c + s] = l_run[s];
      }
    }
  }

  // Fold another warp's state, left in buf by store_rows (f = 1), into this lane's rows.
  __device__ __forceinline__ void merge_rows(const float *buf, int lane) {
    constexpr int MS = MergeRow<FP8>::kStride;
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const float m2 = buf[16 * MS + 2 * c + s], l2 = buf[16 * MS + 16 + 2 * c + s];
      const float m1 = m_run[s];
      const float m = fmaxf(m1, m2);
      const float a1 = m1 == -INFINITY ? 0.f : fast_exp2(m1 - m);
      const float a2 = m2 == -INFINITY ? 0.f : fast_exp2(m2 - m);
      const float *row = buf + (2 * c + s) * MS;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        o[t][s] = o[t][s] * a1 + row[dim_lo(t, g)] * a2;
        o[t][2 + s] = o[t][2 + s] * a1 + row[dim_hi(t, g)] * a2;
      }
      l_run[s] = l_run[s] * a1 + l2 * a2;
      m_run[s] = m;
    }
  }
};

}  // namespace msa
