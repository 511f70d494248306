// Warp-level 16-row attention tiles on mma.sync (m16n8k16, bf16 -> fp32).
//
// Used where one query token's GQA group supplies the rows (G <= 16 heads,
// padded to 16): the selected-block branch of the prefill and every decode
// branch. K and V tiles of 64 keys sit in shared memory exactly as a 3-D TMA
// box with 128-byte swizzle leaves them: D/64 boxes of [64 keys][64 elements],
// 8 KB each, rows of 128 bytes.
#pragma once

#include "common.cuh"

namespace nsa {

// A fragments of Q (rows = heads of the group, zero above G).
template <int DK>
__device__ __forceinline__ void load_q_frags(uint32_t (&qa)[DK / 16][4], const __nv_bfloat16* q, int G,
                                             int lane) {
  const int r0 = lane >> 2, cq = (lane & 3) * 2;
#pragma unroll
  for (int kk = 0; kk < DK / 16; ++kk) {
    const int c = kk * 16 + cq;
    qa[kk][0] = r0 < G ? *reinterpret_cast<const uint32_t*>(q + (size_t)r0 * DK + c) : 0u;
    qa[kk][1] = r0 + 8 < G ? *reinterpret_cast<const uint32_t*>(q + (size_t)(r0 + 8) * DK + c) : 0u;
    qa[kk][2] = r0 < G ? *reinterpret_cast<const uint32_t*>(q + (size_t)r0 * DK + c + 8) : 0u;
    qa[kk][3] = r0 + 8 < G ? *reinterpret_cast<const uint32_t*>(q + (size_t)(r0 + 8) * DK + c + 8) : 0u;
  }
}

// s[nt][*] = raw scores of the 16 rows against keys nt*8 .. nt*8+7 of the tile.
// Fragment layout: s[nt][0..1] row lane/4, keys nt*8 + (lane%4)*2 + {0,1};
// s[nt][2..3] row lane/4 + 8, same keys.
template <int DK>
__device__ __forceinline__ void warp_qk(const uint32_t (&qa)[DK / 16][4], uint32_t kbase, float (&s)[8][4],
                                        int lane) {
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
  const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
  for (int kk = 0; kk < DK / 16; ++kk) {
    const uint32_t box = kbase + (kk >> 2) * 8192;
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      const int key = np * 16 + (mi >> 1) * 8 + rr;
      const int chunk = (kk & 3) * 2 + (mi & 1);
      uint32_t bfr[4];
      ldmatrix_x4(bfr, box + sw128(key, chunk));
      mma_bf16_16816(s[2 * np], qa[kk], bfr);
      mma_bf16_16816(s[2 * np + 1], qa[kk], bfr + 2);
    }
  }
}

// Same as warp_qk with Q read from shared memory (TMA box [rows][64] per 64-wide
// chunk, 128-byte swizzle, chunks `qchunk` bytes apart); rows qrow0 .. qrow0+15;
// the key tile has NT*8 keys (K boxes of [NT*8 keys][64], NT*1 KB apart).
template <int DK, int NT = 8>
__device__ __forceinline__ void warp_qk_sq(uint32_t qbase, uint32_t qchunk, int qrow0, uint32_t kbase,
                                           float (&s)[NT][4], int lane) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
  const int mi = lane >> 3, rr = lane & 7;
  const uint32_t qrow = (uint32_t)(qrow0 + (lane & 15));
#pragma unroll
  for (int kk = 0; kk < DK / 16; ++kk) {
    uint32_t qa[4];
    ldmatrix_x4(qa, qbase + (kk >> 2) * qchunk + sw128(qrow, (kk & 3) * 2 + (lane >> 4)));
    const uint32_t box = kbase + (kk >> 2) * (NT * 1024);
#pragma unroll
    for (int np = 0; np < NT / 2; ++np) {
      const int key = np * 16 + (mi >> 1) * 8 + rr;
      const int chunk = (kk & 3) * 2 + (mi & 1);
      uint32_t bfr[4];
      ldmatrix_x4(bfr, box + sw128(key, chunk));
      mma_bf16_16816(s[2 * np], qa, bfr);
      mma_bf16_16816(s[2 * np + 1], qa, bfr + 2);
    }
  }
}

// warp_qk_sq with the K reduction split over two independent accumulator sets
// (even / odd 16-wide steps), halving the dependent MMA chain.
template <int DK, int NT = 8>
__device__ __forceinline__ void warp_qk_sq2(uint32_t qbase, uint32_t qchunk, int qrow0, uint32_t kbase,
                                            float (&s)[NT][4], int lane) {
  float s2[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[nt][e] = s2[nt][e] = 0.f;
  const int mi = lane >> 3, rr = lane & 7;
  const uint32_t qrow = (uint32_t)(qrow0 + (lane & 15));
#pragma unroll
  for (int kk = 0; kk < DK / 16; ++kk) {
    uint32_t qa[4];
    ldmatrix_x4(qa, qbase + (kk >> 2) * qchunk + sw128(qrow, (kk & 3) * 2 + (lane >> 4)));
    const uint32_t box = kbase + (kk >> 2) * (NT * 1024);
#pragma unroll
    for (int np = 0; np < NT / 2; ++np) {
      const int key = np * 16 + (mi >> 1) * 8 + rr;
      const int chunk = (kk & 3) * 2 + (mi & 1);
      uint32_t bfr[4];
      ldmatrix_x4(bfr, box + sw128(key, chunk));
      if (kk & 1) {
        mma_bf16_16816(s2[2 * np], qa, bfr);
        mma_bf16_16816(s2[2 * np + 1], qa, bfr + 2);
      } else {
        mma_bf16_16816(s[2 * np], qa, bfr);
        mma_bf16_16816(s[2 * np + 1], qa, bfr + 2);
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[nt][e] += s2[nt][e];
}

// o += P V for one tile of NT*8 keys, P given as fp32 probabilities in the
// score layout; V boxes of [NT*8 keys][64 dv], NT*1 KB apart.
template <int DV, int NT = 8>
__device__ __forceinline__ void warp_pv(const float (&p)[NT][4], uint32_t vbase, float (&o)[DV / 8][4], int lane) {
  const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
  for (int kk = 0; kk < NT / 2; ++kk) {
    uint32_t pa[4];
    pa[0] = pack_bf16x2(p[2 * kk][0], p[2 * kk][1]);
    pa[1] = pack_bf16x2(p[2 * kk][2], p[2 * kk][3]);
    pa[2] = pack_bf16x2(p[2 * kk + 1][0], p[2 * kk + 1][1]);
    pa[3] = pack_bf16x2(p[2 * kk + 1][2], p[2 * kk + 1][3]);
#pragma unroll
    for (int np = 0; np < DV / 16; ++np) {
      const int key = kk * 16 + (mi & 1) * 8 + rr;
      const int c16 = np * 2 + (mi >> 1);
      uint32_t bfr[4];
      ldmatrix_x4_trans(bfr, vbase + (c16 >> 3) * (NT * 1024) + sw128(key, c16 & 7));
      mma_bf16_16816(o[2 * np], pa, bfr);
      mma_bf16_16816(o[2 * np + 1], pa, bfr + 2);
    }
  }
}

__device__ __forceinline__ float quad_max(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
  return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}
__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

// Online-softmax state of the two rows a lane holds.
template <int DV>
struct RowState {
  float o[DV / 8][4];
  float m[2], l[2];   // l: this lane's partial sum (quad-reduce before use)
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int i = 0; i < DV / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    m[0] = m[1] = -1e30f;
    l[0] = l[1] = 0.f;
  }
  // x: scaled scores (log2 domain, -inf where masked); turns x into
  // probabilities relative to the new running max and rescales o and l.
  template <int NT>
  __device__ __forceinline__ void update(float (&x)[NT][4]) {
    float mx0 = -1e30f, mx1 = -1e30f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      mx0 = fmaxf(mx0, fmaxf(x[nt][0], x[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(x[nt][2], x[nt][3]));
    }
    mx0 = quad_max(mx0);
    mx1 = quad_max(mx1);
    const float mn0 = fmaxf(m[0], mx0), mn1 = fmaxf(m[1], mx1);
    const float al0 = ex2(m[0] - mn0), al1 = ex2(m[1] - mn1);
    m[0] = mn0;
    m[1] = mn1;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      x[nt][0] = ex2(x[nt][0] - mn0);
      x[nt][1] = ex2(x[nt][1] - mn0);
      x[nt][2] = ex2(x[nt][2] - mn1);
      x[nt][3] = ex2(x[nt][3] - mn1);
      s0 += x[nt][0] + x[nt][1];
      s1 += x[nt][2] + x[nt][3];
    }
    l[0] = l[0] * al0 + s0;
    l[1] = l[1] * al1 + s1;
#pragma unroll
    for (int i = 0; i < DV / 8; ++i) {
      o[i][0] *= al0;
      o[i][1] *= al0;
      o[i][2] *= al1;
      o[i][3] *= al1;
    }
  }
  __device__ __forceinline__ void finish() {
    l[0] = quad_sum(l[0]);
    l[1] = quad_sum(l[1]);
  }
  // write rows (o, m, l) to a [16][DV + 2] fp32 staging area
  __device__ __forceinline__ void stage(float* dst, int lane) const {
    const int r0 = lane >> 2, cq = (lane & 3) * 2;
#pragma unroll
    for (int i = 0; i < DV / 8; ++i) {
      dst[r0 * (DV + 2) + i * 8 + cq] = o[i][0];
      dst[r0 * (DV + 2) + i * 8 + cq + 1] = o[i][1];
      dst[(r0 + 8) * (DV + 2) + i * 8 + cq] = o[i][2];
      dst[(r0 + 8) * (DV + 2) + i * 8 + cq + 1] = o[i][3];
    }
    if ((lane & 3) == 0) {
      dst[r0 * (DV + 2) + DV] = m[0];
      dst[r0 * (DV + 2) + DV + 1] = l[0];
      dst[(r0 + 8) * (DV + 2) + DV] = m[1];
      dst[(r0 + 8) * (DV + 2) + DV + 1] = l[1];
    }
  }
};

}  // namespace nsa
