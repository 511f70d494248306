// NSA decode: one new query per sequence at position L-1 against a KV cache.
//
// Same five steps as the prefill ("Разреженное внимание — NSA и DSA",
// ai.flicky.cc, section "NSA: три ветви"; the cache holds the new token), laid
// out as coalesced HBM streaming: decode reads every compressed key once and the
// raw keys of the selected blocks and the window once, so the bound is HBM
// bandwidth. Every KV tile is loaded once per GQA group (TMA, 64 keys) and
// consumed by mma.sync with the group's heads as the 16 rows.
//
//   D1  split-K over the compressed cache, 512 keys per CTA: per-chunk online
//       softmax state (o, m, l) per head, and per 64-key tile the block sums
//       sum_i exp(s_i - m_ref) * omega(i, j) of the selection blocks it touches.
//   D2  per (sequence, KV head): merge the chunks, normalise, finish
//       g_cmp * o_cmp, reduce the block sums over the group's heads into the
//       importance, run the top-n selection.
//   D3  split over the union of selected blocks and window blocks, 4 blocks per
//       CTA: one score tile serves both branches, each with its own softmax. The
//       last CTA of each (sequence, KV head) to finish (atomic counter, no
//       waiting) merges the partials and writes
//       out = g_cmp o_cmp + g_slc o_slc + g_win o_win.
#include "common.cuh"
#include "kernels.h"
#include "topn.cuh"
#include "warp_mma.cuh"

namespace nsa {

namespace {

constexpr int kDecStages = 4;
constexpr int kDecConsumers = 4;
constexpr int kDecThreads = (kDecConsumers + 1) * 32;
constexpr int kCmpChunk = 512;         // compressed keys per D1 CTA
constexpr int kTilesPerChunk = kCmpChunk / 64;
constexpr int kFineBlocks = 4;         // 64-key blocks per D3 CTA
constexpr int kTP = 18;                // tile partial: m_ref + 17 block sums

template <int DK, int DV>
struct DecSmem {
  static constexpr int K_BYTES = 64 * DK * 2;
  static constexpr int V_BYTES = 64 * DV * 2;
  static constexpr int STAGE = K_BYTES + V_BYTES;
  static constexpr int RING = kDecStages * STAGE;
  static constexpr int MERGE = 2 * kDecConsumers * 16 * (DV + 2) * 4;
  static constexpr int PSCR = kDecConsumers * 16 * 64 * 4;   // probabilities for block sums
  static constexpr int BODY = (RING > MERGE ? RING : MERGE);
  static constexpr int TOTAL = 1024 + BODY + PSCR + 1024;
};

__device__ __forceinline__ int n_cmp_dev(int L, int l, int s) { return L >= l ? (L - l) / s + 1 : 0; }

struct PartLayout {
  // offsets in floats; every row of DV floats starts 16-byte aligned
  size_t cp_o, cp_ml, tp, fp_o, fp_ml, cnt, total;
  int n_tiles;
};
__host__ __device__ inline PartLayout part_layout(const DecodeArgs& a) {
  PartLayout p;
  const size_t BG = (size_t)a.B * a.H_kv;
  p.n_tiles = a.n_cmp_chunks * kTilesPerChunk;
  p.cp_o = 0;                                                      // [BG][nch][G][DV]
  p.cp_ml = p.cp_o + BG * a.n_cmp_chunks * a.G * a.d_v;            // [BG][nch][G][2]
  p.tp = p.cp_ml + BG * a.n_cmp_chunks * a.G * 2;                  // [BG][tiles][18][G]
  p.tp = (p.tp + 3) & ~size_t(3);
  p.fp_o = p.tp + BG * p.n_tiles * kTP * a.G;                      // [BG][nsw][2][G][DV]
  p.fp_ml = p.fp_o + BG * a.n_sw_chunks * 2 * a.G * a.d_v;         // [BG][nsw][2][G][2]
  p.cnt = p.fp_ml + BG * a.n_sw_chunks * 2 * a.G * 2;              // [BG] int counters
  p.total = p.cnt + BG;
  return p;
}

// merge 4 staged warp states ([w][16][DV+2]) into one state per row < G:
// o relative to the merged max M -> dst_o[row][DV], (M, L) -> dst_ml[row][2]
template <int DV>
__device__ __forceinline__ void merge_warps(const float* stg, int G, float* dst_o, float* dst_ml, int tid) {
  const int per_row = (kDecConsumers * 32) / 16;
  const int row = tid / per_row, part = tid % per_row;
  if (row >= G) return;
  float M = -1e30f;
  for (int w = 0; w < kDecConsumers; ++w) M = fmaxf(M, stg[(w * 16 + row) * (DV + 2) + DV]);
  float f[kDecConsumers], Ls = 0.f;
  for (int w = 0; w < kDecConsumers; ++w) {
    const float* r = stg + (w * 16 + row) * (DV + 2);
    f[w] = r[DV + 1] > 0.f ? exp2f(r[DV] - M) : 0.f;
    Ls += f[w] * r[DV + 1];
  }
  const int span = DV / per_row;
  for (int c = part * span; c < (part + 1) * span; ++c) {
    float v = 0.f;
    for (int w = 0; w < kDecConsumers; ++w) v += f[w] * stg[(w * 16 + row) * (DV + 2) + c];
    dst_o[row * DV + c] = v;
  }
  if (part == 0) {
    dst_ml[row * 2 + 0] = M;
    dst_ml[row * 2 + 1] = Ls;
  }
}

}  // namespace

size_t decode_partials_floats(const DecodeArgs& a) { return part_layout(a).total; }

// ---------------------------------------------------------------------------
// D1: compressed keys, split-K
// ---------------------------------------------------------------------------
template <int DK, int DV>
__global__ void __launch_bounds__(kDecThreads, 1) dec_cmp_kernel(const DecodeArgs a,
                                                                 const __grid_constant__ DecodeMaps mp) {
  using S = DecSmem<DK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  float* pscr = reinterpret_cast<float*>(smem + S::BODY);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::BODY + S::PSCR);
  uint64_t* empty = full + kDecStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kDecStages);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int L = a.lens[b];
  if (L < 1 || L > a.max_len) {
    if (tid == 0 && chunk == 0 && g == 0) atomicOr(a.status, DEV_ERR_BOUNDS);
    return;
  }
  const int nc = n_cmp_dev(L, a.l, a.s);
  const int c0 = chunk * kCmpChunk;
  if (c0 >= nc) return;
  const int ntl = min(kTilesPerChunk, (nc - c0 + 63) / 64);
  const int G = a.G;
  const PartLayout pl = part_layout(a);

  if (tid == 0) {
    for (int i = 0; i < kDecStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kDecConsumers) {
    if (lane == 0) {
      const int row0 = b * a.Lmax_cmp + c0;
      for (int i = 0; i < ntl; ++i) {
        const int st = i % kDecStages;
        if (i >= kDecStages && !mbar_wait(&empty[st], ((i / kDecStages) - 1) & 1, abort_flag, a.status, 401)) break;
        uint8_t* Ks = ring + st * S::STAGE;
        mbar_arrive_expect_tx(&full[st], S::STAGE);
        for (int kb = 0; kb < DK / 64; ++kb) tma_load_3d(Ks + kb * 8192, &mp.kc, &full[st], kb * 64, g, row0 + i * 64);
        for (int vb = 0; vb < DV / 64; ++vb)
          tma_load_3d(Ks + S::K_BYTES + vb * 8192, &mp.vc, &full[st], vb * 64, g, row0 + i * 64);
      }
    }
  } else {
    uint32_t qa[DK / 16][4];
    RowState<DV> rs;
    rs.init();
    const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(a.q) + ((size_t)b * a.H_q + (size_t)g * G) * DK;
    load_q_frags<DK>(qa, qp, G, lane);
    float* ps = pscr + warp * 16 * 64;
    for (int i = warp; i < ntl; i += kDecConsumers) {
      const int st = i % kDecStages;
      if (!mbar_wait(&full[st], (i / kDecStages) & 1, abort_flag, a.status, 402)) break;
      const uint32_t kb = smem_u32(ring + st * S::STAGE);
      float s[8][4];
      warp_qk<DK>(qa, kb, s, lane);
      const int kc0 = c0 + i * 64 + (lane & 3) * 2;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool vis = kc0 + nt * 8 + e < nc;
          s[nt][e] = vis ? s[nt][e] * a.scale_log2 : -INFINITY;
          s[nt][2 + e] = vis ? s[nt][2 + e] * a.scale_log2 : -INFINITY;
        }
      }
      rs.update(s);   // s now holds exp2(x - m) for the running max m
      // stage probabilities for the block sums of this tile
      {
        const int r0 = lane >> 2, cq = (lane & 3) * 2;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          ps[r0 * 64 + nt * 8 + cq] = s[nt][0];
          ps[r0 * 64 + nt * 8 + cq + 1] = s[nt][1];
          ps[(r0 + 8) * 64 + nt * 8 + cq] = s[nt][2];
          ps[(r0 + 8) * 64 + nt * 8 + cq + 1] = s[nt][3];
        }
      }
      warp_pv<DV>(s, kb + S::K_BYTES, rs.o, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      // block sums: compressed key 4q+u covers tokens [16(4q+u), +32): u<3 -> 2p
      // into block q of the tile, u = 3 -> p into q and q+1 (17 relative blocks).
      // Tile partial layout [18][G]: row 0 = reference max per head, rows 1..17 =
      // block sums per head.
      {
        const int tile = (c0 / 64) + i;
        float* tpb = a.part + pl.tp + (((size_t)b * a.H_kv + g) * pl.n_tiles + tile) * kTP * G;
        const int row = lane >> 1, half = lane & 1;
        if (row < G) {
          const float* pr = ps + row * 64;
          const int q0 = half * 8;
          for (int q = q0; q < q0 + 8; ++q) {
            float v = 2.f * (pr[4 * q] + pr[4 * q + 1] + pr[4 * q + 2]) + pr[4 * q + 3];
            if (q > 0) v += pr[4 * q - 1];
            tpb[(1 + q) * G + row] = v;
          }
          if (half == 1) tpb[17 * G + row] = pr[63];
        }
        if ((lane & 3) == 0) {
          const int r0 = lane >> 2;
          if (r0 < G) tpb[r0] = rs.m[0];
          if (r0 + 8 < G) tpb[r0 + 8] = rs.m[1];
        }
      }
      __syncwarp();
    }
    rs.finish();
    named_bar_sync(1, kDecConsumers * 32);
    float* stg = reinterpret_cast<float*>(ring);
    rs.stage(stg + warp * 16 * (DV + 2), lane);
    named_bar_sync(1, kDecConsumers * 32);
    const size_t ci = ((size_t)b * a.H_kv + g) * a.n_cmp_chunks + chunk;
    merge_warps<DV>(stg, G, a.part + pl.cp_o + ci * G * DV, a.part + pl.cp_ml + ci * G * 2, tid);
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// D2: merge compressed chunks, importance, selection (one CTA per (b, g))
// ---------------------------------------------------------------------------
constexpr int kSelThreadsD2 = 256;

template <int DV, int PER>
__global__ void __launch_bounds__(kSelThreadsD2) dec_select_kernel(const DecodeArgs a) {
  extern __shared__ float sm[];
  const int g = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int G = a.G;
  const int L = a.lens[b];
  if (L < 1 || L > a.max_len) return;
  const int nc = n_cmp_dev(L, a.l, a.s);
  const int nch = (nc + kCmpChunk - 1) / kCmpChunk;
  const int ntl = (nc + 63) / 64;
  const int t = L - 1;
  const int jt = t / a.ls;
  const PartLayout pl = part_layout(a);
  const size_t bg = (size_t)b * a.H_kv + g;
  float* Mh = sm;                           // [16]
  float* Li = sm + 16;                      // [16] 1/L
  float* Fc = sm + 32;                      // [nch][16]   chunk factors
  float* Ft = Fc + a.n_cmp_chunks * 16;     // [ntl][16]   tile factors (incl. 1/L)
  float* imp_s = Ft + pl.n_tiles * 16;      // [nb_stride]
  const float* cpo = a.part + pl.cp_o + bg * a.n_cmp_chunks * G * DV;
  const float* cpm = a.part + pl.cp_ml + bg * a.n_cmp_chunks * G * 2;
  const float* tp = a.part + pl.tp + bg * pl.n_tiles * kTP * G;
  if (tid == 0) reinterpret_cast<int*>(a.part + pl.cnt)[bg] = 0;   // D3 completion counter
  if (tid < G) {
    float M = -1e30f;
    for (int c = 0; c < nch; ++c)
      if (cpm[(c * G + tid) * 2 + 1] > 0.f) M = fmaxf(M, cpm[(c * G + tid) * 2]);
    float Ls = 0.f;
    for (int c = 0; c < nch; ++c) {
      const float l = cpm[(c * G + tid) * 2 + 1];
      const float f = l > 0.f ? exp2f(cpm[(c * G + tid) * 2] - M) : 0.f;
      Fc[c * 16 + tid] = f;
      Ls += f * l;
    }
    Mh[tid] = M;
    Li[tid] = Ls > 0.f ? 1.f / Ls : 0.f;
  }
  __syncthreads();
  for (int idx = tid; idx < ntl * G; idx += kSelThreadsD2) {
    const int tj = idx / G, h = idx % G;
    Ft[tj * 16 + h] = exp2f(tp[(size_t)tj * kTP * G + h] - Mh[h]) * Li[h];
  }
  // g_cmp * o_cmp, 4 values per thread
  for (int idx = tid; idx < G * (DV / 4); idx += kSelThreadsD2) {
    const int h = idx / (DV / 4), c4 = (idx % (DV / 4)) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < nch; ++c) {
      const float f = Fc[c * 16 + h];
      const float4 v = *reinterpret_cast<const float4*>(cpo + ((size_t)c * G + h) * DV + c4);
      acc.x += f * v.x; acc.y += f * v.y; acc.z += f * v.z; acc.w += f * v.w;
    }
    const int hq = g * G + h;
    const float sc = a.gates[((size_t)b * a.H_q + hq) * 3 + 0] * Li[h];
    *reinterpret_cast<float4*>(a.ocmp + ((size_t)b * a.H_q + hq) * DV + c4) =
        make_float4(sc * acc.x, sc * acc.y, sc * acc.z, sc * acc.w);
  }
  __syncthreads();
  // importance of blocks 0..jt: tile tj holds blocks 16 tj .. 16 tj + 16
  for (int j = tid; j <= jt; j += kSelThreadsD2) {
    const int tj = j >> 4, q = j & 15;
    float v = 0.f;
    if (tj < ntl) {
      const float* r = tp + ((size_t)tj * kTP + 1 + q) * G;
      for (int h = 0; h < G; ++h) v += Ft[tj * 16 + h] * r[h];
    }
    if (q == 0 && tj >= 1 && tj - 1 < ntl) {
      const float* r = tp + ((size_t)(tj - 1) * kTP + 17) * G;
      for (int h = 0; h < G; ++h) v += Ft[(tj - 1) * 16 + h] * r[h];
    }
    imp_s[j] = v;
    a.imp[bg * a.nb_stride + j] = v;
  }
  __syncthreads();
  if (tid < 32)
    warp_topn<PER>(imp_s, jt, a.top_n, a.force_first, a.force_local, a.sel + bg * a.top_n, tid);
}

// ---------------------------------------------------------------------------
// D3: selected blocks and window, split over the union of their blocks
// ---------------------------------------------------------------------------
template <int DK, int DV>
__global__ void __launch_bounds__(kDecThreads, 1) dec_fine_kernel(const DecodeArgs a,
                                                                  const __grid_constant__ DecodeMaps mp) {
  using S = DecSmem<DK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::BODY + S::PSCR);
  uint64_t* empty = full + kDecStages;
  int* sel_s = reinterpret_cast<int*>(empty + kDecStages);   // [32]
  int* uni = sel_s + 32;                                       // [64]
  int* nuni = uni + 64;
  volatile int* abort_flag = nuni + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cc = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int L = a.lens[b];
  if (L < 1 || L > a.max_len) return;
  const int t = L - 1, jt = t / a.ls;
  const int wlo = max(0, t - a.window + 1);
  const int G = a.G;
  const PartLayout pl = part_layout(a);
  const size_t bg = (size_t)b * a.H_kv + g;
  float* fpo = a.part + pl.fp_o + (bg * a.n_sw_chunks + cc) * 2 * G * DV;
  float* fpm = a.part + pl.fp_ml + (bg * a.n_sw_chunks + cc) * 2 * G * 2;

  if (tid < 32) sel_s[tid] = tid < a.top_n ? a.sel[((size_t)b * a.H_kv + g) * a.top_n + tid] : -1;
  __syncthreads();
  if (tid == 0) {
    // ascending union of the selected blocks and the blocks the window touches
    int ns = 0;
    while (ns < a.top_n && sel_s[ns] >= 0) ++ns;
    int i = 0, w = wlo / a.ls, n = 0;
    while (i < ns || w <= jt) {
      int v;
      if (w > jt || (i < ns && sel_s[i] < w)) v = sel_s[i++];
      else if (i < ns && sel_s[i] == w) { v = w; ++i; ++w; }
      else v = w++;
      if (n < 64) uni[n++] = v;
    }
    *nuni = n;
    for (int k = 0; k < kDecStages; ++k) { mbar_init(&full[k], 1); mbar_init(&empty[k], 1); }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int first = cc * kFineBlocks;
  const int nblk = max(0, min(kFineBlocks, *nuni - first));

  if (warp == kDecConsumers) {
    if (lane == 0) {
      for (int i = 0; i < nblk; ++i) {
        const int st = i % kDecStages;
        uint8_t* Ks = ring + st * S::STAGE;
        const int row = b * a.Lmax + uni[first + i] * a.ls;
        mbar_arrive_expect_tx(&full[st], S::STAGE);
        for (int kb = 0; kb < DK / 64; ++kb) tma_load_3d(Ks + kb * 8192, &mp.k, &full[st], kb * 64, g, row);
        for (int vb = 0; vb < DV / 64; ++vb)
          tma_load_3d(Ks + S::K_BYTES + vb * 8192, &mp.v, &full[st], vb * 64, g, row);
      }
    }
  } else {
    RowState<DV> rs_sel, rs_win;
    rs_sel.init();
    rs_win.init();
    if (warp < nblk) {
      uint32_t qa[DK / 16][4];
      const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(a.q) + ((size_t)b * a.H_q + (size_t)g * G) * DK;
      load_q_frags<DK>(qa, qp, G, lane);
      const int st = warp;
      if (mbar_wait(&full[st], 0, abort_flag, a.status, 411)) {
        const uint32_t kb = smem_u32(ring + st * S::STAGE);
        const int blk = uni[first + warp];
        bool in_sel = false;
        for (int k = 0; k < a.top_n; ++k) in_sel |= (sel_s[k] == blk);
        float s[8][4];
        warp_qk<DK>(qa, kb, s, lane);
        const int key0 = blk * a.ls + (lane & 3) * 2;
        float x[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int tau = key0 + nt * 8 + e;
            const bool vis = in_sel && tau <= t;
            x[nt][e] = vis ? s[nt][e] * a.scale_log2 : -INFINITY;
            x[nt][2 + e] = vis ? s[nt][2 + e] * a.scale_log2 : -INFINITY;
          }
        }
        rs_sel.update(x);
        warp_pv<DV>(x, kb + S::K_BYTES, rs_sel.o, lane);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int tau = key0 + nt * 8 + e;
            const bool vis = tau <= t && tau >= wlo;
            x[nt][e] = vis ? s[nt][e] * a.scale_log2 : -INFINITY;
            x[nt][2 + e] = vis ? s[nt][2 + e] * a.scale_log2 : -INFINITY;
          }
        }
        rs_win.update(x);
        warp_pv<DV>(x, kb + S::K_BYTES, rs_win.o, lane);
      }
    }
    rs_sel.finish();
    rs_win.finish();
    named_bar_sync(1, kDecConsumers * 32);
    float* stg = reinterpret_cast<float*>(ring);
    rs_sel.stage(stg + warp * 16 * (DV + 2), lane);
    rs_win.stage(stg + (kDecConsumers + warp) * 16 * (DV + 2), lane);
    named_bar_sync(1, kDecConsumers * 32);
    merge_warps<DV>(stg, G, fpo, fpm, tid);
    merge_warps<DV>(stg + kDecConsumers * 16 * (DV + 2), G, fpo + G * DV, fpm + G * 2, tid);
  }
  // the last CTA of this (b, g) to get here combines the three branches
  __shared__ int last;
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const int done = atomicAdd(reinterpret_cast<int*>(a.part + pl.cnt) + bg, 1);
    last = done == a.n_sw_chunks - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  float* fac = reinterpret_cast<float*>(ring);       // [2][nsw][16] factors, then [2][16] 1/den
  const float* po = a.part + pl.fp_o + bg * a.n_sw_chunks * 2 * G * DV;
  const volatile float* pm = a.part + pl.fp_ml + bg * a.n_sw_chunks * 2 * G * 2;
  float* inv = fac + 2 * a.n_sw_chunks * 16;
  if (tid < 2 * G) {
    const int br = tid / G, h = tid % G;
    float M = -1e30f;
    for (int c = 0; c < a.n_sw_chunks; ++c) {
      const size_t r = (((size_t)c * 2 + br) * G + h) * 2;
      if (pm[r + 1] > 0.f) M = fmaxf(M, pm[r]);
    }
    float den = 0.f;
    for (int c = 0; c < a.n_sw_chunks; ++c) {
      const size_t r = (((size_t)c * 2 + br) * G + h) * 2;
      const float f = pm[r + 1] > 0.f ? exp2f(pm[r] - M) : 0.f;
      fac[(br * a.n_sw_chunks + c) * 16 + h] = f;
      den += f * pm[r + 1];
    }
    const float gate = a.gates[((size_t)b * a.H_q + g * G + h) * 3 + 1 + br];
    inv[br * 16 + h] = den > 0.f ? gate / den : 0.f;
  }
  __syncthreads();
  for (int idx = tid; idx < G * (DV / 4); idx += kDecThreads) {
    const int h = idx / (DV / 4), c4 = (idx % (DV / 4)) * 4;
    const int hq = g * G + h;
    float4 res = *reinterpret_cast<const float4*>(a.ocmp + ((size_t)b * a.H_q + hq) * DV + c4);
    for (int br = 0; br < 2; ++br) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int c = 0; c < a.n_sw_chunks; ++c) {
        const float f = fac[(br * a.n_sw_chunks + c) * 16 + h];
        const float4 v = __ldcg(reinterpret_cast<const float4*>(po + (((size_t)c * 2 + br) * G + h) * DV + c4));
        acc.x += f * v.x; acc.y += f * v.y; acc.z += f * v.z; acc.w += f * v.w;
      }
      const float s_ = inv[br * 16 + h];
      res.x += s_ * acc.x; res.y += s_ * acc.y; res.z += s_ * acc.z; res.w += s_ * acc.w;
    }
    uint2 pk;
    pk.x = pack_bf16x2(res.x, res.y);
    pk.y = pack_bf16x2(res.z, res.w);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + ((size_t)b * a.H_q + hq) * DV + c4) = pk;
  }
}

// ---------------------------------------------------------------------------
template <int DK, int DV>
static cudaError_t launch_dec_t(const DecodeArgs& a, const DecodeMaps& m, cudaStream_t st) {
  using S = DecSmem<DK, DV>;
  cudaError_t e;
  auto k1 = dec_cmp_kernel<DK, DV>;
  auto k3 = dec_fine_kernel<DK, DV>;
  if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, S::TOTAL)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, S::TOTAL)) != cudaSuccess) return e;
  if (a.Lmax_cmp > 0) {
    prof_begin(P_DEC_CMP, st);
    k1<<<dim3(a.n_cmp_chunks, a.H_kv, a.B), kDecThreads, S::TOTAL, st>>>(a, m);
    prof_end(P_DEC_CMP, st, 1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const int per = (a.nb_stride + 31) / 32;
  const size_t sm2 = (32 + (size_t)a.n_cmp_chunks * 16 + (size_t)a.n_cmp_chunks * kTilesPerChunk * 16 +
                      (size_t)a.nb_stride) * 4;
  if (sm2 > 48 * 1024) {
    cudaError_t e2 = cudaSuccess;
    if (per <= 4) e2 = cudaFuncSetAttribute(dec_select_kernel<DV, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
    else if (per <= 8) e2 = cudaFuncSetAttribute(dec_select_kernel<DV, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
    else if (per <= 16) e2 = cudaFuncSetAttribute(dec_select_kernel<DV, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
    else if (per <= 32) e2 = cudaFuncSetAttribute(dec_select_kernel<DV, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
    else if (per <= 64) e2 = cudaFuncSetAttribute(dec_select_kernel<DV, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
    else e2 = cudaFuncSetAttribute(dec_select_kernel<DV, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
    if (e2 != cudaSuccess) return e2;
  }
  dim3 g2(a.H_kv, a.B);
  prof_begin(P_DEC_SELECT, st);
  if (per <= 4) dec_select_kernel<DV, 4><<<g2, kSelThreadsD2, sm2, st>>>(a);
  else if (per <= 8) dec_select_kernel<DV, 8><<<g2, kSelThreadsD2, sm2, st>>>(a);
  else if (per <= 16) dec_select_kernel<DV, 16><<<g2, kSelThreadsD2, sm2, st>>>(a);
  else if (per <= 32) dec_select_kernel<DV, 32><<<g2, kSelThreadsD2, sm2, st>>>(a);
  else if (per <= 64) dec_select_kernel<DV, 64><<<g2, kSelThreadsD2, sm2, st>>>(a);
  else if (per <= 128) dec_select_kernel<DV, 128><<<g2, kSelThreadsD2, sm2, st>>>(a);
  else return cudaErrorInvalidValue;
  prof_end(P_DEC_SELECT, st, 1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  prof_begin(P_DEC_FINE, st);
  k3<<<dim3(a.n_sw_chunks, a.H_kv, a.B), kDecThreads, S::TOTAL, st>>>(a, m);
  prof_end(P_DEC_FINE, st, 1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, const DecodeMaps& m, cudaStream_t st) {
  if (a.d_k == 192 && a.d_v == 128) return launch_dec_t<192, 128>(a, m, st);
  if (a.d_k == 64 && a.d_v == 64) return launch_dec_t<64, 64>(a, m, st);
  if (a.d_k == 128 && a.d_v == 128) return launch_dec_t<128, 128>(a, m, st);
  if (a.d_k == 192 && a.d_v == 64) return launch_dec_t<192, 64>(a, m, st);
  if (a.d_k == 64 && a.d_v == 128) return launch_dec_t<64, 128>(a, m, st);
  if (a.d_k == 128 && a.d_v == 64) return launch_dec_t<128, 64>(a, m, st);
  return cudaErrorInvalidValue;
}

}  // namespace nsa
