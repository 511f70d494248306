// NSA decode: one new query per sequence at position L-1 against a KV cache.
//
// Same five steps as the prefill ("Разреженное внимание — NSA и DSA",
// ai.flicky.cc, section "NSA: три ветви"; the cache holds the new token), laid
// out as coalesced HBM streaming: decode reads every compressed key once and the
// raw keys of the selected blocks and the window once, so the bound is HBM
// bandwidth. Every KV tile (TMA, 32 keys) is loaded once per GQA group and
// consumed by mma.sync with the group's heads as the 16 rows.
//
//   D1  dec_cmp, persistent over (sequence, KV head, 512-key chunk) items:
//       per-chunk online softmax state (o, m, l) per head, and per 32-key tile
//       the block sums sum_i exp(s_i - m_ref) * omega(i, j) of the selection
//       blocks it touches. A dedicated warp merges the consumer warps' states
//       while they go on with the next item.
//   D2  (prologue of the D3 CTA of each (sequence, KV head), after waiting for
//       D1 through programmatic dependent launch): merge the chunks' softmax
//       states, reduce the block sums over the group's heads into the
//       importance, run the top-n selection over the CTA's warps.
//   D3  dec_fine streams the union of the selected blocks and the window blocks
//       once (the window is prefetched into L2 while D2 runs); four warps run
//       the selected branch and four the window branch, each with its own
//       softmax; the combine forms g_cmp o_cmp from the chunk outputs (L2) with
//       the merge factors of D2 and writes out = g_cmp o_cmp + g_slc o_slc +
//       g_win o_win.
#include "common.cuh"
#include "kernels.h"
#include "topn.cuh"
#include "warp_mma.cuh"

namespace nsa {

namespace {

// Key tiles of 32 keys (20 KB of K+V at d 192/128) in an 8-stage ring: each of
// the 4 consumer warps computes on one stage while the next tiles are in flight.
constexpr int kTileKeys = 32;
constexpr int kNT = kTileKeys / 8;     // 8-key MMA n-tiles per tile
constexpr int kDecStages = 8;
constexpr int kDecBranchWarps = 4;                      // consumer warps per branch (selected, window)
constexpr int kDecConsumers = 2 * kDecBranchWarps;
constexpr int kDecThreads = (kDecConsumers + 1) * 32;   // consumers, producer
// compressed-key pass: consumer warps + producer warp
constexpr int kD1Stages = 8;
constexpr int kD1Consumers = 4;
constexpr int kD1Threads = (kD1Consumers + 2) * 32;   // consumers, producer, merger
constexpr int kCmpChunk = 512;         // compressed keys per D1 work item
constexpr int kTilesPerChunk = kCmpChunk / kTileKeys;
constexpr int kBlkPerTile = kTileKeys / 4;   // selection blocks a tile of compressed keys covers
constexpr int kTP = kBlkPerTile + 2;   // tile partial: m_ref + block sums (+1 spilling into the next)

template <int DK, int DV>
struct DecSmem {
  static constexpr int K_BYTES = kTileKeys * DK * 2;
  static constexpr int V_BYTES = kTileKeys * DV * 2;
  static constexpr int STAGE = K_BYTES + V_BYTES;
  static constexpr int RING = kDecStages * STAGE;
  static constexpr int MERGE = kDecConsumers * 16 * (DV + 2) * 4;   // one staged state per consumer warp
  static constexpr int PSCR = 16 * 1024;                              // the group's Q (16 rows x d_k <= 256)
  static constexpr int BODY = (RING > MERGE ? RING : MERGE);
  static constexpr int TOTAL = 1024 + BODY + PSCR + 1024;
};

__device__ __forceinline__ int n_cmp_dev(int L, int l, int s) { return L >= l ? (L - l) / s + 1 : 0; }

// tensor-map row of raw token `tok` / compressed entry `e` of sequence b
__device__ __forceinline__ int kv_row(const DecodeArgs& a, int b, int tok) {
  return a.kv_pt.table ? (int)paged_row(a.kv_pt, b, tok, a.status) : b * a.Lmax + tok;
}
__device__ __forceinline__ int cmp_row(const DecodeArgs& a, int b, int e) {
  return a.cmp_pt.table ? (int)paged_row(a.cmp_pt, b, e, a.status) : b * a.Lmax_cmp + e;
}

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
  p.total = p.cnt + BG + 16;   // slack: bulk copies round their size up to 16 bytes
  return p;
}

// Merge NW staged warp states ([w][16][DV+2]) into one state per row < G, by one
// warp: lanes 2r, 2r+1 take row r (< G <= 16), half of its columns each; o is
// written relative to the merged max M -> dst_o[row][DV], (M, L) -> dst_ml[row][2]
template <int DV, int NW>
__device__ __forceinline__ void merge_warps_w32(const float* stg, int G, float* dst_o, float* dst_ml, int lane) {
  const int row = lane >> 1, part = lane & 1;
  if (row >= G) return;
  float M = -1e30f;
#pragma unroll
  for (int w = 0; w < NW; ++w) M = fmaxf(M, stg[(w * 16 + row) * (DV + 2) + DV]);
  float f[NW], Ls = 0.f;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const float* r = stg + (w * 16 + row) * (DV + 2);
    f[w] = r[DV + 1] > 0.f ? ex2(r[DV] - M) : 0.f;
    Ls += f[w] * r[DV + 1];
  }
  const int c0 = part * (DV / 2);
#pragma unroll 4
  for (int c = c0; c < c0 + DV / 2; c += 4) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float* r = stg + (w * 16 + row) * (DV + 2) + c;   // 8-byte aligned rows
      const float2 x = *reinterpret_cast<const float2*>(r);
      const float2 y = *reinterpret_cast<const float2*>(r + 2);
      v.x += f[w] * x.x; v.y += f[w] * x.y; v.z += f[w] * y.x; v.w += f[w] * y.y;
    }
    *reinterpret_cast<float4*>(dst_o + row * DV + c) = v;
  }
  if (part == 0) {
    dst_ml[row * 2 + 0] = M;
    dst_ml[row * 2 + 1] = Ls;
  }
}

}  // namespace

// Optional timeline of the fine pass (compiled only with -DNSA_DECODE_TRACE): thread
// 0 of the CTAs of KV head 0 and sequences 0..7 records clock64() at fixed points;
// nsa_decode_trace_read copies the records out. Off in the library build.
#ifdef NSA_DECODE_TRACE
__device__ unsigned long long g_dtrace[8][16];
#define TRD(k)                                                                   \
  do {                                                                           \
    if (blockIdx.x == 0 && blockIdx.y < 8 && threadIdx.x == 0) g_dtrace[blockIdx.y][(k)] = clock64(); \
  } while (0)
// compressed pass: CTA 0, per consumer tile of warp 0 / per item; every CTA's start / end (global timer)
__device__ unsigned long long g_ctrace[2][64][4];
__device__ unsigned long long g_cspan[256][3];
__device__ unsigned long long g_fspan[512][3];
#define TRC(kind, i, k)                                                          \
  do {                                                                           \
    if (blockIdx.x == 0 && lane == 0 && (i) < 64) g_ctrace[kind][i][k] = clock64(); \
  } while (0)
#else
#define TRD(k) do {} while (0)
#define TRC(kind, i, k) do {} while (0)
#endif

size_t decode_partials_floats(const DecodeArgs& a) { return part_layout(a).total; }

// ---------------------------------------------------------------------------
// D1: compressed keys, split into 512-key chunks. Persistent: one CTA per SM takes
// (sequence, KV head, chunk) items from a shared counter; the producer warp keeps the
// ring full across item boundaries (Q of the next item double-buffered), so the
// HBM stream never drains between items.
// ---------------------------------------------------------------------------
template <int DK, int DV>
struct D1Smem {
  static constexpr int STAGE = kTileKeys * (DK + DV) * 2;
  static constexpr int RING = kD1Stages * STAGE;
  static constexpr int QBUF = (DK / 64) * 16 * 128;                 // one item's Q, 16 rows
  static constexpr int STG = kD1Consumers * 16 * (DV + 2) * 4;       // per-warp states for the merge
  static constexpr int PSCR = kD1Consumers * 16 * kTileKeys * 4;     // probabilities for block sums
  static constexpr int TOTAL = 1024 + RING + 2 * QBUF + STG + PSCR + 256;
};

template <int DK, int DV>
__global__ void __launch_bounds__(kD1Threads, 1) dec_cmp_kernel(const DecodeArgs a,
                                                                 const __grid_constant__ DecodeMaps mp) {
  using S = D1Smem<DK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* qbuf = smem + S::RING;
  float* stg = reinterpret_cast<float*>(qbuf + 2 * S::QBUF);
  float* pscr = stg + S::STG / 4;
  uint64_t* full = reinterpret_cast<uint64_t*>(pscr + S::PSCR / 4);
  uint64_t* empty = full + kD1Stages;
  uint64_t* q_full = empty + kD1Stages;     // [2]
  uint64_t* q_empty = q_full + 2;            // [2]
  uint64_t* stg_full = q_empty + 2;          // the consumers' item states are staged
  uint64_t* stg_free = stg_full + 1;         // the merger has read them
  volatile int* abort_flag = reinterpret_cast<volatile int*>(stg_free + 1);
  // ring position each stage currently holds: a consumer waits on a stage's
  // barrier only once the stage holds its tile (consecutive tiles of one warp are
  // not consecutive uses of a stage, so a parity wait alone could alias)
  volatile int* stage_tag = abort_flag + 1;    // [kD1Stages]
  volatile int* q_item = stage_tag + kD1Stages;  // [2] item of each Q slot (-1: no more items)
  volatile int* stg_item = q_item + 2;           // item of the staged states (-1: no more)
  // items are handed out by a counter in the workspace header, so CTAs whose
  // stream runs faster take more of them; the last CTA to finish sets the
  // counter back to 0 for the next launch
  WsHeader* hdr = reinterpret_cast<WsHeader*>(a.status);
  int* item_ctr = reinterpret_cast<int*>(&hdr->sched_next);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G;
  const PartLayout pl = part_layout(a);
  const int n_items = a.B * a.H_kv * a.n_cmp_chunks;
  // the fine pass may be scheduled on SMs this kernel's CTAs leave; it waits for
  // this whole grid before it reads the partials
  pdl_launch_dependents();

  if (tid == 0) {
    for (int i = 0; i < kD1Stages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); stage_tag[i] = -1; }
    for (int i = 0; i < 2; ++i) { mbar_init(&q_full[i], 1); mbar_init(&q_empty[i], kD1Consumers); }
    mbar_init(stg_full, kD1Consumers * 32);
    mbar_init(stg_free, 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
#ifdef NSA_DECODE_TRACE
  if (threadIdx.x == 0 && blockIdx.x < 256) {
    g_cspan[blockIdx.x][0] = globaltimer_ns();
    unsigned int smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    g_cspan[blockIdx.x][2] = smid;
  }
#endif
  __syncthreads();

  // item -> (b, g, chunk); returns the number of 64-key tiles (0: nothing to do)
  auto item_tiles = [&](int item, int& b, int& g, int& chunk) -> int {
    chunk = item % a.n_cmp_chunks;
    const int bg = item / a.n_cmp_chunks;
    g = bg % a.H_kv;
    b = bg / a.H_kv;
    const int L = a.lens[b];
    if (L < 1 || L > a.max_len) {
      if (chunk == 0 && g == 0) atomicOr(a.status, DEV_ERR_BOUNDS);   // called by the producer only
      return 0;
    }
    const int nc = n_cmp_dev(L, a.l, a.s);
    const int c0 = chunk * kCmpChunk;
    return c0 < nc ? min(kTilesPerChunk, (nc - c0 + kTileKeys - 1) / kTileKeys) : 0;
  };

  if (warp == kD1Consumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int u = 0, it = 0;
      bool ok = true;
      while (ok) {
        const int item = atomicAdd(item_ctr, 1);
        if (item >= n_items) break;
        int b, g, chunk;
        const int ntl = item_tiles(item, b, g, chunk);
        if (ntl == 0) continue;
        const int qi = it & 1;
        if (it >= 2 && !mbar_wait(&q_empty[qi], ((it >> 1) - 1) & 1, abort_flag, a.status, 403)) break;
        q_item[qi] = item;   // published by the arrival on q_full
        mbar_arrive_expect_tx(&q_full[qi], (uint32_t)(DK / 64) * G * 128);
        for (int kb = 0; kb < DK / 64; ++kb)
          tma_load_3d(qbuf + qi * S::QBUF + kb * 2048, &mp.q, &q_full[qi], kb * 64, g * G, b);
        if (!NSA_BOUNDS(chunk * kCmpChunk + ntl * kTileKeys <= a.Lmax_cmp + kTileKeys - 1, a.status, 513)) {
          *abort_flag = 1;   // stop the consumers; the copies issued so far are drained below
          break;
        }
        for (int i = 0; i < ntl; ++i, ++u) {
          const int st = u % kD1Stages;
          if (u >= kD1Stages && !mbar_wait(&empty[st], ((u / kD1Stages) - 1) & 1, abort_flag, a.status, 401)) {
            ok = false;
            break;
          }
          TRC(0, u, 2);
          uint8_t* Ks = ring + st * S::STAGE;
          // a 32-entry tile never straddles a page (page sizes are multiples of 32)
          const int row = cmp_row(a, b, chunk * kCmpChunk + i * kTileKeys);
          stage_tag[st] = u;
          mbar_arrive_expect_tx(&full[st], S::STAGE);
          for (int kb = 0; kb < DK / 64; ++kb)
            tma_load_3d(Ks + kb * (kTileKeys * 128), &mp.kc, &full[st], kb * 64, g, row);
          for (int vb = 0; vb < DV / 64; ++vb)
            tma_load_3d(Ks + DK * kTileKeys * 2 + vb * (kTileKeys * 128), &mp.vc, &full[st], vb * 64, g, row);
        }
        ++it;
      }
      // no more items: an empty Q slot tells the consumers
      if (ok && !*abort_flag) {
        const int qi = it & 1;
        if (it < 2 || mbar_wait(&q_empty[qi], ((it >> 1) - 1) & 1, abort_flag, a.status, 408)) {
          q_item[qi] = -1;
          mbar_arrive(&q_full[qi]);
        }
      }
      if (*abort_flag) {
        // let the copies still in flight land before the CTA exits
        for (int v = u - kD1Stages < 0 ? 0 : u - kD1Stages; v < u; ++v)
          mbar_wait_drain(&full[v % kD1Stages], (v / kD1Stages) & 1);
        for (int q2 = it - 2 < 0 ? 0 : it - 2; q2 < it; ++q2) mbar_wait_drain(&q_full[q2 & 1], (q2 >> 1) & 1);
      }
    }
  } else if (warp == kD1Consumers + 1) {
    // ------------------------------------------------------------ merger
    for (int it = 0;; ++it) {
      if (!__all_sync(0xffffffffu, mbar_wait(stg_full, it & 1, abort_flag, a.status, 407))) break;
      const int item = *stg_item;
      if (item < 0) break;
      const int chunk = item % a.n_cmp_chunks;
      const int g = (item / a.n_cmp_chunks) % a.H_kv, b = (item / a.n_cmp_chunks) / a.H_kv;
      const size_t ci = ((size_t)b * a.H_kv + g) * a.n_cmp_chunks + chunk;
      merge_warps_w32<DV, kD1Consumers>(stg, G, a.part + pl.cp_o + ci * G * DV, a.part + pl.cp_ml + ci * G * 2, lane);
      __syncwarp();
      mbar_arrive(stg_free);
    }
  } else {
    // ------------------------------------------------------------ consumers
    float* ps = pscr + warp * 16 * kTileKeys;
    int u_base = 0, it = 0;
    bool ok = true;
    while (ok) {
      const int qi = it & 1;
      if (warp == 0) TRC(1, it, 0);
      ok = __all_sync(0xffffffffu, mbar_wait(&q_full[qi], (it >> 1) & 1, abort_flag, a.status, 404));
      if (!ok) break;
      const int item = q_item[qi];
      if (item < 0) {   // no more items: release the merger
        if (it > 0 && !__all_sync(0xffffffffu, mbar_wait(stg_free, (it - 1) & 1, abort_flag, a.status, 409))) break;
        if (warp == 0 && lane == 0) *stg_item = -1;
        mbar_arrive(stg_full);
        break;
      }
      const int chunk = item % a.n_cmp_chunks;
      const int g = (item / a.n_cmp_chunks) % a.H_kv, b = (item / a.n_cmp_chunks) / a.H_kv;
      const int nc = n_cmp_dev(a.lens[b], a.l, a.s);
      const int c0 = chunk * kCmpChunk;
      const int ntl = min(kTilesPerChunk, (nc - c0 + kTileKeys - 1) / kTileKeys);
      // every warp reaches the three item-end barriers even when a wait gave up
      if (warp == 0) TRC(1, it, 1);
      const uint32_t qbase = smem_u32(qbuf + qi * S::QBUF);
      RowState<DV> rs;
      rs.init();
      for (int i = warp; i < ntl && ok; i += kD1Consumers) {
        const int u = u_base + i;
        const int st = u % kD1Stages;
        const bool got = smem_wait_eq(&stage_tag[st], u, abort_flag, a.status, 405) &&
                         mbar_wait(&full[st], (u / kD1Stages) & 1, abort_flag, a.status, 402);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        if (warp == 0) TRC(0, u, 0);
        const uint32_t kb = smem_u32(ring + st * S::STAGE);
        float s[kNT][4];
        warp_qk_sq<DK, kNT>(qbase, 2048, 0, kb, s, lane);
        const int kc0 = c0 + i * kTileKeys + (lane & 3) * 2;
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const bool vis = kc0 + nt * 8 + e < nc;
            s[nt][e] = vis ? s[nt][e] * a.scale_log2 : -INFINITY;
            s[nt][2 + e] = vis ? s[nt][2 + e] * a.scale_log2 : -INFINITY;
          }
        }
        rs.update(s);   // s now holds exp2(x - m) for the running max m
        {
          const int r0 = lane >> 2, cq = (lane & 3) * 2;
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt) {
            ps[r0 * kTileKeys + nt * 8 + cq] = s[nt][0];
            ps[r0 * kTileKeys + nt * 8 + cq + 1] = s[nt][1];
            ps[(r0 + 8) * kTileKeys + nt * 8 + cq] = s[nt][2];
            ps[(r0 + 8) * kTileKeys + nt * 8 + cq + 1] = s[nt][3];
          }
        }
        warp_pv<DV, kNT>(s, kb + DK * kTileKeys * 2, rs.o, lane);
        __syncwarp();
        if (warp == 0) TRC(0, u, 1);
        if (lane == 0) mbar_arrive(&empty[st]);
        // block sums: compressed key 4q+u covers tokens [16(4q+u), +32): u<3 -> 2p
        // into block q of the tile, u = 3 -> p into q and q+1. Tile partial layout
        // [kTP][G]: row 0 = reference max per head, rows 1..kBlkPerTile+1 = block
        // sums per head (the last one spills into the next tile's first block).
        {
          const int tile = c0 / kTileKeys + i;
          float* tpb = a.part + pl.tp + (((size_t)b * a.H_kv + g) * pl.n_tiles + tile) * kTP * G;
          const int row = lane >> 1, half = lane & 1;
          if (row < G) {
            const float* pr = ps + row * kTileKeys;
            const int q0 = half * (kBlkPerTile / 2);
            for (int q = q0; q < q0 + kBlkPerTile / 2; ++q) {
              float v = 2.f * (pr[4 * q] + pr[4 * q + 1] + pr[4 * q + 2]) + pr[4 * q + 3];
              if (q > 0) v += pr[4 * q - 1];
              tpb[(1 + q) * G + row] = v;
            }
            if (half == 1) tpb[(1 + kBlkPerTile) * G + row] = pr[kTileKeys - 1];
          }
          if ((lane & 3) == 0) {
            const int r0 = lane >> 2;
            if (r0 < G) tpb[r0] = rs.m[0];
            if (r0 + 8 < G) tpb[r0 + 8] = rs.m[1];
          }
        }
        __syncwarp();
      }
      if (warp == 0) TRC(1, it, 2);
      rs.finish();
      // the merger warp combines the four warps' states while the consumers go on
      // with the next item; the staging area is single-buffered
      if (it > 0 && !__all_sync(0xffffffffu, mbar_wait(stg_free, (it - 1) & 1, abort_flag, a.status, 406)))
        ok = false;
      if (ok) rs.stage(stg + warp * 16 * (DV + 2), lane);
      if (warp == 0 && lane == 0) *stg_item = item;   // published by the arrival on stg_full
      mbar_arrive(stg_full);
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_empty[qi]);
      if (warp == 0) TRC(1, it, 3);
      if (!ok) break;
      u_base += ntl;
      ++it;
    }
  }
  __syncthreads();
  if (tid == 0) {
    // this CTA's producer has stopped taking items; the last CTA out resets the
    // counters (kernels after this one in the stream see the reset)
    __threadfence();
    if (atomicAdd(&hdr->sched_done, 1u) == gridDim.x - 1) {
      atomicExch(&hdr->sched_next, 0u);
      atomicExch(&hdr->sched_done, 0u);
    }
  }
#ifdef NSA_DECODE_TRACE
  if (threadIdx.x == 0 && blockIdx.x < 256) g_cspan[blockIdx.x][1] = globaltimer_ns();
#endif
}

// ---------------------------------------------------------------------------
// D3: selected blocks and window for one (sequence, KV head) per CTA. The
// ascending union of the selected blocks and the blocks the window touches is
// streamed once through the TMA ring in 32-key halves; warps 0-3 (selected
// branch) and 4-7 (window) take halves w, w+4, ... and compute on those their
// branch reads, each warp with one online softmax. The warps' states are merged
// in shared memory and out = g_cmp o_cmp + g_slc o_slc + g_win o_win is written.
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
  int* uni = reinterpret_cast<int*>(empty + kDecStages);      // [64]
  int* nuni = uni + 64;
  volatile int* abort_flag = nuni + 1;
  uint32_t* flags = reinterpret_cast<uint32_t*>(nuni + 2);     // [64] 1 = selected block
  uint64_t* d2bar = reinterpret_cast<uint64_t*>(flags + 64);    // bulk copy of the chunk partials
  uint8_t* qs = smem + S::BODY;                                 // Q: DK/64 chunks of [16 rows][128 B]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.x, b = blockIdx.y;
  const int L = a.lens[b];
  if (L < 1 || L > a.max_len) return;
  const int t = L - 1, jt = t / a.ls;
  const int wlo = max(0, t - a.window + 1);
  const int G = a.G;
  const size_t bg = (size_t)b * a.H_kv + g;

  TRD(0);
#ifdef NSA_DECODE_TRACE
  const int fsp = blockIdx.y * gridDim.x + blockIdx.x;
  if (threadIdx.x == 0 && fsp < 512) g_fspan[fsp][0] = globaltimer_ns();
#endif
  // K/V of one 32-key half of block blk into L2 (the stream reads them from there)
  auto prefetch_half = [&](int blk, int half) {
    const int row = kv_row(a, b, blk * a.ls + half * kTileKeys);   // pages hold whole blocks
    for (int kb = 0; kb < DK / 64; ++kb) tma_prefetch_3d(&mp.k, kb * 64, g, row);
    for (int vb = 0; vb < DV / 64; ++vb) tma_prefetch_3d(&mp.v, vb * 64, g, row);
  };
  if (warp == kDecConsumers && lane == 0) {
    // the window does not depend on the selection: its blocks travel to L2 while
    // the chunk partials are merged and the blocks are selected
    for (int blk = wlo / a.ls; blk <= jt; ++blk)
      for (int h = 0; h < 2; ++h)
        if (blk * a.ls + h * kTileKeys <= t) prefetch_half(blk, h);
  }
  if (tid == 0) {
    for (int k = 0; k < kDecStages; ++k) { mbar_init(&full[k], 1); mbar_init(&empty[k], 2); }   // one warp per branch
    mbar_init(d2bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  {   // the group's Q (an input: staged before the wait on the previous kernel)
    const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(a.q) + ((size_t)b * a.H_q + (size_t)g * G) * DK;
    for (int idx = tid; idx < 16 * (DK / 8); idx += kDecThreads) {   // 16-byte chunks
      const int row = idx / (DK / 8), c = idx % (DK / 8);
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (row < G) v = *reinterpret_cast<const uint4*>(qp + (size_t)row * DK + c * 8);
      *reinterpret_cast<uint4*>(qs + (c >> 3) * 2048 + sw128(row, c & 7)) = v;
    }
  }
  __syncthreads();
  pdl_wait();   // the compressed pass (the previous kernel) has finished: its partials are visible
  // ---- D2 (in this CTA, before the ring is used): merge the compressed chunks of
  // (b, g) (the factors are kept for the combine step), form the importance,
  // select the top-n blocks
  {
    const PartLayout pl = part_layout(a);
    const int nc = n_cmp_dev(L, a.l, a.s);
    const int nch = (nc + kCmpChunk - 1) / kCmpChunk;   // <= 32 (checked on the host)
    const int ntl = (nc + kTileKeys - 1) / kTileKeys;
    float* Mh = reinterpret_cast<float*>(ring);   // [16] max per head
    // 1 / denominator and the chunk factors outlive the prologue (the o_cmp warp
    // reads them while the ring streams): they sit behind Q (<= 6 KB) in its area
    float* Li = reinterpret_cast<float*>(qs + 8192);   // [16]
    float* Fc = Li + 16;                               // [nch][16] chunk factors (<= 2 KB)
    float* Ft = Mh + 16;                               // [ntl][16] tile factors (incl. 1/L)
    float* imp_s = Ft + pl.n_tiles * 16;          // [nb_stride]
    const float* cpm = a.part + pl.cp_ml + bg * a.n_cmp_chunks * G * 2;
    const float* tp = a.part + pl.tp + bg * pl.n_tiles * kTP * G;
    // the tile partials come into shared memory with bulk copies when they fit
    // next to the scratch (otherwise they are read in place)
    constexpr int kTopnWarps = 8;   // slices of the CTA-wide top-n
    uint32_t* ck = reinterpret_cast<uint32_t*>(imp_s + ((a.nb_stride + 3) & ~3));   // top-n scratch [8][32]
    int* ci = reinterpret_cast<int*>(ck + kTopnWarps * 32);
    float* tp_s = reinterpret_cast<float*>(ci + kTopnWarps * 32);
    const uint32_t tp_bytes = (uint32_t)(((size_t)ntl * kTP * G * 4 + 15) & ~size_t(15));
    const bool bulk = (size_t)((uint8_t*)tp_s - ring) + tp_bytes <= (size_t)S::BODY && nc > 0;
    if (bulk) {
      if (warp == 0) {   // 8 KB pieces from several lanes keep more copies in flight
        if (lane == 0) mbar_arrive_expect_tx(d2bar, tp_bytes);
        __syncwarp();
        constexpr uint32_t kPiece = 8192;
        const uint32_t ntp = (tp_bytes + kPiece - 1) / kPiece;
        for (uint32_t i = lane; i < ntp; i += 32) {
          const uint32_t off = i * kPiece;
          const uint32_t n = min(kPiece, tp_bytes - off);
          bulk_load(reinterpret_cast<uint8_t*>(tp_s) + off, reinterpret_cast<const uint8_t*>(tp) + off, n, d2bar);
        }
      }
      const bool got = mbar_wait(d2bar, 0, abort_flag, a.status, 410);
      if (__syncthreads_or(!got)) {   // one decision for the whole CTA
        if (tid == 0) mbar_wait_drain(d2bar, 0);   // let the copies land before the CTA leaves
        return;
      }
      tp = tp_s;
    }
    TRD(1);
    // one warp per head, the chunks in its lanes
    for (int h = warp; h < G; h += kDecThreads / 32) {
      float m = -1e30f, l = 0.f;
      if (lane < nch) {
        m = cpm[(lane * G + h) * 2];
        l = cpm[(lane * G + h) * 2 + 1];
      }
      float M = l > 0.f ? m : -1e30f;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
      const float f = (lane < nch && l > 0.f) ? exp2f(m - M) : 0.f;
      float Ls = f * l;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, off);
      if (lane < nch) Fc[lane * 16 + h] = f;
      if (lane == 0) {
        Mh[h] = M;
        Li[h] = Ls > 0.f ? 1.f / Ls : 0.f;
      }
    }
    __syncthreads();
    TRD(2);
    for (int idx = tid; idx < ntl * G; idx += kDecThreads) {
      const int tj = idx / G, h = idx % G;
      Ft[tj * 16 + h] = exp2f(tp[(size_t)tj * kTP * G + h] - Mh[h]) * Li[h];
    }
    // (g_cmp * o_cmp is formed in the combine step, from the chunk outputs in L2)
    __syncthreads();
    TRD(3);
    // importance of blocks 0..jt: tile tj holds blocks kBlkPerTile*tj .. + kBlkPerTile
    for (int j = tid; j <= jt; j += kDecThreads) {
      const int tj = j / kBlkPerTile, q = j % kBlkPerTile;
      float v = 0.f;
      auto head_sum = [&](int tile, int rowi) -> float {
        const float* rr = tp + ((size_t)tile * kTP + rowi) * G;
        const float* ff = Ft + tile * 16;
        float acc = 0.f;
        if ((G & 3) == 0) {
#pragma unroll 4
          for (int h = 0; h < G; h += 4) {
            const float4 x = *reinterpret_cast<const float4*>(rr + h);
            const float4 y = *reinterpret_cast<const float4*>(ff + h);
            acc += x.x * y.x + x.y * y.y + x.z * y.z + x.w * y.w;
          }
        } else {
          for (int h = 0; h < G; ++h) acc += ff[h] * rr[h];
        }
        return acc;
      };
      if (tj < ntl) v += head_sum(tj, 1 + q);
      if (q == 0 && tj >= 1 && tj - 1 < ntl) v += head_sum(tj - 1, 1 + kBlkPerTile);
      imp_s[j] = v;
      a.imp[bg * a.nb_stride + j] = v;
    }
    __syncthreads();
    TRD(4);
    if (!cta_topn(imp_s, jt, a.top_n, a.force_first, a.force_local, a.sel + bg * a.top_n, ck, ci, kTopnWarps,
                  warp, lane) &&
        warp == 0)
      warp_topn_any(imp_s, jt, a.top_n, a.force_first, a.force_local, a.sel + bg * a.top_n, lane);
    __syncthreads();
#ifdef NSA_DEBUG_BOUNDS
    if (warp == 0 && lane < a.top_n) {   // ascending, in 0..jt, -1 only as padding
      const int32_t* sl = a.sel + bg * a.top_n;
      const int v = sl[lane];
      const bool fine = v == -1 ? (lane + 1 >= a.top_n || sl[lane + 1] == -1)
                                : (v >= 0 && v <= jt && (lane == 0 || sl[lane - 1] < v));
      NSA_BOUNDS(fine, a.status, 512);
    }
    __syncthreads();
#endif
  }
  TRD(5);
  if (warp == kDecConsumers && lane == 0) {   // selected blocks below the window, ahead of the stream
    const int32_t* sel = a.sel + bg * a.top_n;
    for (int i = 0; i < a.top_n; ++i) {
      const int blk = sel[i];
      if (blk >= 0 && blk < wlo / a.ls) {
        prefetch_half(blk, 0);
        prefetch_half(blk, 1);
      }
    }
  }
  if (warp == 0) {
    // union of the selected blocks (ascending, -1 padded) and the window blocks
    // [wlo / l', jt]: the selected blocks below the window first, then the window
    // blocks, each flagged when it was also selected
    const int32_t* sel = a.sel + bg * a.top_n;
    const int wb = wlo / a.ls;
    const int nwin = jt - wb + 1;
    int ns = 0;
    for (int i = lane; i < a.top_n; i += 32) ns += sel[i] >= 0;
    ns = __reduce_add_sync(0xffffffffu, ns);
    if (nwin <= 32 && ns <= 32) {
      const int si = lane < ns ? sel[lane] : 0x7fffffff;
      const bool below = lane < ns && si < wb;
      const uint32_t bb = __ballot_sync(0xffffffffu, below);
      const int nbelow = __popc(bb);
      if (below) {
        const int pos = __popc(bb & ((1u << lane) - 1u));
        uni[pos] = si;
        flags[pos] = 1u;
      }
      const uint32_t wsel =
          __reduce_or_sync(0xffffffffu, (lane < ns && si >= wb && si <= jt) ? 1u << (si - wb) : 0u);
      if (lane < nwin && nbelow + lane < 64) {
        uni[nbelow + lane] = wb + lane;
        flags[nbelow + lane] = (wsel >> lane) & 1u;
      }
      if (lane == 0) *nuni = nbelow + nwin < 64 ? nbelow + nwin : 64;
    } else {
      // general walk over the candidate range in chunks of 32 blocks
      int cnt = 0, sj = 0;
      int next_sel = ns > 0 ? sel[0] : 0x7fffffff;
      for (int j0 = 0; j0 <= jt; j0 += 32) {
        if (j0 + 31 < wb && next_sel > j0 + 31) {   // neither a selected block nor the window here
          const int target = next_sel < wb ? next_sel : wb;
          j0 = (target / 32) * 32 - 32;
          continue;
        }
        const int j = j0 + lane;
        bool is_sel = false;
        for (int i = sj; i < ns; ++i) {
          const int v = sel[i];
          if (v > j0 + 31) break;
          is_sel |= (v == j);
        }
        const bool in = j <= jt && (is_sel || j >= wb);
        const uint32_t bal = __ballot_sync(0xffffffffu, in);
        if (in) {
          const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
          if (pos < 64) {
            uni[pos] = j;
            flags[pos] = is_sel ? 1u : 0u;
          }
        }
        cnt += __popc(bal);
        while (sj < ns && sel[sj] <= j0 + 31) ++sj;
        next_sel = sj < ns ? sel[sj] : 0x7fffffff;
      }
      if (lane == 0) *nuni = cnt < 64 ? cnt : 64;
    }
  }
  __syncthreads();
  TRD(6);
  const int nu = *nuni;

  // work units: the two 32-key halves of every union block
  const int nh = 2 * nu;
  if (warp == kDecConsumers) {
    if (lane == 0) {
      int issued = 0;
      for (int u = 0; u < nh; ++u) {
        const int st = u % kDecStages;
        if (u >= kDecStages && !mbar_wait(&empty[st], ((u / kDecStages) - 1) & 1, abort_flag, a.status, 411)) break;
        if (u == 0 && NSA_INJECT(a, FAULT_DECODE_FINE_TILE)) {   // checking build: withhold the first tile
          issued = 1;
          continue;
        }
        uint8_t* Ks = ring + st * S::STAGE;
        if (!NSA_BOUNDS(uni[u >> 1] >= 0 && uni[u >> 1] <= jt, a.status, 511)) {
          *abort_flag = 1;   // stop the consumers; the copies issued so far are drained below
          break;
        }
        const int row = kv_row(a, b, uni[u >> 1] * a.ls + (u & 1) * kTileKeys);
        mbar_arrive_expect_tx(&full[st], S::STAGE);
        for (int kb = 0; kb < DK / 64; ++kb)
          tma_load_3d(Ks + kb * (kTileKeys * 128), &mp.k, &full[st], kb * 64, g, row);
        for (int vb = 0; vb < DV / 64; ++vb)
          tma_load_3d(Ks + S::K_BYTES + vb * (kTileKeys * 128), &mp.v, &full[st], vb * 64, g, row);
        issued = u + 1;
      }
      if (*abort_flag)   // let the copies still in flight land before the CTA exits
        for (int v = issued - kDecStages < 0 ? 0 : issued - kDecStages; v < issued; ++v)
          mbar_wait_drain(&full[v % kDecStages], (v / kDecStages) & 1);
    }
  } else {
    // warps 0..3 run the selected branch, warps 4..7 the window branch: warp
    // (br, wq) takes the 32-key halves u with u % 4 == wq and computes on those its
    // branch reads; both warps of a half release its stage
    const int br = warp / kDecBranchWarps, wq = warp % kDecBranchWarps;
    RowState<DV> rs;
    rs.init();
    const uint32_t qbase = smem_u32(qs);
    for (int u = wq; u < nh; u += kDecBranchWarps) {
      const int st = u % kDecStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (u / kDecStages) & 1, abort_flag, a.status, 412))) break;
      const uint32_t kb = smem_u32(ring + st * S::STAGE);
      const int blk = uni[u >> 1];
      const bool in_sel = flags[u >> 1] != 0u;
      const int first_key = blk * a.ls + (u & 1) * kTileKeys;
      const bool use = first_key <= t && (br == 0 ? in_sel : first_key + kTileKeys - 1 >= wlo);
      if (use) {
        float s[kNT][4];
        warp_qk_sq<DK, kNT>(qbase, 16 * 128, 0, kb, s, lane);
        const int key0 = first_key + (lane & 3) * 2;
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int tau0 = key0 + nt * 8 + e;
            const bool vis0 = tau0 <= t && (br == 0 || tau0 >= wlo);
            s[nt][e] = vis0 ? s[nt][e] * a.scale_log2 : -INFINITY;
            s[nt][2 + e] = vis0 ? s[nt][2 + e] * a.scale_log2 : -INFINITY;
          }
        }
        rs.update(s);
        warp_pv<DV, kNT>(s, kb + S::K_BYTES, rs.o, lane);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    rs.finish();
    // g_cmp * o_cmp of this thread's (row, 4 columns) items of the combine, from the
    // chunk outputs (L2) and the merge factors kept behind Q: formed before the
    // barrier, so their loads overlap the warps that are still streaming
    constexpr int kItems = 2;   // G * DV / 4 <= 512 items over 256 threads
    float4 ocm[kItems];
    {
      const PartLayout pl = part_layout(a);
      const int nch = (n_cmp_dev(L, a.l, a.s) + kCmpChunk - 1) / kCmpChunk;
      const float* cpo = a.part + pl.cp_o + bg * a.n_cmp_chunks * G * DV;
      const float* Li = reinterpret_cast<const float*>(qs + 8192);
      const float* Fc = Li + 16;
#pragma unroll
      for (int it = 0; it < kItems; ++it) {
        const int idx = tid + it * kDecConsumers * 32;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (idx < G * (DV / 4)) {
          const int row = idx / (DV / 4), c4 = (idx % (DV / 4)) * 4;
#pragma unroll 8
          for (int c = 0; c < nch; ++c) {   // independent L2 loads, issued together
            const float fc = Fc[c * 16 + row];
            const float4 v = *reinterpret_cast<const float4*>(cpo + ((size_t)c * G + row) * DV + c4);
            acc.x += fc * v.x; acc.y += fc * v.y; acc.z += fc * v.z; acc.w += fc * v.w;
          }
          const float scg = a.gates[((size_t)b * a.H_q + g * G + row) * 3 + 0] * Li[row];
          acc = make_float4(scg * acc.x, scg * acc.y, scg * acc.z, scg * acc.w);
        }
        ocm[it] = acc;
      }
    }
    named_bar_sync(1, kDecConsumers * 32);   // every block consumed: the ring is free
    TRD(7);
    float* stg = reinterpret_cast<float*>(ring);
    rs.stage(stg + warp * 16 * (DV + 2), lane);   // [branch][warp of branch][16][DV + 2]
    named_bar_sync(1, kDecConsumers * 32);
    // merge the four warps of each branch and combine: thread per (row, 4 columns)
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
      const int idx = tid + it * kDecConsumers * 32;
      if (idx >= G * (DV / 4)) break;
      const int row = idx / (DV / 4), c4 = (idx % (DV / 4)) * 4;
      const int hq = g * G + row;
      float4 res = ocm[it];
#pragma unroll
      for (int br = 0; br < 2; ++br) {
        const float* base = stg + (size_t)br * kDecBranchWarps * 16 * (DV + 2);
        float M = -1e30f;
#pragma unroll
        for (int w = 0; w < kDecBranchWarps; ++w) {
          const float* r = base + (w * 16 + row) * (DV + 2);
          if (r[DV + 1] > 0.f) M = fmaxf(M, r[DV]);
        }
        float den = 0.f;
        float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kDecBranchWarps; ++w) {
          const float* r = base + (w * 16 + row) * (DV + 2);
          if (r[DV + 1] > 0.f) {
            const float f = ex2(r[DV] - M);
            den += f * r[DV + 1];
            num.x += f * r[c4]; num.y += f * r[c4 + 1]; num.z += f * r[c4 + 2]; num.w += f * r[c4 + 3];
          }
        }
        const float gate = a.gates[((size_t)b * a.H_q + hq) * 3 + 1 + br];
        const float sc = den > 0.f ? gate / den : 0.f;
        res.x += sc * num.x; res.y += sc * num.y; res.z += sc * num.z; res.w += sc * num.w;
      }
      uint2 pk;
      pk.x = pack_bf16x2(res.x, res.y);
      pk.y = pack_bf16x2(res.z, res.w);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + ((size_t)b * a.H_q + hq) * DV + c4) = pk;
    }
  }
  __syncthreads();
  TRD(8);
#ifdef NSA_DECODE_TRACE
  if (threadIdx.x == 0 && fsp < 512) g_fspan[fsp][1] = globaltimer_ns();
#endif
}

template <int DK, int DV>
static cudaError_t launch_dec_t(const DecodeArgs& a, const DecodeMaps& m, cudaStream_t st) {
  using S = DecSmem<DK, DV>;
  cudaError_t e;
  auto k1 = dec_cmp_kernel<DK, DV>;
  auto k3 = dec_fine_kernel<DK, DV>;
  using S1 = D1Smem<DK, DV>;
  if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, S1::TOTAL)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, S::TOTAL)) != cudaSuccess) return e;
  if (a.Lmax_cmp > 0) {
    int dev = 0, n_sm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    const int n_items = a.B * a.H_kv * a.n_cmp_chunks;
    prof_begin(P_DEC_CMP, st);
    k1<<<n_items < n_sm ? n_items : n_sm, kD1Threads, S1::TOTAL, st>>>(a, m);
    prof_end(P_DEC_CMP, st, 1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  prof_begin(P_DEC_FINE, st);
  {
    // programmatic dependent launch: the fine pass's CTAs start (barriers, L2
    // prefetch of the window) while the compressed pass finishes
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.H_kv, a.B);
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = S::TOTAL;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, k3, a, m)) != cudaSuccess) return e;
  }
  prof_end(P_DEC_FINE, st, 1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return cudaGetLastError();
}

#ifdef NSA_DECODE_TRACE
extern "C" int nsa_decode_trace_read(void* dst) {
  return cudaMemcpyFromSymbol(dst, g_dtrace, sizeof(g_dtrace)) == cudaSuccess ? 0 : 1;
}
extern "C" int nsa_decode_fspan_read(void* dst) {
  return cudaMemcpyFromSymbol(dst, g_fspan, sizeof(g_fspan)) == cudaSuccess ? 0 : 1;
}
extern "C" int nsa_decode_cspan_read(void* dst) {
  return cudaMemcpyFromSymbol(dst, g_cspan, sizeof(g_cspan)) == cudaSuccess ? 0 : 1;
}
extern "C" int nsa_decode_ctrace_read(void* dst) {
  return cudaMemcpyFromSymbol(dst, g_ctrace, sizeof(g_ctrace)) == cudaSuccess ? 0 : 1;
}
#endif

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
