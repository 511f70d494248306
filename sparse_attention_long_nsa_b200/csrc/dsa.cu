// DSA variant: lightning indexer, token-level top-k, attention over the kept
// tokens ("Разреженное внимание — NSA и DSA", ai.flicky.cc, section "DSA:
// молниеносный индексатор"; the fused index-score + top-k idea of the DSA-vs-NSA
// post on web3.okx.com).
//
// For query t of a sequence: I[s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]) for
// every s <= t (FP8 E4M3 indexer queries and keys, fp32 weights); the top_k
// tokens by I (ties to the lower index; all of 0..t when t + 1 <= top_k) are kept
// and each query head attends to the raw keys/values of those tokens (GQA: head
// h uses KV head h / G; one selection serves every head).
//
// A query is (query row, first cache row of its sequence, position t); decode
// has one per sequence (t = len - 1), prefill one per token. Three kernels:
//   dsa_index  CTA = one query x 4096 keys: the indexer on warp-level FP8 MMA
//              (m16n8k32, e4m3 x e4m3 -> fp32): 16 rows = indexer heads, 8 keys
//              per MMA column block; ReLU, weights and the head sum in registers;
//              128-key tiles through a 3-stage cp.async ring
//   dsa_topk   CTA = one query: radix select of the top_k-th score over the
//              order-preserving bit pattern (digits of 12, 12 and 8 bits, shared-
//              memory histograms; each warp reads a contiguous run of scores with
//              coalesced float4 loads), then one pass in token order that keeps
//              every larger score and the first equal ones (ties to the lower
//              index); per-warp counts and lane scans place the kept tokens in
//              ascending order
//   dsa_attn   CTA = one query x one KV group: 8 warps take 256 kept tokens each,
//              gather their K/V rows with 16-byte cp.async into swizzled tiles of
//              16 keys and run an online softmax (16 rows = the group's heads);
//              the warps' states merge in shared memory into the bf16 output
#include "common.cuh"
#include "kernels.h"
#include "warp_mma.cuh"

namespace nsa {

namespace {

constexpr int kIdxChunk = 4096;     // keys per indexer CTA
constexpr int kIdxTile = 128;       // keys per shared-memory tile (32 per warp)
constexpr int kIdxStages = 3;
constexpr int kTopkThreads = 1024;
constexpr int kTopkBins = 4096;     // 12-bit digits in the first two radix passes
constexpr int kAttnWarps = 8;
constexpr int kAttnTile = 16;       // keys per gathered tile

__device__ __forceinline__ uint32_t ord_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// (query row, first cache row of the sequence, position t); false when the query
// does not exist (a decode length outside [1, max_len] is recorded)
__device__ __forceinline__ bool dsa_query(const DsaArgs& a, int slot, int64_t& qrow, int64_t& base, int& t) {
  const int64_t n = a.q0 + slot;
  if (a.lens) {   // decode: one query per sequence
    const int L = a.lens[n];
    if (L < 1 || L > a.max_len) {
      if (threadIdx.x == 0) atomicOr(a.status, DEV_ERR_BOUNDS);
      return false;
    }
    qrow = n;
    base = n * (int64_t)a.Lmax;
    t = L - 1;
    return true;
  }
  int lo = 0, hi = a.seqs.n - 1;   // prefill: token n of the packed batch
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.seqs.tok_off[mid] <= n) lo = mid; else hi = mid - 1;
  }
  qrow = n;
  base = a.seqs.tok_off[lo];
  t = (int)(n - base);
  return t < a.seqs.len[lo];
}

__device__ __forceinline__ void mma_e4m3_16832(float* c, const uint32_t* av, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(av[0]), "r"(av[1]), "r"(av[2]), "r"(av[3]), "r"(b0), "r"(b1));
}

}  // namespace

// ---------------------------------------------------------------------------
// indexer scores
// ---------------------------------------------------------------------------
template <int DI>
__global__ void __launch_bounds__(128) dsa_index_kernel(const DsaArgs a) {
  constexpr int ROW = DI + 16;                 // padded smem row (bytes): conflict-free fragment loads
  extern __shared__ __align__(16) uint8_t kt[];   // [kIdxStages][kIdxTile * ROW]
  __shared__ float wsm[16];
  const int slot = blockIdx.y;
  int64_t qrow, base;
  int t;
  if (!dsa_query(a, slot, qrow, base, t)) return;
  const int n_keys = t + 1;
  const int k0 = blockIdx.x * kIdxChunk;
  if (k0 >= n_keys) return;
  const int k1 = min(n_keys, k0 + kIdxChunk);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint8_t* qi = static_cast<const uint8_t*>(a.qi) + qrow * a.H_I * DI;
  const uint8_t* ki = static_cast<const uint8_t*>(a.ki) + base * DI;
  if (tid < 16) wsm[tid] = tid < a.H_I ? a.wi[qrow * a.H_I + tid] : 0.f;
  // A fragments of the indexer queries (rows = heads, zero above H_I), kept in registers
  uint32_t af[DI / 32][4];
  {
    const int r0 = lane >> 2, c4 = (lane & 3) * 4;
#pragma unroll
    for (int ks = 0; ks < DI / 32; ++ks) {
      af[ks][0] = r0 < a.H_I ? *reinterpret_cast<const uint32_t*>(qi + r0 * DI + ks * 32 + c4) : 0u;
      af[ks][1] = r0 + 8 < a.H_I ? *reinterpret_cast<const uint32_t*>(qi + (r0 + 8) * DI + ks * 32 + c4) : 0u;
      af[ks][2] = r0 < a.H_I ? *reinterpret_cast<const uint32_t*>(qi + r0 * DI + ks * 32 + 16 + c4) : 0u;
      af[ks][3] = r0 + 8 < a.H_I ? *reinterpret_cast<const uint32_t*>(qi + (r0 + 8) * DI + ks * 32 + 16 + c4) : 0u;
    }
  }
  const int n_tiles = (k1 - k0 + kIdxTile - 1) / kIdxTile;
  auto load_tile = [&](int it) {   // one commit group per tile (empty past the end)
    if (it < n_tiles) {
      constexpr int CH = DI / 16;   // 16-byte chunks per key
      uint8_t* dst = kt + (it % kIdxStages) * (kIdxTile * ROW);
      const int kb = k0 + it * kIdxTile;
      for (int i = tid; i < kIdxTile * CH; i += 128) {
        const int r = i / CH, c = i % CH;
        const int key = kb + r;
        cp_async16_zfill(dst + r * ROW + c * 16, ki + (int64_t)min(key, k1 - 1) * DI + c * 16, key < k1);
      }
    }
    cp_async_commit();
  };
  for (int it = 0; it < kIdxStages - 1; ++it) load_tile(it);
  __syncthreads();
  const float w0 = wsm[lane >> 2], w1 = wsm[(lane >> 2) + 8];
  float* dst = a.scores + (int64_t)slot * a.ld_scores;
  for (int it = 0; it < n_tiles; ++it) {
    load_tile(it + kIdxStages - 1);
    cp_async_wait<kIdxStages - 1>();
    __syncthreads();
    const uint8_t* tb = kt + (it % kIdxStages) * (kIdxTile * ROW);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {   // this warp's 32 keys: four blocks of 8
      const int kr = warp * 32 + nt * 8 + (lane >> 2);   // B column (key) of this lane
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < DI / 32; ++ks) {
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(tb + kr * ROW + ks * 32 + (lane & 3) * 4);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(tb + kr * ROW + ks * 32 + 16 + (lane & 3) * 4);
        mma_e4m3_16832(c, af[ks], b0, b1);
      }
      // c[0], c[1]: head lane/4, keys 2*(lane%4) + {0,1}; c[2], c[3]: head lane/4 + 8
      float s0 = fmaxf(c[0], 0.f) * w0 + fmaxf(c[2], 0.f) * w1;
      float s1 = fmaxf(c[1], 0.f) * w0 + fmaxf(c[3], 0.f) * w1;
#pragma unroll
      for (int off = 4; off <= 16; off <<= 1) {
        s0 += __shfl_xor_sync(0xffffffffu, s0, off);
        s1 += __shfl_xor_sync(0xffffffffu, s1, off);
      }
      if (lane < 4) {
        const int key = k0 + it * kIdxTile + warp * 32 + nt * 8 + lane * 2;
        if (key < k1) dst[key] = s0;
        if (key + 1 < k1) dst[key + 1] = s1;
      }
    }
    __syncthreads();   // the stage is reloaded kIdxStages - 1 tiles later
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// top-k over one query's scores
// ---------------------------------------------------------------------------
// exclusive prefix of `v` over the CTA's threads in index order (32 warps);
// `total` gets the CTA-wide sum. Uses wsum[32]; synchronises the CTA twice.
__device__ __forceinline__ uint32_t cta_excl_scan(uint32_t v, uint32_t* wsum, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += o;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = wsum[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t o = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += o;
    }
    wsum[lane] = w;   // inclusive prefix over warps
  }
  __syncthreads();
  total = wsum[31];
  const uint32_t before = warp > 0 ? wsum[warp - 1] : 0u;
  return before + x - v;
}

// The bin b of hist[0..nbins) with above(b) < need <= above(b) + hist[b], where
// above(b) counts the elements in the bins above b; sel = {b, above(b)}. Thread
// i owns bins nbins - 1 - (per i .. per i + per - 1), so the CTA scan runs from
// the top bin down. Synchronises the CTA.
__device__ __forceinline__ void topk_find_bin(const uint32_t* hist, int nbins, uint32_t need, uint32_t* wsum,
                                              uint32_t* sel) {
  const int tid = threadIdx.x;
  const int per = nbins >= kTopkThreads ? nbins / kTopkThreads : 1;
  const bool own = tid * per < nbins;
  uint32_t sum = 0u;
  if (own)
    for (int j = 0; j < per; ++j) sum += hist[nbins - 1 - (tid * per + j)];
  uint32_t total;
  uint32_t above = cta_excl_scan(sum, wsum, total);
  if (own && above < need && above + sum >= need) {
    for (int j = 0; j < per; ++j) {
      const int bin = nbins - 1 - (tid * per + j);
      if (above + hist[bin] >= need) {
        sel[0] = (uint32_t)bin;
        sel[1] = above;
        break;
      }
      above += hist[bin];
    }
  }
  __syncthreads();
}

// exclusive prefix of v over the lanes of a warp; `total` gets the warp's sum
__device__ __forceinline__ uint32_t warp_excl_scan(uint32_t v, uint32_t& total) {
  const int lane = threadIdx.x & 31;
  uint32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += o;
  }
  total = __shfl_sync(0xffffffffu, x, 31);
  return x - v;
}

__global__ void __launch_bounds__(kTopkThreads) dsa_topk_kernel(const DsaArgs a) {
  constexpr int kWarps = kTopkThreads / 32;
  __shared__ uint32_t hist[kTopkBins];
  __shared__ uint32_t wsum[32];
  __shared__ uint32_t sel[2];
  __shared__ uint32_t wcnt[2][kWarps];   // per warp: keys above the threshold, keys equal to it
  const int slot = blockIdx.x;
  int64_t qrow, base;
  int t;
  if (!dsa_query(a, slot, qrow, base, t)) return;
  const int n = t + 1, K = a.top_k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* out = a.idx + (int64_t)slot * K;
  const float* sc = a.scores + (int64_t)slot * a.ld_scores;
  if (n <= K) {
    for (int i = tid; i < K; i += kTopkThreads) out[i] = i < n ? i : -1;
    return;
  }
  // warp w owns the scores [wb, we) (a multiple of 128 long); it reads them in
  // chunks of 128, lane l taking 4 consecutive scores (float4 when aligned), so
  // every load is coalesced and the chunks go in token order
  const int span = ((n + kWarps - 1) / kWarps + 127) & ~127;
  const int wb = min(n, warp * span), we = min(n, wb + span);
  const bool vec = (reinterpret_cast<uintptr_t>(sc) & 15u) == 0;
  auto load4 = [&](int i, uint32_t* u) {   // keys of i .. i + 3 (0 beyond we: never selected)
    if (vec && i + 3 < we) {
      const float4 v = *reinterpret_cast<const float4*>(sc + i);
      u[0] = ord_key(v.x);
      u[1] = ord_key(v.y);
      u[2] = ord_key(v.z);
      u[3] = ord_key(v.w);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) u[e] = i + e < we ? ord_key(sc[i + e]) : 0u;
    }
  };
  auto visit = [&](auto&& f) {
    for (int i = wb + 4 * lane; i < we; i += 128) {
      uint32_t u[4];
      load4(i, u);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (i + e < we) f(u[e]);
    }
  };
  auto clear = [&](int nbins) {
    for (int i = tid; i < nbins; i += kTopkThreads) hist[i] = 0u;
    __syncthreads();
  };
  // radix select of the K-th largest order key: bits 31..20, 19..8, 7..0
  clear(kTopkBins);
  visit([&](uint32_t u) { atomicAdd(&hist[u >> 20], 1u); });
  __syncthreads();
  topk_find_bin(hist, kTopkBins, (uint32_t)K, wsum, sel);
  const uint32_t b1 = sel[0];
  uint32_t need = (uint32_t)K - sel[1];
  __syncthreads();
  clear(kTopkBins);
  visit([&](uint32_t u) {
    if ((u >> 20) == b1) atomicAdd(&hist[(u >> 8) & 4095u], 1u);
  });
  __syncthreads();
  topk_find_bin(hist, kTopkBins, need, wsum, sel);
  const uint32_t hi24 = (b1 << 12) | sel[0];
  need -= sel[1];
  __syncthreads();
  clear(256);
  visit([&](uint32_t u) {
    if ((u >> 8) == hi24) atomicAdd(&hist[u & 255u], 1u);
  });
  __syncthreads();
  topk_find_bin(hist, 256, need, wsum, sel);
  const uint32_t thr = (hi24 << 8) | sel[0];
  need -= sel[1];   // keys equal to thr still to take, in token order
  // every key above thr and the first `need` equal ones, in token order: the
  // warps' counts give each warp its starting rank and position, then each
  // chunk's ranks come from lane scans
  uint32_t gt = 0u, eq = 0u;
  visit([&](uint32_t u) {
    gt += u > thr ? 1u : 0u;
    eq += u == thr ? 1u : 0u;
  });
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    gt += __shfl_xor_sync(0xffffffffu, gt, off);
    eq += __shfl_xor_sync(0xffffffffu, eq, off);
  }
  if (lane == 0) {
    wcnt[0][warp] = gt;
    wcnt[1][warp] = eq;
  }
  __syncthreads();
  uint32_t gt_base = 0u, eq_rank = 0u;
  for (int w = 0; w < warp; ++w) {
    gt_base += wcnt[0][w];
    eq_rank += wcnt[1][w];
  }
  uint32_t pos = gt_base + min(eq_rank, need);
  for (int i = wb + 4 * lane; i - 4 * lane < we; i += 128) {   // warp-uniform trip count
    uint32_t u[4];
    load4(i, u);
    uint32_t ne = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) ne += (i + e < we && u[e] == thr) ? 1u : 0u;
    uint32_t ne_tot;
    uint32_t r = eq_rank + warp_excl_scan(ne, ne_tot);
    bool keep[4];
    uint32_t nk = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool in = i + e < we;
      keep[e] = in && u[e] > thr;
      if (in && u[e] == thr) keep[e] = r++ < need;
      nk += keep[e] ? 1u : 0u;
    }
    uint32_t nk_tot;
    uint32_t p = pos + warp_excl_scan(nk, nk_tot);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (keep[e]) {
        if (NSA_BOUNDS(p < (uint32_t)K, a.status, 701)) out[p] = i + e;
        ++p;
      }
    eq_rank += ne_tot;
    pos += nk_tot;
  }
}

// ---------------------------------------------------------------------------
// attention over the kept tokens
// ---------------------------------------------------------------------------
template <int DK, int DV>
struct DsaAttnSmem {
  static constexpr int KT = kAttnTile * DK * 2;     // one tile of K: DK/64 boxes of [16 keys][128 B]
  static constexpr int VT = kAttnTile * DV * 2;
  static constexpr int WARP = 2 * (KT + VT);        // double buffer per warp
  static constexpr int QS = (DK / 64) * 16 * 128;   // the group's query rows
  static constexpr int MERGE = kAttnWarps * 16 * (DV + 2) * 4;
  static constexpr int BODY = kAttnWarps * WARP > MERGE ? kAttnWarps * WARP : MERGE;
  static constexpr int TOTAL = 1024 + BODY + QS + 64;
};

template <int DK, int DV>
__global__ void __launch_bounds__(kAttnWarps * 32, 1) dsa_attn_kernel(const DsaArgs a) {
  using S = DsaAttnSmem<DK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* body = smem;
  uint8_t* qs = smem + S::BODY;
  const int slot = blockIdx.x, g = blockIdx.y;
  int64_t qrow, base;
  int t;
  if (!dsa_query(a, slot, qrow, base, t)) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G;
  const int n_kept = min(t + 1, a.top_k);
  const int32_t* kept = a.idx + (int64_t)slot * a.top_k;
  // the group's query rows (zero above G)
  for (int idx = tid; idx < 16 * (DK / 8); idx += kAttnWarps * 32) {
    const int row = idx / (DK / 8), c = idx % (DK / 8);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (row < G)
      v = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) +
                                          (qrow * a.H_q + g * G + row) * DK + c * 8);
    *reinterpret_cast<uint4*>(qs + (c >> 3) * 2048 + sw128(row, c & 7)) = v;
  }
  __syncthreads();
  const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(a.k);
  const __nv_bfloat16* vg = static_cast<const __nv_bfloat16*>(a.v);
  uint8_t* wbuf = body + warp * S::WARP;
  const int per_warp = (a.top_k + kAttnWarps - 1) / kAttnWarps;
  const int w_lo = warp * per_warp, w_hi = min(n_kept, w_lo + per_warp);
  const int n_tiles = w_hi > w_lo ? (w_hi - w_lo + kAttnTile - 1) / kAttnTile : 0;
  // gather the K/V rows of kept tokens w_lo + 16 it .. + 15 into buffer `buf`
  auto gather = [&](int buf, int it) {
    uint8_t* Kt = wbuf + buf * (S::KT + S::VT);
    uint8_t* Vt = Kt + S::KT;
    const int j0 = w_lo + it * kAttnTile;
    for (int i = lane; i < kAttnTile * (DK / 8); i += 32) {
      const int r = i / (DK / 8), c = i % (DK / 8);
      const int j = j0 + r;
      const int s = j < w_hi ? kept[j] : -1;
      const bool ok = s >= 0 && s <= t;
      cp_async16_zfill(Kt + (c >> 3) * (kAttnTile * 128) + sw128(r, c & 7),
                       kg + ((base + (ok ? s : 0)) * a.H_kv + g) * DK + c * 8, ok);
    }
    for (int i = lane; i < kAttnTile * (DV / 8); i += 32) {
      const int r = i / (DV / 8), c = i % (DV / 8);
      const int j = j0 + r;
      const int s = j < w_hi ? kept[j] : -1;
      const bool ok = s >= 0 && s <= t;
      cp_async16_zfill(Vt + (c >> 3) * (kAttnTile * 128) + sw128(r, c & 7),
                       vg + ((base + (ok ? s : 0)) * a.H_kv + g) * DV + c * 8, ok);
    }
    cp_async_commit();
  };
  RowState<DV> rs;
  rs.init();
  const uint32_t qbase = smem_u32(qs);
  if (n_tiles > 0) gather(0, 0);
  for (int it = 0; it < n_tiles; ++it) {
    if (it + 1 < n_tiles) {
      gather((it + 1) & 1, it + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();
    const uint32_t kb = smem_u32(wbuf + (it & 1) * (S::KT + S::VT));
    float s[2][4];
    warp_qk_sq<DK, 2>(qbase, 2048, 0, kb, s, lane);
    const int j0 = w_lo + it * kAttnTile + (lane & 3) * 2;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = j0 + nt * 8 + (e & 1);
        s[nt][e] = j < w_hi ? s[nt][e] * a.scale_log2 : -INFINITY;
      }
    rs.update(s);
    warp_pv<DV, 2>(s, kb + S::KT, rs.o, lane);
    __syncwarp();
  }
  rs.finish();
  __syncthreads();   // every warp is done with its gather buffers
  float* stg = reinterpret_cast<float*>(body);
  rs.stage(stg + warp * 16 * (DV + 2), lane);
  __syncthreads();
  for (int idx = tid; idx < G * (DV / 4); idx += kAttnWarps * 32) {
    const int row = idx / (DV / 4), c4 = (idx % (DV / 4)) * 4;
    float M = -1e30f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) {
      const float* r = stg + (w * 16 + row) * (DV + 2);
      if (r[DV + 1] > 0.f) M = fmaxf(M, r[DV]);
    }
    float den = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) {
      const float* r = stg + (w * 16 + row) * (DV + 2);
      if (r[DV + 1] > 0.f) {
        const float f = ex2(r[DV] - M);
        den += f * r[DV + 1];
        num.x += f * r[c4]; num.y += f * r[c4 + 1]; num.z += f * r[c4 + 2]; num.w += f * r[c4 + 3];
      }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    uint2 pk;
    pk.x = pack_bf16x2(num.x * inv, num.y * inv);
    pk.y = pack_bf16x2(num.z * inv, num.w * inv);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + (qrow * a.H_q + g * G + row) * DV + c4) = pk;
  }
}

// ---------------------------------------------------------------------------
// launch
// ---------------------------------------------------------------------------
template <int DK, int DV>
static cudaError_t launch_attn_t(const DsaArgs& a, int n_slots, cudaStream_t st) {
  using S = DsaAttnSmem<DK, DV>;
  auto k = dsa_attn_kernel<DK, DV>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, S::TOTAL);
  if (e != cudaSuccess) return e;
  k<<<dim3(n_slots, a.H_kv), kAttnWarps * 32, S::TOTAL, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dsa(const DsaArgs& a, int n_slots, int max_keys, int d_k, int d_v, int d_i, cudaStream_t st) {
  if (n_slots <= 0) return cudaSuccess;
  const dim3 gi((max_keys + kIdxChunk - 1) / kIdxChunk, n_slots);
  const size_t ism = (size_t)kIdxStages * kIdxTile * (d_i + 16);
  cudaError_t e = cudaSuccess;
  if (d_i == 64) e = cudaFuncSetAttribute(dsa_index_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ism);
  else if (d_i == 128) e = cudaFuncSetAttribute(dsa_index_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ism);
  else if (d_i == 32) e = cudaFuncSetAttribute(dsa_index_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ism);
  if (e != cudaSuccess) return e;
  prof_begin(P_DSA_INDEX, st);
  if (d_i == 64) dsa_index_kernel<64><<<gi, 128, ism, st>>>(a);
  else if (d_i == 128) dsa_index_kernel<128><<<gi, 128, ism, st>>>(a);
  else if (d_i == 32) dsa_index_kernel<32><<<gi, 128, ism, st>>>(a);
  else return cudaErrorInvalidValue;
  prof_end(P_DSA_INDEX, st, 1);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  prof_begin(P_DSA_TOPK, st);
  dsa_topk_kernel<<<n_slots, kTopkThreads, 0, st>>>(a);
  prof_end(P_DSA_TOPK, st, 1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  prof_begin(P_DSA_ATTN, st);
  if (d_k == 192 && d_v == 128) e = launch_attn_t<192, 128>(a, n_slots, st);
  else if (d_k == 64 && d_v == 64) e = launch_attn_t<64, 64>(a, n_slots, st);
  else if (d_k == 128 && d_v == 128) e = launch_attn_t<128, 128>(a, n_slots, st);
  else if (d_k == 192 && d_v == 64) e = launch_attn_t<192, 64>(a, n_slots, st);
  else if (d_k == 64 && d_v == 128) e = launch_attn_t<64, 128>(a, n_slots, st);
  else if (d_k == 128 && d_v == 64) e = launch_attn_t<128, 64>(a, n_slots, st);
  else e = cudaErrorInvalidValue;
  prof_end(P_DSA_ATTN, st, 1);
  return e;
}

}  // namespace nsa
