// Dense-tile attention on tcgen05 for two NSA branches of the prefill:
//
//  * compressed attention + importance ("Разреженное внимание — NSA и DSA",
//    ai.flicky.cc, section "NSA: три ветви": compression branch, and the
//    selection branch whose block scores are recomputed from the compressed
//    attention weights). Two passes over the compressed keys: pass 1 finds the
//    row max and softmax denominator, pass 2 forms the normalised probabilities,
//    spreads them over the selection blocks in proportion to token overlap
//    (summed over the GQA group's heads) and accumulates o_cmp = P.V_cmp.
//    Writes acc = g_cmp * o_cmp (fp32) and the block importance.
//
//  * sliding-window attention + gated combine (section "NSA: три ветви",
//    window branch; mask rule from section "Практика": key j visible to query i
//    iff j <= i and i - j < w). One online-softmax pass; the epilogue writes
//    out = bf16(acc + g_win * o_win), acc already holding the other branches.
//
// A CTA owns two query tiles of M = 128 rows, each (128/G tokens) x (G heads of
// one KV group), so every K/V tile staged in shared memory serves the group's
// heads of 2*128/G tokens. Roles (320 threads):
//   warps 0-3 / 4-7  softmax warpgroup of query tile 0 / 1, one accumulator row
//                    (TMEM lane) per thread
//   warp 8           TMA producer (both Q tiles once, then K/V tiles of 64 keys
//                    through a 3-stage ring)
//   warp 9           tcgen05.mma issuer, alternating the two tiles so that one
//                    tile's softmax overlaps the other tile's products:
//                    QK0(j) QK1(j) | PV0(j) QK0(j+1) PV1(j) QK1(j+1) | ...
// S = Q.K^T lands in TMEM; the softmax threads read it with tcgen05.ld, write P
// (bf16) back to TMEM, and O += P.V runs with A = P from TMEM and V as an
// MN-major shared-memory operand, accumulating in TMEM. The window pass keeps a
// reference max per row and rescales O in TMEM only when the running max grows
// by more than 8 (log2 units); exact, since O and the denominator always share
// the reference.
#include "common.cuh"
#include "kernels.h"

namespace nsa {

namespace {

constexpr int kStages = 3;
constexpr int kKeyTile = 64;
constexpr int kThreads = 320;
constexpr float kRescaleThreshold = 8.f;

// TMEM columns (512 allocated): S, P and O of query tile q
__device__ __forceinline__ uint32_t col_s(int q) { return q ? 64u : 0u; }
__device__ __forceinline__ uint32_t col_p(int q) { return q ? 160u : 128u; }
__device__ __forceinline__ uint32_t col_o(int q) { return q ? 384u : 256u; }

struct Bars {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full[2];
  uint64_t o_done[2];
  uint64_t drain;       // MMA issuer: all its products finished (exit path)
  uint32_t tmem_base;
  int abort;
};

template <int DK, int DV>
struct TcSmem {
  static constexpr int Q_BYTES = 128 * DK * 2;   // one query tile
  static constexpr int K_BYTES = kKeyTile * DK * 2;
  static constexpr int V_BYTES = kKeyTile * DV * 2;
  static constexpr int STAGE = K_BYTES + V_BYTES;
  static constexpr int TOTAL = 1024 + 2 * Q_BYTES + kStages * STAGE + (int)sizeof(Bars) + 64;
};

__device__ __forceinline__ int seq_of_tile(const SeqTable& t, int tile) {
  int lo = 0, hi = t.n - 1;
  while (lo < hi) {   // last b with tile_prefix[b] <= tile
    const int mid = (lo + hi + 1) >> 1;
    if (t.tile_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int cmp_visible_dev(int t, int l, int s) {
  return t >= l - 1 ? (t - l + 1) / s + 1 : 0;
}

}  // namespace

// MODE 0: compressed attention + importance; MODE 1: window attention + combine
template <int MODE, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const PrefillArgs a, const __grid_constant__ PrefillMaps m) {
  using S = TcSmem<DK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Qs = smem;                                 // [2][Q_BYTES]
  uint8_t* KVs = smem + 2 * S::Q_BYTES;               // [kStages][STAGE]
  Bars* bars = reinterpret_cast<Bars*>(KVs + kStages * S::STAGE);
  volatile int* abort_flag = &bars->abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G;
  const int TOK = 128 / G;                            // tokens per query tile
  const int tile = blockIdx.x;
  const int g = blockIdx.y;
  const int b = seq_of_tile(a.seqs, tile);
  const int L = a.seqs.len[b];
  const int64_t tok0 = a.seqs.tok_off[b];
  const int t0 = (tile - a.seqs.tile_prefix[b]) * 2 * TOK;
  const int t_last = min(t0 + 2 * TOK - 1, L - 1);

  // key tiles shared by both query tiles
  int nk, key0;
  if (MODE == 0) {
    const int nv = cmp_visible_dev(t_last, a.l, a.s);
    nk = (nv + kKeyTile - 1) / kKeyTile;
    key0 = 0;
  } else {
    const int lo = max(0, t0 - a.window + 1);
    key0 = (lo / kKeyTile) * kKeyTile;
    nk = (t_last - key0) / kKeyTile + 1;
  }
  const int n_s = (MODE == 0) ? 2 * nk : nk;         // S tiles per query tile

  if (tid == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < kStages; ++i) { mbar_init(&bars->kv_full[i], 1); mbar_init(&bars->kv_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], 128);
      mbar_init(&bars->p_full[i], 128);
      mbar_init(&bars->o_done[i], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&bars->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nk > 0) {
      prefetch_tmap(&m.q);
      const CUtensorMap* mk = MODE == 0 ? &m.kc : &m.k;
      const CUtensorMap* mv = MODE == 0 ? &m.vc : &m.v;
      const int64_t krow0 = MODE == 0 ? a.seqs.cmp_off[b] : tok0;
      mbar_arrive_expect_tx(&bars->q_full, 2 * S::Q_BYTES);
      for (int qt = 0; qt < 2; ++qt)
        for (int kb = 0; kb < DK / 64; ++kb)
          tma_load_3d(Qs + qt * S::Q_BYTES + kb * 16384, &m.q, &bars->q_full, kb * 64, g * G,
                      (int)(tok0 + t0 + qt * TOK));
      int issued = 0;
      for (int jj = 0; jj < n_s; ++jj) {
        const int st = jj % kStages;
        const int j = (MODE == 0 && jj >= nk) ? jj - nk : jj;
        const bool with_v = (MODE == 1) || jj >= nk;
        if (jj >= kStages &&
            !mbar_wait(&bars->kv_empty[st], ((jj / kStages) - 1) & 1, abort_flag, a.status, 201))
          break;
        issued = jj + 1;
        uint8_t* Ks = KVs + st * S::STAGE;
        mbar_arrive_expect_tx(&bars->kv_full[st], S::K_BYTES + (with_v ? S::V_BYTES : 0));
        const int row = (int)(krow0 + key0 + j * kKeyTile);
        for (int kb = 0; kb < DK / 64; ++kb) tma_load_3d(Ks + kb * 8192, mk, &bars->kv_full[st], kb * 64, g, row);
        if (with_v)
          for (int vb = 0; vb < DV / 64; ++vb)
            tma_load_3d(Ks + S::K_BYTES + vb * 8192, mv, &bars->kv_full[st], vb * 64, g, row);
      }
      if (*abort_flag) {   // let the copies still in flight land before the CTA exits
        mbar_wait_drain(&bars->q_full, 0);
        for (int v = issued - kStages < 0 ? 0 : issued - kStages; v < issued; ++v)
          mbar_wait_drain(&bars->kv_full[v % kStages], (v / kStages) & 1);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nk > 0) {
      const uint32_t idesc_qk = umma_idesc_bf16(128, kKeyTile, false, false);
      const uint32_t idesc_pv = umma_idesc_bf16(128, DV, false, true);
      const uint32_t q_addr = smem_u32(Qs);
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, a.status, 211);
      auto qk = [&](int q, int jj) -> bool {
        if (jj >= 1 && !mbar_wait(&bars->s_free[q], (jj - 1) & 1, abort_flag, a.status, 212)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(KVs + (jj % kStages) * S::STAGE);
        const uint32_t qa = q_addr + q * S::Q_BYTES;
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint64_t dq = umma_desc_sw128(qa + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t dk = umma_desc_sw128(k_addr + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
          umma_ss(tmem + col_s(q), dq, dk, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full[q]);
        return true;
      };
      auto pv = [&](int q, int jj, int jp) -> bool {
        if (!mbar_wait(&bars->p_full[q], jp & 1, abort_flag, a.status, 213)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(KVs + (jj % kStages) * S::STAGE + S::K_BYTES);
#pragma unroll
        for (int kk = 0; kk < kKeyTile / 16; ++kk) {
          const uint64_t dv = umma_desc_sw128(v_addr + kk * 2048, 8192, 1024);
          umma_ts(tmem + col_o(q), tmem + col_p(q) + kk * 8, dv, idesc_pv, (jp > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars->o_done[q]);
        return true;
      };
      if (ok) ok = mbar_wait(&bars->kv_full[0], 0, abort_flag, a.status, 214);
      if (ok) ok = qk(0, 0) && qk(1, 0);
      for (int jj = 0; jj < n_s && ok; ++jj) {
        const int st = jj % kStages;
        const bool pv_pass = (MODE == 1) || jj >= nk;
        const int jp = MODE == 1 ? jj : jj - nk;
        const bool more = jj + 1 < n_s;
        if (pv_pass && !pv(0, jj, jp)) break;
        if (more) {
          const int s1 = jj + 1;
          if (!mbar_wait(&bars->kv_full[s1 % kStages], (s1 / kStages) & 1, abort_flag, a.status, 215)) break;
          if (!qk(0, s1)) break;
        }
        if (pv_pass && !pv(1, jj, jp)) break;
        umma_commit(&bars->kv_empty[st]);   // every product reading stage st has been issued
        if (more && !qk(1, jj + 1)) break;
      }
      // every issued product has finished before the CTA releases tensor memory
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int q = warp >> 2;                 // query tile
    const int r = tid & 127;                 // row within the tile = TMEM lane
    const int tt = r / G, hh = r % G;
    const int t = t0 + q * TOK + tt;
    const bool valid = t < L;
    const int h = g * G + hh;
    const int64_t n = tok0 + t;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t colS = tmem + lane_base + col_s(q);
    const uint32_t colP = tmem + lane_base + col_p(q);
    const uint32_t colO = tmem + lane_base + col_o(q);
    const float sc = a.scale_log2;
    float row_m = -1e30f, row_l = 0.f;
    bool ok = true;
    int nvis = 0, wlo = 0;
    if (MODE == 0) nvis = valid ? cmp_visible_dev(t, a.l, a.s) : 0;
    else wlo = max(0, t - a.window + 1);
    const int jt = t / a.ls;
    float* imp_row = a.imp + ((size_t)n * a.H_kv + g) * a.nb_stride;
    float carry = 0.f;
    float linv = 0.f;

    auto load_s = [&](int jj, float* sv) -> bool {
      if (!mbar_wait(&bars->s_full[q], jj & 1, abort_flag, a.status, 221)) return false;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kKeyTile; c += 16) tmem_ld16(colS + c, sv + c);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars->s_free[q]);
      return true;
    };
    // P tile jp into TMEM once PV(jp-1) has finished reading the previous one
    auto store_p = [&](int jp, const float* p, float alpha) -> bool {
      if (jp >= 1) {
        if (!mbar_wait(&bars->o_done[q], (jp - 1) & 1, abort_flag, a.status, 222)) return false;
        tc_fence_after();
        if (MODE == 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
          // rescale this row of O (rare: the running max grew past the threshold)
#pragma unroll 1
          for (int c = 0; c < DV; c += 16) {
            float ov[16];
            tmem_ld16(colO + c, ov);
            tmem_ld_wait();
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) w[i] = __float_as_uint(ov[i] * alpha);
            tmem_st8(colO + c, w);
            tmem_st8(colO + c + 8, w + 8);
          }
        }
      }
#pragma unroll
      for (int c = 0; c < kKeyTile / 16; ++c) {
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(p[c * 16 + 2 * i], p[c * 16 + 2 * i + 1]);
        tmem_st8(colP + c * 8, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[q]);
      return true;
    };

    if (MODE == 0) {
      // ---- pass 1: row max and denominator
      for (int j = 0; j < nk && ok; ++j) {
        float sv[kKeyTile];
        if (!load_s(j, sv)) { ok = false; break; }
        float mx = -1e30f;
#pragma unroll
        for (int c = 0; c < kKeyTile; ++c) {
          sv[c] = (j * kKeyTile + c < nvis) ? sv[c] * sc : -INFINITY;
          mx = fmaxf(mx, sv[c]);
        }
        const float m_new = fmaxf(row_m, mx);
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < kKeyTile; ++c) sum += ex2(sv[c] - m_new);
        row_l = row_l * ex2(row_m - m_new) + sum;
        row_m = m_new;
      }
      linv = row_l > 0.f ? 1.f / row_l : 0.f;
      // ---- pass 2: probabilities, importance, O += P.V
      for (int j = 0; j < nk && ok; ++j) {
        float sv[kKeyTile];
        if (!load_s(nk + j, sv)) { ok = false; break; }
#pragma unroll
        for (int c = 0; c < kKeyTile; ++c)
          sv[c] = (j * kKeyTile + c < nvis) ? ex2(sv[c] * sc - row_m) * linv : 0.f;
        if (!store_p(j, sv, 1.f)) { ok = false; break; }
        // spread over selection blocks: compressed token i = 4u' + u covers tokens
        // [16i, 16i + 32): u in {0,1,2} -> 2p into block u'; u = 3 -> p into u' and u'+1
        float blk[17];
#pragma unroll
        for (int qb = 0; qb < 16; ++qb) {
          const float* pp = sv + 4 * qb;
          blk[qb] = 2.f * (pp[0] + pp[1] + pp[2]) + pp[3];
        }
        blk[16] = 0.f;
#pragma unroll
        for (int qb = 0; qb < 16; ++qb) blk[qb + 1] += sv[4 * qb + 3];
        // sum over the G heads of this token (G consecutive lanes); the carry from
        // the previous tile is already a group sum, so it is added after
#pragma unroll
        for (int qb = 0; qb < 17; ++qb) {
          float x = blk[qb];
          for (int off = G >> 1; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
          blk[qb] = x;
        }
        blk[0] += carry;
        carry = blk[16];
        if (valid)
          for (int qb = hh; qb < 16; qb += G) {
            const int jb = j * 16 + qb;
            if (jb <= jt) imp_row[jb] = blk[qb];
          }
      }
      if (ok && valid)   // the carried block and blocks no visible compressed token reaches
        for (int jb = nk * 16 + hh; jb <= jt; jb += G) imp_row[jb] = (jb == nk * 16) ? carry : 0.f;
    } else {
      // ---- window: one online-softmax pass with a lazily rescaled reference max
      for (int j = 0; j < nk && ok; ++j) {
        float sv[kKeyTile];
        if (!load_s(j, sv)) { ok = false; break; }
        float mx = -1e30f;
#pragma unroll
        for (int c = 0; c < kKeyTile; ++c) {
          const int tau = key0 + j * kKeyTile + c;
          const bool vis = valid && tau <= t && tau >= wlo;
          sv[c] = vis ? sv[c] * sc : -INFINITY;
          mx = fmaxf(mx, sv[c]);
        }
        float alpha = 1.f;
        if (mx > row_m + kRescaleThreshold) {
          alpha = ex2(row_m - mx);
          row_l *= alpha;
          row_m = mx;
        }
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < kKeyTile; ++c) {
          sv[c] = ex2(sv[c] - row_m);
          sum += sv[c];
        }
        row_l += sum;
        if (!store_p(j, sv, alpha)) { ok = false; break; }
      }
      linv = row_l > 0.f ? 1.f / row_l : 0.f;
    }

    // ---- epilogue: O (TMEM) -> output
    const int n_pv = nk;
    if (ok && n_pv > 0) ok = mbar_wait(&bars->o_done[q], (n_pv - 1) & 1, abort_flag, a.status, 223);
    tc_fence_after();
    if (ok && n_pv > 0) {
      const float* gsrc = a.gates + ((size_t)n * a.H_q + h) * 3;
      float* accp = a.acc + ((size_t)n * a.H_q + h) * DV;
#pragma unroll 1
      for (int c = 0; c < DV; c += 32) {
        float ov[32];
        tmem_ld16(colO + c, ov);
        tmem_ld16(colO + c + 16, ov + 16);
        tmem_ld_wait();
        if (!valid) continue;
        if (MODE == 0) {
          const float gc = gsrc[0];   // P was normalised already
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(accp + c + i) =
                make_float4(gc * ov[i], gc * ov[i + 1], gc * ov[i + 2], gc * ov[i + 3]);
        } else {
          const float gw = gsrc[2] * linv;
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + ((size_t)n * a.H_q + h) * DV + c;
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            const float4 a0 = *reinterpret_cast<const float4*>(accp + c + i);
            const float4 a1 = *reinterpret_cast<const float4*>(accp + c + i + 4);
            uint4 pk;
            pk.x = pack_bf16x2(fmaf(gw, ov[i + 0], a0.x), fmaf(gw, ov[i + 1], a0.y));
            pk.y = pack_bf16x2(fmaf(gw, ov[i + 2], a0.z), fmaf(gw, ov[i + 3], a0.w));
            pk.z = pack_bf16x2(fmaf(gw, ov[i + 4], a1.x), fmaf(gw, ov[i + 5], a1.y));
            pk.w = pack_bf16x2(fmaf(gw, ov[i + 6], a1.z), fmaf(gw, ov[i + 7], a1.w));
            *reinterpret_cast<uint4*>(dst + i) = pk;
          }
        }
      }
    }
    if (MODE == 0 && nk == 0 && valid) {
      // no compressed token visible to any row: o_cmp = 0, importance 0
      for (int jb = hh; jb <= jt; jb += G) imp_row[jb] = 0.f;
      float* accp = a.acc + ((size_t)n * a.H_q + h) * DV;
      for (int c = 0; c < DV; c += 4) *reinterpret_cast<float4*>(accp + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int MODE, int DK, int DV>
static cudaError_t launch_tc(const PrefillArgs& a, const PrefillMaps& m, int n_tiles, cudaStream_t st) {
  using S = TcSmem<DK, DV>;
  auto kern = attn_tc_kernel<MODE, DK, DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::TOTAL);
  if (e != cudaSuccess) return e;
  kern<<<dim3(n_tiles, a.H_kv), kThreads, S::TOTAL, st>>>(a, m);
  return cudaGetLastError();
}

template <int MODE>
static cudaError_t dispatch(const PrefillArgs& a, const PrefillMaps& m, int n_tiles, cudaStream_t st) {
  if (n_tiles <= 0) return cudaSuccess;
  if (a.d_k == 192 && a.d_v == 128) return launch_tc<MODE, 192, 128>(a, m, n_tiles, st);
  if (a.d_k == 64 && a.d_v == 64) return launch_tc<MODE, 64, 64>(a, m, n_tiles, st);
  if (a.d_k == 128 && a.d_v == 128) return launch_tc<MODE, 128, 128>(a, m, n_tiles, st);
  if (a.d_k == 192 && a.d_v == 64) return launch_tc<MODE, 192, 64>(a, m, n_tiles, st);
  if (a.d_k == 64 && a.d_v == 128) return launch_tc<MODE, 64, 128>(a, m, n_tiles, st);
  if (a.d_k == 128 && a.d_v == 64) return launch_tc<MODE, 128, 64>(a, m, n_tiles, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_cmp_attn(const PrefillArgs& a, const PrefillMaps& m, int n_tiles, cudaStream_t st) {
  return dispatch<0>(a, m, n_tiles, st);
}
cudaError_t launch_win_attn(const PrefillArgs& a, const PrefillMaps& m, int n_tiles, cudaStream_t st) {
  return dispatch<1>(a, m, n_tiles, st);
}

}  // namespace nsa
