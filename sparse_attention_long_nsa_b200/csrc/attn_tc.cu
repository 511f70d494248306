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
// Tile: M = 128 rows = (128/G tokens) x (G heads of one KV group), so every
// K/V tile staged in shared memory serves the whole GQA group. Roles:
//   warps 0-3  softmax + epilogue, one accumulator row (TMEM lane) per thread
//   warp 4     TMA producer (Q once, then K/V tiles of 64 keys, 2-stage ring)
//   warp 5     tcgen05.mma issuer (S = Q.K^T into TMEM; O_tile = P.V with P
//              read from TMEM and V as an MN-major shared-memory operand)
#include "common.cuh"
#include "kernels.h"

namespace nsa {

namespace {

constexpr int kStages = 2;
constexpr int kKeyTile = 64;
constexpr int kThreads = 192;

// TMEM column map (512 allocated)
constexpr uint32_t kColS0 = 0, kColS1 = 64, kColP0 = 128, kColP1 = 160, kColO = 256;

struct Bars {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full[2];
  uint64_t o_full;
  uint64_t o_free;
  uint32_t tmem_base;
  int abort;
};

template <int DK, int DV>
struct TcSmem {
  static constexpr int Q_BYTES = 128 * DK * 2;
  static constexpr int K_BYTES = kKeyTile * DK * 2;
  static constexpr int V_BYTES = kKeyTile * DV * 2;
  static constexpr int STAGE = K_BYTES + V_BYTES;
  static constexpr int TOTAL = 1024 + Q_BYTES + kStages * STAGE + (int)sizeof(Bars) + 64;
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
  uint8_t* Qs = smem;
  uint8_t* KVs = smem + S::Q_BYTES;
  Bars* bars = reinterpret_cast<Bars*>(KVs + kStages * S::STAGE);
  volatile int* abort_flag = &bars->abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G;
  const int TOK = 128 / G;
  const int tile = blockIdx.x;
  const int g = blockIdx.y;
  const int b = seq_of_tile(a.seqs, tile);
  const int L = a.seqs.len[b];
  const int64_t tok0 = a.seqs.tok_off[b];
  const int t0 = (tile - a.seqs.tile_prefix[b]) * TOK;
  const int t_last = min(t0 + TOK - 1, L - 1);

  // key tiles
  int nk, key0;   // number of 64-key tiles and the first key (sequence-local)
  if (MODE == 0) {
    const int nv = cmp_visible_dev(t_last, a.l, a.s);
    nk = (nv + kKeyTile - 1) / kKeyTile;
    key0 = 0;
  } else {
    const int lo = max(0, t0 - a.window + 1);
    key0 = (lo / kKeyTile) * kKeyTile;
    nk = (t_last - key0) / kKeyTile + 1;
  }
  const int n_s = (MODE == 0) ? 2 * nk : nk;   // S tiles produced

  if (tid == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < kStages; ++i) { mbar_init(&bars->kv_full[i], 1); mbar_init(&bars->kv_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], 128);
      mbar_init(&bars->p_full[i], 128);
    }
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->o_free, 128);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&bars->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nk > 0) {
      prefetch_tmap(&m.q);
      const CUtensorMap* mk = MODE == 0 ? &m.kc : &m.k;
      const CUtensorMap* mv = MODE == 0 ? &m.vc : &m.v;
      const int64_t krow0 = MODE == 0 ? a.seqs.cmp_off[b] : tok0;
      mbar_arrive_expect_tx(&bars->q_full, S::Q_BYTES);
      for (int kb = 0; kb < DK / 64; ++kb)
        tma_load_3d(Qs + kb * 16384, &m.q, &bars->q_full, kb * 64, g * G, (int)(tok0 + t0));
      int it = 0;
      const int passes = MODE == 0 ? 2 : 1;
      bool ok = true;
      for (int pass = 0; pass < passes && ok; ++pass) {
        const bool with_v = (MODE == 1) || pass == 1;
        for (int j = 0; j < nk; ++j, ++it) {
          const int st = it % kStages;
          if (it >= kStages &&
              !mbar_wait(&bars->kv_empty[st], ((it / kStages) - 1) & 1, abort_flag, a.status, 201)) {
            ok = false;
            break;
          }
          uint8_t* Ks = KVs + st * S::STAGE;
          uint8_t* Vs = Ks + S::K_BYTES;
          mbar_arrive_expect_tx(&bars->kv_full[st], S::K_BYTES + (with_v ? S::V_BYTES : 0));
          const int row = (int)(krow0 + key0 + j * kKeyTile);
          for (int kb = 0; kb < DK / 64; ++kb) tma_load_3d(Ks + kb * 8192, mk, &bars->kv_full[st], kb * 64, g, row);
          if (with_v)
            for (int vb = 0; vb < DV / 64; ++vb) tma_load_3d(Vs + vb * 8192, mv, &bars->kv_full[st], vb * 64, g, row);
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nk > 0) {
      const uint32_t idesc_qk = umma_idesc_bf16(128, kKeyTile, false, false);
      const uint32_t idesc_pv = umma_idesc_bf16(128, DV, false, true);
      const uint32_t q_addr = smem_u32(Qs);
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, a.status, 211);
      int it = 0;          // K/V stage counter
      int pv = 0;          // PV products issued
      int prev_st = 0;
      auto issue_pv = [&](int jp, int st) -> bool {
        // P_jp ready, previous O tile consumed
        if (!mbar_wait(&bars->p_full[jp & 1], (jp >> 1) & 1, abort_flag, a.status, 212)) return false;
        if (pv >= 1 && !mbar_wait(&bars->o_free, (pv - 1) & 1, abort_flag, a.status, 213)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(KVs + st * S::STAGE + S::K_BYTES);
        const uint32_t p_col = (jp & 1) ? kColP1 : kColP0;
#pragma unroll
        for (int kk = 0; kk < kKeyTile / 16; ++kk) {
          const uint64_t dv = umma_desc_sw128(v_addr + kk * 2048, 8192, 1024);
          umma_ts(tmem + kColO, tmem + p_col + kk * 8, dv, idesc_pv, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->o_full);
        umma_commit(&bars->kv_empty[st]);
        ++pv;
        return true;
      };
      for (int jj = 0; jj < n_s && ok; ++jj, ++it) {
        const int st = it % kStages;
        if (!mbar_wait(&bars->kv_full[st], (it / kStages) & 1, abort_flag, a.status, 214)) { ok = false; break; }
        const int sb = jj & 1;
        if (jj >= 2 && !mbar_wait(&bars->s_free[sb], ((jj - 2) >> 1) & 1, abort_flag, a.status, 215)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(KVs + st * S::STAGE);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint64_t dq = umma_desc_sw128(q_addr + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t dk = umma_desc_sw128(k_addr + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
          umma_ss(tmem + (sb ? kColS1 : kColS0), dq, dk, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full[sb]);
        const bool pv_pass = (MODE == 1) || jj >= nk;
        const int jp = MODE == 1 ? jj : jj - nk;   // index within the PV pass
        if (!pv_pass) {
          umma_commit(&bars->kv_empty[st]);      // K-only stage is free once S is done
        } else if (jp >= 1) {
          if (!issue_pv(jp - 1, prev_st)) { ok = false; break; }
        }
        prev_st = st;
      }
      if (ok) issue_pv(MODE == 1 ? nk - 1 : nk - 1, prev_st);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int r = tid;                 // accumulator row
    const int tt = r / G, hh = r % G;
    const int t = t0 + tt;
    const bool valid = t < L;
    const int h = g * G + hh;
    const int64_t n = tok0 + t;        // global token row
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float o_acc[DV];
#pragma unroll
    for (int i = 0; i < DV; ++i) o_acc[i] = 0.f;
    float row_m = -1e30f, row_l = 0.f;
    const float sc = a.scale_log2;
    bool ok = true;

    // visibility of key c of tile j for this row
    int nvis = 0, wlo = 0;
    if (MODE == 0) nvis = valid ? cmp_visible_dev(t, a.l, a.s) : 0;
    else wlo = max(0, t - a.window + 1);

    // importance state (MODE 0): tile j covers blocks 16j .. 16j+16
    float carry = 0.f;
    const int jt = t / a.ls;
    const int nb_stride = a.nb_stride;
    float* imp_row = a.imp + ((size_t)n * a.H_kv + g) * nb_stride;

    auto load_s = [&](int jj, float* sv) -> bool {
      const int sb = jj & 1;
      if (!mbar_wait(&bars->s_full[sb], (jj >> 1) & 1, abort_flag, a.status, 221)) return false;
      tc_fence_after();
      const uint32_t col = sb ? kColS1 : kColS0;
#pragma unroll
      for (int c = 0; c < kKeyTile; c += 16) tmem_ld16(tmem + lane_base + col + c, sv + c);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars->s_free[sb]);
      return true;
    };
    auto store_p = [&](int jp, const float* p) {
      const uint32_t col = (jp & 1) ? kColP1 : kColP0;
#pragma unroll
      for (int c = 0; c < kKeyTile / 16; ++c) {
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(p[c * 16 + 2 * i], p[c * 16 + 2 * i + 1]);
        tmem_st8(tmem + lane_base + col + c * 8, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[jp & 1]);
    };
    auto add_o = [&](int jp, float alpha) -> bool {
      if (!mbar_wait(&bars->o_full, jp & 1, abort_flag, a.status, 222)) return false;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < DV; c += 16) {
        float ov[16];
        tmem_ld16(tmem + lane_base + kColO + c, ov);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) o_acc[c + i] = fmaf(o_acc[c + i], alpha, ov[i]);
      }
      tc_fence_before();
      mbar_arrive(&bars->o_free);
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
          const int i = j * kKeyTile + c;
          sv[c] = (i < nvis) ? sv[c] * sc : -INFINITY;
          mx = fmaxf(mx, sv[c]);
        }
        const float m_new = fmaxf(row_m, mx);
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < kKeyTile; ++c) sum += exp2f(sv[c] - m_new);
        row_l = row_l * exp2f(row_m - m_new) + sum;
        row_m = m_new;
      }
      const float linv = row_l > 0.f ? 1.f / row_l : 0.f;
      // ---- pass 2: probabilities, importance, P.V
      for (int j = 0; j < nk && ok; ++j) {
        float sv[kKeyTile];
        if (!load_s(nk + j, sv)) { ok = false; break; }
#pragma unroll
        for (int c = 0; c < kKeyTile; ++c) {
          const int i = j * kKeyTile + c;
          sv[c] = (i < nvis) ? exp2f(sv[c] * sc - row_m) * linv : 0.f;
        }
        store_p(j, sv);
        // spread over selection blocks: compressed token i = 4q + u covers tokens
        // [16i, 16i + 32): u in {0,1,2} -> 2p into block q; u = 3 -> p into q and q+1
        float blk[17];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float* pp = sv + 4 * q;
          blk[q] = 2.f * (pp[0] + pp[1] + pp[2]) + pp[3];
        }
        blk[16] = 0.f;
#pragma unroll
        for (int q = 0; q < 16; ++q) blk[q + 1] += sv[4 * q + 3];
        // sum over the G heads of this token (G consecutive lanes); the carry
        // from the previous tile is already a group sum, so it is added after
#pragma unroll
        for (int q = 0; q < 17; ++q) {
          float x = blk[q];
          for (int off = G >> 1; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
          blk[q] = x;
        }
        blk[0] += carry;
        carry = blk[16];
        if (valid) {
          for (int q = hh; q < 16; q += G) {
            const int jb = j * 16 + q;
            if (jb <= jt) imp_row[jb] = blk[q];
          }
        }
        if (j >= 1 && !add_o(j - 1, 1.f)) { ok = false; break; }
      }
      if (ok && nk > 0 && !add_o(nk - 1, 1.f)) ok = false;
      if (ok && valid) {
        // the carried block and blocks no visible compressed token reaches
        for (int jb = nk * 16 + hh; jb <= jt; jb += G) imp_row[jb] = (jb == nk * 16) ? carry : 0.f;
        float* dst = a.acc + ((size_t)n * a.H_q + h) * DV;
        const float gc = a.gates[((size_t)n * a.H_q + h) * 3 + 0];
#pragma unroll
        for (int c = 0; c < DV; c += 4)
          *reinterpret_cast<float4*>(dst + c) =
              make_float4(gc * o_acc[c], gc * o_acc[c + 1], gc * o_acc[c + 2], gc * o_acc[c + 3]);
      }
    } else {
      // ---- window: single online-softmax pass
      float alpha_prev = 1.f;
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
        const float m_new = fmaxf(row_m, mx);
        const float alpha = exp2f(row_m - m_new);
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < kKeyTile; ++c) {
          sv[c] = exp2f(sv[c] - m_new);
          sum += sv[c];
        }
        row_l = row_l * alpha + sum;
        row_m = m_new;
        store_p(j, sv);
        if (j >= 1 && !add_o(j - 1, alpha_prev)) { ok = false; break; }
        alpha_prev = alpha;
      }
      if (ok && !add_o(nk - 1, alpha_prev)) ok = false;
      if (ok && valid) {
        const float linv = row_l > 0.f ? 1.f / row_l : 0.f;
        const float gw = a.gates[((size_t)n * a.H_q + h) * 3 + 2] * linv;
        const float* src = a.acc + ((size_t)n * a.H_q + h) * DV;
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + ((size_t)n * a.H_q + h) * DV;
#pragma unroll
        for (int c = 0; c < DV; c += 8) {
          const float4 a0 = *reinterpret_cast<const float4*>(src + c);
          const float4 a1 = *reinterpret_cast<const float4*>(src + c + 4);
          uint4 pk;
          pk.x = pack_bf16x2(fmaf(gw, o_acc[c + 0], a0.x), fmaf(gw, o_acc[c + 1], a0.y));
          pk.y = pack_bf16x2(fmaf(gw, o_acc[c + 2], a0.z), fmaf(gw, o_acc[c + 3], a0.w));
          pk.z = pack_bf16x2(fmaf(gw, o_acc[c + 4], a1.x), fmaf(gw, o_acc[c + 5], a1.y));
          pk.w = pack_bf16x2(fmaf(gw, o_acc[c + 6], a1.z), fmaf(gw, o_acc[c + 7], a1.w));
          *reinterpret_cast<uint4*>(dst + c) = pk;
        }
      }
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
