// NSA backward (causal prefill): gradients of the forward with the selection
// held fixed.
//
// "Native Sparse Attention" lesson (aiengineeringfromscratch.com), section on
// native trainability: the top-n step is not differentiable and is a no-op on
// the computation graph (it only chooses which blocks are loaded); gradients
// flow through the compressed branch and through the selected blocks' and the
// window's contributions. "Разреженное внимание — NSA и DSA" (ai.flicky.cc),
// "Сколько это экономит": the NSA kernels come in forward and backward versions.
//
// Per query t, head h, branch b with key set K_b(t), probabilities P and output
// O_b, upstream dout:  dgate_b = <dout, O_b>;  dO_b = g_b dout;  dV_j += P_j dO_b;
// dP_j = <dO_b, V_j>;  dz_j = P_j (dP_j - <dO_b, O_b>);  dq += scale sum_j dz_j K_j;
// dK_j += scale dz_j q. The compressed keys/values pass their gradients back
// through the linear compression c_i = vec(x[i s : i s + l] + pe) . W.
//
// Kernels (warp-level mma.sync, 16 rows = one token's GQA heads, as in decode):
//   bwd_query  CTA = 8 tokens x one KV group, one warp per token; a producer warp
//              streams 32-key tiles (compressed keys, window keys, the union of
//              the 8 tokens' selected blocks) through a TMA ring twice: pass 1
//              recomputes every branch's output, log-sum-exp and <dout, O_b> and
//              writes dgates; pass 2 accumulates dq over all three branches.
//   bwd_keys   CTA = 64 keys x one KV group (4 warps x 16 keys), keys resident,
//              query tokens streamed through a TMA ring: raw keys take the window
//              tokens and the tokens whose selection holds the block (an inverted
//              index); compressed keys take every later token. The token
//              sequence of a block is split over grid.z; shares are added
//              atomically into dk, dv (raw) / dk_cmp, dv_cmp.
//   inv_*      the inverted selection index (counts, scan, fill).
//   cmp_bwd_*  the compression backward: column sums -> dpe; dx per residue of
//              the token index modulo the stride (no atomics) added into dk/dv;
//              dW as a split outer-product reduction.
// All waits are bounded (NSA_WAIT_LIMIT_NS); on a timeout a CTA stops issuing
// work, lets its copies land and leaves, and the status word records it.
#include "common.cuh"
#include "kernels.h"
#include "warp_mma.cuh"

namespace nsa {

namespace {

constexpr int kBqWarps = 8;                    // query-side consumer warps (one token each)
constexpr int kBqThreads = (kBqWarps + 1) * 32;
constexpr int kBqStages = 5;
constexpr int kBqKeys = 32;                    // keys per tile
constexpr int kBqNT = kBqKeys / 8;
constexpr int kBqQch = 128 * 128;              // one 64-column chunk of the 128-row Q / dout stage
constexpr int kBkWarps = 4;                    // key-side consumer warps (16 keys each)
constexpr int kBkThreads = (kBkWarps + 1) * 32;
constexpr int kBkStages = 8;
constexpr float kNoKeys = 1e30f;               // log-sum-exp of a row without keys (P = 0)

__device__ __forceinline__ int seq_of(const int32_t* prefix, int n, int x) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {   // last b with prefix[b] <= x
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}
__device__ __forceinline__ int cmp_vis(int t, int l, int s) { return t >= l - 1 ? (t - l + 1) / s + 1 : 0; }

template <int DK, int DV>
struct BqSmem {
  static constexpr int Q_BYTES = (DK / 64) * kBqQch;
  static constexpr int DO_BYTES = (DV / 64) * kBqQch;
  static constexpr int K_BYTES = kBqKeys * DK * 2;
  static constexpr int V_BYTES = kBqKeys * DV * 2;
  static constexpr int STAGE = K_BYTES + V_BYTES;
};

// dout . O over the lane's two rows (o normalised by 1/l), from the bf16 dout
// stage (rows warp*16 .., 128-byte swizzled 64-column chunks kBqQch apart)
template <int DV>
__device__ __forceinline__ void row_dot(const uint8_t* dos, int warp, const float (&o)[DV / 8][4], float il0,
                                        float il1, float& d0, float& d1, int lane) {
  const int r0 = lane >> 2, cq = (lane & 3) * 2;
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int i = 0; i < DV / 8; ++i) {
    const int c = i * 8 + cq;
    const uint8_t* base = dos + (c >> 6) * kBqQch;
    const __nv_bfloat162 x0 = *reinterpret_cast<const __nv_bfloat162*>(base + sw128(warp * 16 + r0, (c & 63) >> 3) + (c & 7) * 2);
    const __nv_bfloat162 x1 = *reinterpret_cast<const __nv_bfloat162*>(base + sw128(warp * 16 + r0 + 8, (c & 63) >> 3) + (c & 7) * 2);
    a0 += __bfloat162float(x0.x) * o[i][0] + __bfloat162float(x0.y) * o[i][1];
    a1 += __bfloat162float(x1.x) * o[i][2] + __bfloat162float(x1.y) * o[i][3];
  }
  d0 = quad_sum(a0) * il0;
  d1 = quad_sum(a1) * il1;
}

}  // namespace

// ---------------------------------------------------------------------------
// query side: dq, dgates, per-branch log-sum-exp and <dout, O_b>
// ---------------------------------------------------------------------------
template <int DK, int DV>
__global__ void __launch_bounds__(kBqThreads, 1) bwd_query_kernel(const BackwardArgs a,
                                                                   const __grid_constant__ BackwardMaps mp) {
  using S = BqSmem<DK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qs = smem;
  uint8_t* dos = qs + S::Q_BYTES;
  uint8_t* ring = dos + S::DO_BYTES;
  float* rowv = reinterpret_cast<float*>(ring + kBqStages * S::STAGE);   // [warp][branch][lse|dd][16]
  int* uni = reinterpret_cast<int*>(rowv + kBqWarps * 3 * 2 * 16);      // [256] union blocks
  uint32_t* umask = reinterpret_cast<uint32_t*>(uni + 256);             // [256] tokens that chose them
  uint64_t* full = reinterpret_cast<uint64_t*>(umask + 256);
  uint64_t* empty = full + kBqStages;
  int* misc = reinterpret_cast<int*>(empty + kBqStages);                // [0] abort, [1] union size
  volatile int* abort_flag = misc;
  uint32_t* bm = reinterpret_cast<uint32_t*>(misc + 4);                 // [nb] token bits per block

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, g = blockIdx.y;
  const int b = seq_of(a.seqs.tile_prefix, a.seqs.n, tile);
  const int L = a.seqs.len[b];
  const int64_t tok0 = a.seqs.tok_off[b];
  const int64_t cmp0 = a.seqs.cmp_off[b];
  const int t0 = (tile - a.seqs.tile_prefix[b]) * kBqWarps;
  const int t_last = min(t0 + kBqWarps - 1, L - 1);
  const int G = a.G;
  const int jt_max = t_last / a.ls;
  const int ncT = (cmp_vis(t_last, a.l, a.s) + kBqKeys - 1) / kBqKeys;
  const int key0w = max(0, t0 - a.window + 1);
  const int nwT = (t_last - key0w) / kBqKeys + 1;

  for (int i = tid; i <= jt_max; i += kBqThreads) bm[i] = 0u;
  if (tid == 0) {
    for (int i = 0; i < kBqStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kBqWarps);
    }
    misc[0] = 0;
    misc[1] = 0;
    fence_mbar_init();
  }
  // Q and dout of the 8 tokens (rows warp*16 + h, zero for h >= G or t >= L)
  for (int idx = tid; idx < 128 * (DK / 8); idx += kBqThreads) {
    const int row = idx / (DK / 8), c = idx % (DK / 8);
    const int tk = row >> 4, h = row & 15, t = t0 + tk;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (h < G && t < L)
      v = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) +
                                          ((size_t)(tok0 + t) * a.H_q + g * G + h) * DK + c * 8);
    *reinterpret_cast<uint4*>(qs + (c >> 3) * kBqQch + sw128(row, c & 7)) = v;
  }
  for (int idx = tid; idx < 128 * (DV / 8); idx += kBqThreads) {
    const int row = idx / (DV / 8), c = idx % (DV / 8);
    const int tk = row >> 4, h = row & 15, t = t0 + tk;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (h < G && t < L)
      v = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.dout) +
                                          ((size_t)(tok0 + t) * a.H_q + g * G + h) * DV + c * 8);
    *reinterpret_cast<uint4*>(dos + (c >> 3) * kBqQch + sw128(row, c & 7)) = v;
  }
  __syncthreads();
  // union of the tokens' selected blocks (bit tk of bm[j]: token t0 + tk chose block j)
  for (int idx = tid; idx < kBqWarps * a.top_n; idx += kBqThreads) {
    const int tk = idx / a.top_n, t = t0 + tk;
    if (t >= L) continue;
    const int j = a.sel[((size_t)(tok0 + t) * a.H_kv + g) * a.top_n + idx % a.top_n];
    if (j < 0) continue;
    if (j > t / a.ls) {   // not a block of this token (the selection is caller input): recorded, skipped
      atomicOr(a.status, DEV_ERR_BOUNDS);
      continue;
    }
    atomicOr(&bm[j], 1u << tk);
  }
  __syncthreads();
  if (warp == 0) {
    int cnt = 0;
    for (int j0 = 0; j0 <= jt_max; j0 += 32) {
      const int jb = j0 + lane;
      const uint32_t m = jb <= jt_max ? bm[jb] : 0u;
      const uint32_t bal = __ballot_sync(0xffffffffu, m != 0u);
      const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
      if (m != 0u && pos < 256) {
        uni[pos] = jb;
        umask[pos] = m;
      }
      cnt += __popc(bal);
    }
    if (lane == 0) misc[1] = cnt < 256 ? cnt : 256;
  }
  __syncthreads();
  const int nu = misc[1];
  const int per = ncT + nwT + 2 * nu;   // tiles of one pass
  const int n_tiles = 2 * per;

  if (warp == kBqWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int u = 0; u < n_tiles; ++u) {
        const int st = u % kBqStages;
        if (u >= kBqStages && !mbar_wait(&empty[st], ((u / kBqStages) - 1) & 1, abort_flag, a.status, 611)) break;
        const int r = u % per;
        const CUtensorMap *mk, *mv;
        int row;
        if (r < ncT) {
          mk = &mp.kc32; mv = &mp.vc32; row = (int)(cmp0 + r * kBqKeys);
        } else if (r < ncT + nwT) {
          mk = &mp.k32; mv = &mp.v32; row = (int)(tok0 + key0w + (r - ncT) * kBqKeys);
        } else {
          const int x = r - ncT - nwT;
          mk = &mp.k32; mv = &mp.v32; row = (int)(tok0 + (int64_t)uni[x >> 1] * a.ls + (x & 1) * kBqKeys);
        }
        uint8_t* Ks = ring + st * S::STAGE;
        mbar_arrive_expect_tx(&full[st], S::STAGE);
#pragma unroll
        for (int kb = 0; kb < DK / 64; ++kb) tma_load_3d(Ks + kb * (kBqKeys * 128), mk, &full[st], kb * 64, g, row);
#pragma unroll
        for (int vb = 0; vb < DV / 64; ++vb)
          tma_load_3d(Ks + S::K_BYTES + vb * (kBqKeys * 128), mv, &full[st], vb * 64, g, row);
        issued = u + 1;
      }
      if (*abort_flag)
        for (int v = issued - kBqStages < 0 ? 0 : issued - kBqStages; v < issued; ++v)
          mbar_wait_drain(&full[v % kBqStages], (v / kBqStages) & 1);
    }
    return;
  }

  // ------------------------------------------------------------ consumer warps
  const int t = t0 + warp;
  const bool valid = t < L;
  const int nvis = valid ? cmp_vis(t, a.l, a.s) : 0;
  const uint32_t qbase = smem_u32(qs), dobase = smem_u32(dos);
  const int r0 = lane >> 2;
  float* lse_w = rowv + warp * 96;          // [branch][16]
  float* dd_w = lse_w + 48;                 // [branch][16]
  bool ok = true;
  int u = 0;
  // key index of fragment element (nt, e) inside a tile and the row it belongs to
  auto key_of = [&](int nt, int e) { return nt * 8 + (lane & 3) * 2 + (e & 1); };
  // does the tile (branch br, index i inside the branch) hold a key of this token?
  auto needed = [&](int br, int i) -> bool {
    if (!valid) return false;
    if (br == 0) return i * kBqKeys < nvis;
    if (br == 1) return key0w + i * kBqKeys <= t && key0w + (i + 1) * kBqKeys - 1 > t - a.window;
    return ((umask[i >> 1] >> warp) & 1u) && uni[i >> 1] * a.ls + (i & 1) * kBqKeys <= t;
  };
  // scaled score (log2 units) or -inf where the key is not in the branch's set
  auto masked = [&](int br, int i, int nt, int e, float sraw) -> float {
    const int kk = key_of(nt, e);
    bool in;
    if (br == 0) in = i * kBqKeys + kk < nvis;
    else if (br == 1) { const int tau = key0w + i * kBqKeys + kk; in = tau <= t && tau > t - a.window; }
    else { const int tau = uni[i >> 1] * a.ls + (i & 1) * kBqKeys + kk; in = tau <= t; }
    return in ? sraw * a.scale_log2 : -INFINITY;
  };
  const int nb[3] = {ncT, nwT, 2 * nu};

  // ---- pass 1: per branch, output O_b (online softmax), lse, <dout, O_b>, dgates
#pragma unroll 1
  for (int br = 0; br < 3; ++br) {
    RowState<DV> rs;
    rs.init();
#pragma unroll 1
    for (int i = 0; i < nb[br]; ++i, ++u) {
      const int st = u % kBqStages;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&full[st], (u / kBqStages) & 1, abort_flag, a.status, 612));
      if (ok && needed(br, i)) {
        const uint32_t kb = smem_u32(ring + st * S::STAGE);
        float s[kBqNT][4];
        warp_qk_sq<DK, kBqNT>(qbase, kBqQch, warp * 16, kb, s, lane);
#pragma unroll
        for (int nt = 0; nt < kBqNT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) s[nt][e] = masked(br, i, nt, e, s[nt][e]);
        rs.update(s);
        warp_pv<DV, kBqNT>(s, kb + S::K_BYTES, rs.o, lane);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    rs.finish();
    const int gs = br == 0 ? 0 : (br == 1 ? 2 : 1);   // gate slot: tiles run (cmp, win, slc), gates are (cmp, slc, win)
    const float il0 = rs.l[0] > 0.f ? 1.f / rs.l[0] : 0.f, il1 = rs.l[1] > 0.f ? 1.f / rs.l[1] : 0.f;
    float d0, d1;
    row_dot<DV>(dos, warp, rs.o, il0, il1, d0, d1, lane);
    const float lse0 = rs.l[0] > 0.f ? rs.m[0] + __log2f(rs.l[0]) : kNoKeys;
    const float lse1 = rs.l[1] > 0.f ? rs.m[1] + __log2f(rs.l[1]) : kNoKeys;
    if ((lane & 3) == 0) {
      lse_w[br * 16 + r0] = lse0;
      lse_w[br * 16 + r0 + 8] = lse1;
      dd_w[br * 16 + r0] = d0;
      dd_w[br * 16 + r0 + 8] = d1;
      if (valid && ok) {
        const size_t base = ((size_t)(tok0 + t) * a.H_q + g * G) * 3 + gs;
        if (r0 < G) {
          a.dgates[base + (size_t)r0 * 3] = d0;
          a.lse[base + (size_t)r0 * 3] = lse0;
          a.dd[base + (size_t)r0 * 3] = d0;
        }
        if (r0 + 8 < G) {
          a.dgates[base + (size_t)(r0 + 8) * 3] = d1;
          a.lse[base + (size_t)(r0 + 8) * 3] = lse1;
          a.dd[base + (size_t)(r0 + 8) * 3] = d1;
        }
      }
    }
  }
  __syncwarp();

  // ---- pass 2: dq over all branches
  float dq[DK / 8][4];
#pragma unroll
  for (int i = 0; i < DK / 8; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
#pragma unroll 1
  for (int br = 0; br < 3; ++br) {
    const float l0 = lse_w[br * 16 + r0], l1 = lse_w[br * 16 + r0 + 8];
    const float dd0 = dd_w[br * 16 + r0], dd1 = dd_w[br * 16 + r0 + 8];
    float g0 = 0.f, g1 = 0.f;
    if (valid) {
      const float* gp = a.gates + ((size_t)(tok0 + t) * a.H_q + g * G) * 3 + (br == 0 ? 0 : (br == 1 ? 2 : 1));
      if (r0 < G) g0 = gp[(size_t)r0 * 3];
      if (r0 + 8 < G) g1 = gp[(size_t)(r0 + 8) * 3];
    }
#pragma unroll 1
    for (int i = 0; i < nb[br]; ++i, ++u) {
      const int st = u % kBqStages;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&full[st], (u / kBqStages) & 1, abort_flag, a.status, 613));
      if (ok && needed(br, i)) {
        const uint32_t kb = smem_u32(ring + st * S::STAGE);
        float s[kBqNT][4], dp[kBqNT][4];
        warp_qk_sq<DK, kBqNT>(qbase, kBqQch, warp * 16, kb, s, lane);
        warp_qk_sq<DV, kBqNT>(dobase, kBqQch, warp * 16, kb + S::K_BYTES, dp, lane);
#pragma unroll
        for (int nt = 0; nt < kBqNT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x = masked(br, i, nt, e, s[nt][e]);
            const bool lo = e < 2;
            const float p = ex2(x - (lo ? l0 : l1));
            s[nt][e] = p * (lo ? g0 : g1) * (dp[nt][e] - (lo ? dd0 : dd1));   // dz (unscaled)
          }
        warp_pv<DK, kBqNT>(s, kb, dq, lane);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
  }
  if (valid && ok) {
    const int cq = (lane & 3) * 2;
    float* dst = a.dq + ((size_t)(tok0 + t) * a.H_q + g * G) * DK;
#pragma unroll
    for (int i = 0; i < DK / 8; ++i) {
      if (r0 < G)
        *reinterpret_cast<float2*>(dst + (size_t)r0 * DK + i * 8 + cq) = make_float2(a.scale * dq[i][0], a.scale * dq[i][1]);
      if (r0 + 8 < G)
        *reinterpret_cast<float2*>(dst + (size_t)(r0 + 8) * DK + i * 8 + cq) =
            make_float2(a.scale * dq[i][2], a.scale * dq[i][3]);
    }
  }
}

// ---------------------------------------------------------------------------
// key side: dk, dv of 64 keys of one KV group (raw keys: window + selected
// branches; compressed keys: the compressed branch)
// ---------------------------------------------------------------------------
template <int DK, int DV>
struct BkSmem {
  static constexpr int KRES = 64 * DK * 2;
  static constexpr int VRES = 64 * DV * 2;
  static constexpr int QST = 16 * DK * 2;    // 16 rows x DK, 2 KB per 64-column chunk
  static constexpr int DST = 16 * DV * 2;
  static constexpr int STAGE = QST + DST;
  static constexpr int TOTAL = 1024 + KRES + VRES + kBkStages * STAGE + 512;
};

template <int DK, int DV, bool CMP>
__global__ void __launch_bounds__(kBkThreads, 1) bwd_keys_kernel(const BackwardArgs a,
                                                                  const __grid_constant__ BackwardMaps mp) {
  using S = BkSmem<DK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kres = smem;
  uint8_t* vres = kres + S::KRES;
  uint8_t* ring = vres + S::VRES;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + kBkStages * S::STAGE);
  uint64_t* empty = full + kBkStages;
  uint64_t* kvbar = empty + kBkStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(kvbar + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y;
  const int32_t* prefix = CMP ? a.cblk_prefix : a.blk_prefix;
  const int b = seq_of(prefix, a.seqs.n, blockIdx.x);
  const int j = blockIdx.x - prefix[b];
  const int L = a.seqs.len[b];
  const int64_t tok0 = a.seqs.tok_off[b];
  const int64_t cmp0 = a.seqs.cmp_off[b];
  const int key0 = j * 64;
  const int G = a.G;
  const int nc = cmp_vis(L - 1, a.l, a.s);   // compressed keys of the sequence
  // tokens: raw keys: the window range, then the block's inverted selection list;
  // compressed keys: this CTA's chunk of the tokens that see key0
  // the concatenated token sequence (window range, then the list) is split over
  // grid.z in chunks of tok_chunk, so a block that every token selects (block 0,
  // forced) spreads over many CTAs; the CTAs add their shares atomically
  int w_lo = 0, w_n = 0, s_n = 0;
  const int32_t* s_list = nullptr;
  if (CMP) {
    w_lo = key0 * a.s + a.l - 1;
    w_n = max(0, L - w_lo);
  } else {
    w_lo = key0;
    w_n = max(0, min(L - 1, key0 + 63 + a.window - 1) - key0 + 1);
    const int ent = (a.blk_prefix[b] + j) * a.H_kv + g;
    const int o0 = a.inv_off[ent];
    s_n = a.inv_off[ent + 1] - o0;
    s_list = a.inv_tok + o0;
  }
  const int c0 = blockIdx.z * a.tok_chunk;
  const int n_tok = max(0, min(w_n + s_n - c0, a.tok_chunk));
  if (n_tok == 0) return;   // nothing for this CTA (before any set-up)
  auto tok_of = [&](int i) -> int { return i + c0 < w_n ? w_lo + i + c0 : s_list[i + c0 - w_n]; };
  auto is_win = [&](int i) -> bool { return i + c0 < w_n; };

  if (tid == 0) {
    for (int i = 0; i < kBkStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kBkWarps);
    }
    mbar_init(kvbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // rows G..15 of every query stage stay zero (TMA writes the first G rows)
  for (int i = tid; i < kBkStages * S::STAGE / 16; i += kBkThreads)
    reinterpret_cast<uint4*>(ring)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  __syncthreads();

  if (warp == kBkWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const CUtensorMap* mk = CMP ? &mp.kc64 : &mp.k64;
      const CUtensorMap* mv = CMP ? &mp.vc64 : &mp.v64;
      const int krow = (int)(CMP ? cmp0 + key0 : tok0 + key0);
      mbar_arrive_expect_tx(kvbar, S::KRES + S::VRES);
#pragma unroll
      for (int kb = 0; kb < DK / 64; ++kb) tma_load_3d(kres + kb * 8192, mk, kvbar, kb * 64, g, krow);
#pragma unroll
      for (int vb = 0; vb < DV / 64; ++vb) tma_load_3d(vres + vb * 8192, mv, kvbar, vb * 64, g, krow);
      const uint32_t qbytes = (uint32_t)G * 128 * (DK / 64 + DV / 64);
      int issued = 0;
      for (int i = 0; i < n_tok; ++i) {
        const int st = i % kBkStages;
        if (i >= kBkStages && !mbar_wait(&empty[st], ((i / kBkStages) - 1) & 1, abort_flag, a.status, 621)) break;
        const int tt = tok_of(i);
        if (!NSA_BOUNDS(tt >= 0 && tt < L, a.status, 622)) {
          *abort_flag = 1;
          break;
        }
        uint8_t* Qs = ring + st * S::STAGE;
        mbar_arrive_expect_tx(&full[st], qbytes);
#pragma unroll
        for (int kb = 0; kb < DK / 64; ++kb) tma_load_3d(Qs + kb * 2048, &mp.qg, &full[st], kb * 64, g * G, (int)(tok0 + tt));
#pragma unroll
        for (int vb = 0; vb < DV / 64; ++vb)
          tma_load_3d(Qs + S::QST + vb * 2048, &mp.dog, &full[st], vb * 64, g * G, (int)(tok0 + tt));
        issued = i + 1;
      }
      if (*abort_flag) {
        mbar_wait_drain(kvbar, 0);
        for (int v = issued - kBkStages < 0 ? 0 : issued - kBkStages; v < issued; ++v)
          mbar_wait_drain(&full[v % kBkStages], (v / kBkStages) & 1);
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumer warps
  bool ok = __all_sync(0xffffffffu, mbar_wait(kvbar, 0, abort_flag, a.status, 623));
  const uint32_t kb_s = smem_u32(kres), vb_s = smem_u32(vres);
  float dk[DK / 8][4], dv[DV / 8][4];
#pragma unroll
  for (int i = 0; i < DK / 8; ++i) dk[i][0] = dk[i][1] = dk[i][2] = dk[i][3] = 0.f;
#pragma unroll
  for (int i = 0; i < DV / 8; ++i) dv[i][0] = dv[i][1] = dv[i][2] = dv[i][3] = 0.f;
  // fragment (nt, e) of a [16 keys x 16 rows] product: key row km, query row qr
  const int cq = (lane & 3) * 2;
  // per query row of this lane (rows cq, cq+1, cq+8, cq+9): the token's lse,
  // <dout, O_b> and gate, loaded one token ahead of their use
  float nlse[4], ndd[4], ngt[4];
  auto load_rows = [&](int i) {
    const int t = tok_of(i);
    const int br = CMP ? 0 : (is_win(i) ? 2 : 1);   // gate / lse slot: 0 cmp, 1 slc, 2 win
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int qr = cq + (x & 1) + 8 * (x >> 1);
      if (qr < G) {
        const size_t o = ((size_t)(tok0 + t) * a.H_q + g * G + qr) * 3 + br;
        nlse[x] = a.lse[o];
        ndd[x] = a.dd[o];
        ngt[x] = a.gates[o];
      } else {
        nlse[x] = kNoKeys;
        ndd[x] = 0.f;
        ngt[x] = 0.f;
      }
    }
  };
  load_rows(0);
#pragma unroll 1
  for (int i = 0; i < n_tok; ++i) {
    const int st = i % kBkStages;
    float lse[4], dd[4], gt[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      lse[x] = nlse[x];
      dd[x] = ndd[x];
      gt[x] = ngt[x];
    }
    if (i + 1 < n_tok) load_rows(i + 1);
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&full[st], (i / kBkStages) & 1, abort_flag, a.status, 624));
    if (ok) {
      const int t = tok_of(i);
      const int br = CMP ? 0 : (is_win(i) ? 2 : 1);
      const uint32_t qst = smem_u32(ring + st * S::STAGE), dst = qst + S::QST;
      float s[2][4], dp[2][4];
      warp_qk_sq<DK, 2>(kb_s, 8192, warp * 16, qst, s, lane);     // S^T = K Q^T
      warp_qk_sq<DV, 2>(vb_s, 8192, warp * 16, dst, dp, lane);    // dP^T = V dout^T
      const int nvis = CMP ? cmp_vis(t, a.l, a.s) : 0;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int km = warp * 16 + (lane >> 2) + 8 * (e >> 1);
          const int x = (e & 1) + 2 * nt;   // query row cq + (e&1) + 8nt
          const int key = key0 + km;
          bool in;
          if (CMP) in = key < nvis && key < nc;
          else in = key <= t && (br == 1 || t - key < a.window);
          const float p = in ? ex2(s[nt][e] * a.scale_log2 - lse[x]) : 0.f;
          const float gp = p * gt[x];
          s[nt][e] = gp;                          // g P^T
          dp[nt][e] = gp * (dp[nt][e] - dd[x]);   // dz^T (unscaled)
        }
      warp_pv<DV, 2>(s, dst, dv, lane);   // dV += (g P)^T dout
      warp_pv<DK, 2>(dp, qst, dk, lane);  // dK += dz^T Q
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }
  if (!ok) return;
  const int r0 = lane >> 2;
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int key = key0 + warp * 16 + r0 + 8 * hr;
    if (CMP ? key >= nc : key >= L) continue;
    float* dkp = (CMP ? a.dkc : a.dk) + ((size_t)((CMP ? cmp0 : tok0) + key) * a.H_kv + g) * DK;
    float* dvp = (CMP ? a.dvc : a.dv) + ((size_t)((CMP ? cmp0 : tok0) + key) * a.H_kv + g) * DV;
#pragma unroll
    for (int i = 0; i < DK / 8; ++i) {
      atomicAdd(dkp + i * 8 + cq, a.scale * dk[i][2 * hr]);
      atomicAdd(dkp + i * 8 + cq + 1, a.scale * dk[i][2 * hr + 1]);
    }
#pragma unroll
    for (int i = 0; i < DV / 8; ++i) {
      atomicAdd(dvp + i * 8 + cq, dv[i][2 * hr]);
      atomicAdd(dvp + i * 8 + cq + 1, dv[i][2 * hr + 1]);
    }
  }
}

// ---------------------------------------------------------------------------
// inverted selection index: for (sequence, block j, KV group g), the tokens
// whose selection holds j
// ---------------------------------------------------------------------------
__device__ __forceinline__ int seq_of_token(const SeqTable& t, int64_t n) {
  int lo = 0, hi = t.n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (t.tok_off[mid] <= n) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void inv_count_kernel(const BackwardArgs a, int64_t n_ent, int32_t* cnt, int32_t* slot) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_ent) return;
  const int64_t n = idx / ((int64_t)a.H_kv * a.top_n);
  const int g = (int)((idx / a.top_n) % a.H_kv);
  const int jj = a.sel[idx];
  slot[idx] = -1;
  if (jj < 0) return;
  const int b = seq_of_token(a.seqs, n);
  const int t = (int)(n - a.seqs.tok_off[b]);
  if (jj > t / a.ls || t >= a.seqs.len[b]) {   // not a block of this token: recorded, skipped
    atomicOr(a.status, DEV_ERR_BOUNDS);
    return;
  }
  const int ent = (a.blk_prefix[b] + jj) * a.H_kv + g;
  slot[idx] = ent;
  atomicAdd(cnt + ent, 1);
}

// exclusive scan of cnt[0..n) into off[0..n] by one CTA of 1024 threads
__global__ void inv_scan_kernel(const int32_t* cnt, int n, int32_t* off, int32_t* cur) {
  __shared__ int32_t part[1024];
  const int tid = threadIdx.x;
  const int per = (n + 1023) / 1024;
  const int lo = tid * per, hi = min(n, lo + per);
  int s = 0;
  for (int i = lo; i < hi; ++i) s += cnt[i];
  part[tid] = s;
  __syncthreads();
  for (int d = 1; d < 1024; d <<= 1) {   // inclusive Hillis-Steele scan of the parts
    const int v = tid >= d ? part[tid - d] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int run = part[tid] - s;
  for (int i = lo; i < hi; ++i) {
    off[i] = run;
    cur[i] = run;
    run += cnt[i];
  }
  if (tid == 1023) off[n] = part[1023];
}

__global__ void inv_fill_kernel(const BackwardArgs a, int64_t n_ent, const int32_t* slot, int32_t* cur,
                                int32_t* tok) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_ent) return;
  const int ent = slot[idx];
  if (ent < 0) return;
  const int64_t n = idx / ((int64_t)a.H_kv * a.top_n);
  const int b = seq_of_token(a.seqs, n);
  tok[atomicAdd(cur + ent, 1)] = (int)(n - a.seqs.tok_off[b]);
}

// ---------------------------------------------------------------------------
// compression backward (per K or V): c_i = sum_r (x[i s + r] + pe_r) W_r
// ---------------------------------------------------------------------------
// colsum[c] = sum over packed rows (compressed token, head) of dc[row][c]
__global__ void cmp_colsum_kernel(const float* dc, int64_t rows, int d_out, float* colsum) {
  const int c = threadIdx.x;
  if (c >= d_out) return;
  float s = 0.f;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) s += dc[r * d_out + c];
  atomicAdd(colsum + c, s);
}

// dpe[r][e] = sum_c colsum[c] W[r*d_in + e][c]
__global__ void cmp_dpe_kernel(const float* colsum, const float* W, int K, int d_out, float* dpe) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;   // r*d_in + e
  if (row >= K) return;
  float s = 0.f;
  for (int c = 0; c < d_out; ++c) s += colsum[c] * W[(size_t)row * d_out + c];
  dpe[row] = s;
}

// dx[16 i + rho] += dc_i W_rho^T + dc_{i-1} W_{rho+16}^T (for l = 2 s): the CTA
// owns residue rho, one head and 64 input columns, so every output row has one
// writer. W tiles (fp32, rows padded by one word) sit in shared memory.
struct CmpDxArgs {
  const float* dc;    // [Nc, H_kv, d_out]
  const float* W;     // [l * d_in, d_out]
  float* dx;          // [N, H_kv, d_in] (added to)
  int H_kv, d_in, d_out, l, s;
  int i_chunk;
  SeqTable seqs;      // tile_prefix: i-chunks per sequence
};
__global__ void __launch_bounds__(64) cmp_dx_kernel(const CmpDxArgs a) {
  extern __shared__ float sm[];
  const int rho = blockIdx.x;                          // 0 .. s-1
  const int h = blockIdx.y / (a.d_in / 64), e0 = (blockIdx.y % (a.d_in / 64)) * 64;
  const int b = seq_of(a.seqs.tile_prefix, a.seqs.n, blockIdx.z);
  const int L = a.seqs.len[b];
  const int nc = L >= a.l ? (L - a.l) / a.s + 1 : 0;
  const int i0 = (blockIdx.z - a.seqs.tile_prefix[b]) * a.i_chunk;
  const int ld = a.d_out + 1;
  float* w0 = sm;                    // W_rho rows e0 .. e0+63
  float* w1 = w0 + 64 * ld;          // W_{rho+s}
  float* dcs = w1 + 64 * ld;         // dc_i, dc_{i-1}
  const int e = threadIdx.x;
  for (int idx = threadIdx.x; idx < 64 * a.d_out; idx += 64) {
    const int r = idx / a.d_out, c = idx % a.d_out;
    w0[r * ld + c] = a.W[((size_t)rho * a.d_in + e0 + r) * a.d_out + c];
    w1[r * ld + c] = a.W[((size_t)(rho + a.s) * a.d_in + e0 + r) * a.d_out + c];
  }
  const int n_i = (L + a.s - 1) / a.s;   // token rows 16 i + rho cover the sequence
  for (int i = i0; i < min(n_i, i0 + a.i_chunk); ++i) {
    const int tau = i * a.s + rho;
    __syncthreads();
    for (int c = threadIdx.x; c < a.d_out; c += 64) {
      dcs[c] = i < nc ? a.dc[((size_t)(a.seqs.cmp_off[b] + i) * a.H_kv + h) * a.d_out + c] : 0.f;
      dcs[a.d_out + c] = (i >= 1 && i - 1 < nc) ? a.dc[((size_t)(a.seqs.cmp_off[b] + i - 1) * a.H_kv + h) * a.d_out + c] : 0.f;
    }
    __syncthreads();
    if (tau >= L) continue;
    float acc = 0.f;
    for (int c = 0; c < a.d_out; ++c) acc += dcs[c] * w0[e * ld + c] + dcs[a.d_out + c] * w1[e * ld + c];
    a.dx[((size_t)(a.seqs.tok_off[b] + tau) * a.H_kv + h) * a.d_in + e0 + e] += acc;
  }
}

// dW[r*d_in + e][c] += sum over packed compressed rows (i, h) of x[i s + r][h][e] dc[i][h][c];
// CTA: one r, 32 e x 64 c, a chunk of the packed rows; results added atomically
struct CmpDwArgs {
  const float* dc;          // [Nc, H_kv, d_out]
  const void* x;            // bf16 [N, H_kv, d_in]
  float* dW;                // [l * d_in, d_out]
  int H_kv, d_in, d_out, l, s;
  int64_t rows;             // Nc * H_kv
  int row_chunk;
  SeqTable seqs;
  int32_t ncmp_prefix[kMaxBatch + 1];   // packed compressed rows per sequence (prefix, in tokens i)
};
__global__ void __launch_bounds__(256) cmp_dw_kernel(const CmpDwArgs a) {
  __shared__ float xs[16][32];
  __shared__ float cs[16][64];
  const int r = blockIdx.x / (a.d_in / 32), e0 = (blockIdx.x % (a.d_in / 32)) * 32;
  const int c0 = blockIdx.y * 64;
  const int64_t q0 = (int64_t)blockIdx.z * a.row_chunk;
  const int64_t q1 = min(a.rows, q0 + a.row_chunk);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;   // 16 x 16: 2 e x 4 c each
  float acc[2][4] = {};
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(a.x);
  for (int64_t q = q0; q < q1; q += 16) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < 16 * 32; idx += 256) {
      const int k = idx / 32, e = idx % 32;
      const int64_t row = q + k;
      float v = 0.f;
      if (row < q1) {
        const int ig = (int)(row / a.H_kv), h = (int)(row % a.H_kv);
        const int b = seq_of(a.ncmp_prefix, a.seqs.n, ig);
        const int i = ig - a.ncmp_prefix[b];
        v = __bfloat162float(x[((size_t)(a.seqs.tok_off[b] + (int64_t)i * a.s + r) * a.H_kv + h) * a.d_in + e0 + e]);
      }
      xs[k][e] = v;
    }
    for (int idx = threadIdx.x; idx < 16 * 64; idx += 256) {
      const int k = idx / 64, c = idx % 64;
      const int64_t row = q + k;
      cs[k][c] = (row < q1 && c0 + c < a.d_out) ? a.dc[row * a.d_out + c0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k)
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] += xs[k][ty * 2 + u] * cs[k][tx * 4 + v];
  }
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int c = c0 + tx * 4 + v;
      if (c < a.d_out) atomicAdd(a.dW + ((size_t)r * a.d_in + e0 + ty * 2 + u) * a.d_out + c, acc[u][v]);
    }
}

// dW[r*d_in + e][c] += pe[r][e] * colsum[c]
__global__ void cmp_dw_pe_kernel(const float* pe, const float* colsum, int K, int d_out, float* dW) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)K * d_out) return;
  dW[idx] += pe[idx / d_out] * colsum[idx % d_out];
}

// ---------------------------------------------------------------------------
// launches
// ---------------------------------------------------------------------------
size_t backward_query_smem(int d_k, int d_v, int nb) {
  const size_t fixed = (size_t)(d_k / 64) * kBqQch + (size_t)(d_v / 64) * kBqQch +
                       (size_t)kBqStages * kBqKeys * (d_k + d_v) * 2 + kBqWarps * 3 * 16 * 2 * 4 + 256 * 8 +
                       512;
  return 1024 + fixed + (size_t)(nb + 1) * 4;
}

template <int DK, int DV>
static cudaError_t launch_bwd_t(const BackwardArgs& a, const BackwardMaps& m, int q_tiles, int raw_blocks,
                                int raw_z, int cmp_tiles, int cmp_z, cudaStream_t st) {
  cudaError_t e;
  const size_t sq = backward_query_smem(DK, DV, a.nb_stride);
  auto kq = bwd_query_kernel<DK, DV>;
  if ((e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sq)) != cudaSuccess) return e;
  if (q_tiles > 0) kq<<<dim3(q_tiles, a.H_kv), kBqThreads, sq, st>>>(a, m);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  using SK = BkSmem<DK, DV>;
  auto kr = bwd_keys_kernel<DK, DV, false>;
  auto kc = bwd_keys_kernel<DK, DV, true>;
  if ((e = cudaFuncSetAttribute(kr, cudaFuncAttributeMaxDynamicSharedMemorySize, SK::TOTAL)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, SK::TOTAL)) != cudaSuccess) return e;
  if (raw_blocks > 0) kr<<<dim3(raw_blocks, a.H_kv, raw_z), kBkThreads, SK::TOTAL, st>>>(a, m);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (cmp_tiles > 0) kc<<<dim3(cmp_tiles, a.H_kv, cmp_z), kBkThreads, SK::TOTAL, st>>>(a, m);
  return cudaGetLastError();
}

cudaError_t launch_backward_attn(const BackwardArgs& a, const BackwardMaps& m, int q_tiles, int raw_blocks,
                                 int raw_z, int cmp_tiles, int cmp_z, cudaStream_t st) {
  if (a.d_k == 192 && a.d_v == 128) return launch_bwd_t<192, 128>(a, m, q_tiles, raw_blocks, raw_z, cmp_tiles, cmp_z, st);
  if (a.d_k == 64 && a.d_v == 64) return launch_bwd_t<64, 64>(a, m, q_tiles, raw_blocks, raw_z, cmp_tiles, cmp_z, st);
  if (a.d_k == 128 && a.d_v == 128) return launch_bwd_t<128, 128>(a, m, q_tiles, raw_blocks, raw_z, cmp_tiles, cmp_z, st);
  if (a.d_k == 192 && a.d_v == 64) return launch_bwd_t<192, 64>(a, m, q_tiles, raw_blocks, raw_z, cmp_tiles, cmp_z, st);
  if (a.d_k == 64 && a.d_v == 128) return launch_bwd_t<64, 128>(a, m, q_tiles, raw_blocks, raw_z, cmp_tiles, cmp_z, st);
  if (a.d_k == 128 && a.d_v == 64) return launch_bwd_t<128, 64>(a, m, q_tiles, raw_blocks, raw_z, cmp_tiles, cmp_z, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_inverted_index(const BackwardArgs& a, int64_t n_ent, int n_lists, int32_t* cnt, int32_t* off,
                                  int32_t* cur, int32_t* slot, int32_t* tok, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(cnt, 0, (size_t)n_lists * 4, st);
  if (e != cudaSuccess) return e;
  if (n_ent > 0) inv_count_kernel<<<(unsigned)((n_ent + 255) / 256), 256, 0, st>>>(a, n_ent, cnt, slot);
  inv_scan_kernel<<<1, 1024, 0, st>>>(cnt, n_lists, off, cur);
  if (n_ent > 0) inv_fill_kernel<<<(unsigned)((n_ent + 255) / 256), 256, 0, st>>>(a, n_ent, slot, cur, tok);
  return cudaGetLastError();
}

cudaError_t launch_compress_backward(const float* dc, const void* x, const float* W, const float* pe, int d_in,
                                     int d_out, int H_kv, int l, int s, const SeqTable& seqs,
                                     const int32_t* ncmp_prefix, int64_t n_cmp_total, float* dx, float* dW,
                                     float* dpe, float* colsum, cudaStream_t st) {
  const int K = l * d_in;
  const int64_t rows = n_cmp_total * H_kv;
  cudaError_t e = cudaMemsetAsync(colsum, 0, (size_t)d_out * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dW, 0, (size_t)K * d_out * 4, st);
  if (e != cudaSuccess) return e;
  if (rows > 0) cmp_colsum_kernel<<<(unsigned)(rows < 1184 ? rows : 1184), 256, 0, st>>>(dc, rows, d_out, colsum);
  cmp_dpe_kernel<<<(K + 127) / 128, 128, 0, st>>>(colsum, W, K, d_out, dpe);
  if (rows > 0) {
    // dx, one residue of the token index per CTA row of the grid
    CmpDxArgs dxa{};
    dxa.dc = dc; dxa.W = W; dxa.dx = dx; dxa.H_kv = H_kv; dxa.d_in = d_in; dxa.d_out = d_out; dxa.l = l; dxa.s = s;
    dxa.i_chunk = 64;
    dxa.seqs = seqs;
    int z = 0;
    for (int b = 0; b < seqs.n; ++b) {
      dxa.seqs.tile_prefix[b] = z;
      z += (((seqs.len[b] + s - 1) / s) + dxa.i_chunk - 1) / dxa.i_chunk;
    }
    dxa.seqs.tile_prefix[seqs.n] = z;
    const size_t smem = ((size_t)2 * 64 * (d_out + 1) + 2 * d_out) * 4;
    if ((e = cudaFuncSetAttribute(cmp_dx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
      return e;
    if (z > 0) cmp_dx_kernel<<<dim3(s, H_kv * (d_in / 64), z), 64, smem, st>>>(dxa);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    CmpDwArgs dwa{};
    dwa.dc = dc; dwa.x = x; dwa.dW = dW; dwa.H_kv = H_kv; dwa.d_in = d_in; dwa.d_out = d_out; dwa.l = l; dwa.s = s;
    dwa.rows = rows;
    dwa.row_chunk = 1024;
    dwa.seqs = seqs;
    for (int b = 0; b <= seqs.n; ++b) dwa.ncmp_prefix[b] = ncmp_prefix[b];
    const int zc = (int)((rows + dwa.row_chunk - 1) / dwa.row_chunk);
    cmp_dw_kernel<<<dim3(l * (d_in / 32), (d_out + 63) / 64, zc), 256, 0, st>>>(dwa);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const int64_t n = (int64_t)K * d_out;
  cmp_dw_pe_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(pe, colsum, K, d_out, dW);
  return cudaGetLastError();
}

}  // namespace nsa
