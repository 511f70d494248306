// Fused NSA prefill attention on tcgen05: compressed branch + block importance,
// top-n block selection, sliding window and selected blocks, gated combine.
//
// Method ("Разреженное внимание — NSA и DSA", ai.flicky.cc, section "NSA: три
// ветви"; "Native Sparse Attention" lesson, aiengineeringfromscratch.com, steps
// 1-5): each query head attends, in three separate softmaxes, to the compressed
// block summaries it can see, to the raw tokens of the top-n selection blocks its
// GQA group chose from the compressed attention weights, and to the last w raw
// tokens; the three outputs are mixed by per-head sigmoid gates.
//
// One CTA owns one query tile of M = 128 rows = (128/G tokens) x (G heads of one
// KV group) and runs every branch for it, so K/V tiles staged in shared memory
// serve all heads of the group and the only global output is bf16 `out` (plus
// the optional importance / selection rows):
//
//   C1  compressed keys, pass 1: row max and softmax denominator
//   C2  compressed keys, pass 2: normalised probabilities p; importance of every
//       selection block (p spread by token overlap, summed over the group's
//       heads); O_A = P.V_cmp
//   --  top-n per token (forced first / local blocks, ties to the lower index),
//       union of the tile's selections
//   W   window keys, online softmax into O_B; O_A = g_cmp O_A + g_win / l * O_B
//   S   union blocks, each row masked to its own token's selection (and to
//       keys <= t inside the current block); online softmax into O_B;
//       out = bf16(O_A + g_slc / l * O_B)
//
// Every tile is 64 keys. Q sits in shared memory (A operand of S = Q.K^T); S has
// four buffers in tensor memory and the softmax writes its bf16 P over the S
// columns it has read (A operand of O += P.V). K and V stream through TMA rings.
// Roles (384 threads): warps 0-7 softmax: warp w owns 16 rows, tensor-memory
// lanes 32 (w % 4) + 16 (w / 4) .. + 15, and all 64 keys of every tile; its two
// half-warps hold keys 0-31 and 32-63 of the same rows and trade row maxima and
// sums by shuffles. With G = 16 a warp's rows are one token, so a selected block
// that token did not pick costs the warp nothing. Warp 8 loads Q and the K tiles, warp 11 the V
// tiles (separate rings: a K tile is released as soon as its S is computed);
// warp 9 issues the S = Q.K^T products (tiles in pairs, up to four tiles ahead
// of the softmax); warp 10 the O += P.V products. Every wait is time-bounded; on
// a timeout the CTA stops issuing work, lets its own copies and products land
// and leaves.
#include "common.cuh"
#include "kernels.h"
#include "topn.cuh"

namespace nsa {

namespace {

constexpr int kKeys = 64;
constexpr int kThreads = 384;   // 8 softmax warps, K producer, S issuer, P.V issuer, V producer
constexpr int kSmThreads = 256;
constexpr float kRescaleLog2 = 8.f;   // O is rescaled only when a row max grows by more (log2 units)
constexpr int kMaxStages = 8;

// tensor-memory columns (512 allocated)
constexpr int kSBuf = 4;          // S/P buffers of 64 columns: tile j uses buffer j % 4
constexpr uint32_t kColS = 0;
constexpr uint32_t kColOA = 256;  // finished branches
constexpr uint32_t kColOB = 384;  // branch in progress
__device__ __forceinline__ uint32_t col_s(int b) { return kColS + 64u * (uint32_t)b; }

struct FBars {
  uint64_t k_full[kMaxStages], k_empty[kMaxStages];   // K ring: released once S = Q.K^T is computed
  uint64_t v_full[kMaxStages], v_empty[kMaxStages];   // V ring: released once O += P.V is computed
  uint64_t q_full, s_full[kSBuf], s_free[kSBuf], p_full[kSBuf], pv_done[kSBuf], ob_free, sel_ready, drain, smx;
  uint32_t tmem_base;
  int abort;
  int nu;
  int ucnt[8];   // blocks per softmax warp's range of the union
};

__device__ __forceinline__ int seq_of_tile(const SeqTable& t, int tile) {
  int lo = 0, hi = t.n - 1;
  while (lo < hi) {   // last b with tile_prefix[b] <= tile
    const int mid = (lo + hi + 1) >> 1;
    if (t.tile_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int cmp_visible_dev(int t, int l, int s) { return t >= l - 1 ? (t - l + 1) / s + 1 : 0; }

// max / sum of N values: 8 interleaved chains, then a tree over the 8 partials
// (dependency depth N/8 + 3 with only 8 temporaries live next to the values)
template <int N>
__device__ __forceinline__ float tree_max(const float* v) {
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = v[i];
#pragma unroll
  for (int i = 8; i < N; ++i) a[i & 7] = fmaxf(a[i & 7], v[i]);
#pragma unroll
  for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) a[i] = fmaxf(a[i], a[i + w]);
  return a[0];
}
template <int N>
__device__ __forceinline__ float tree_sum(const float* v) {
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = v[i];
#pragma unroll
  for (int i = 8; i < N; ++i) a[i & 7] += v[i];
#pragma unroll
  for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) a[i] += a[i + w];
  return a[0];
}

// one warp scales 2 * HALF tensor-memory columns of its 16 rows starting at
// `col`: each half-warp scales HALF columns (the upper one from col + HALF)
template <int HALF>
__device__ __noinline__ void tmem_scale_cols(uint32_t col, float alpha) {
  for (int c = 0; c < HALF; c += 16) {
    float ov[16];
    tmem_ld16_h<HALF>(col + c, ov);
    tmem_ld_wait();
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = __float_as_uint(ov[i] * alpha);
    tmem_st8_h<HALF>(col + c, w);
    tmem_st8_h<HALF>(col + c + 8, w + 8);
  }
  tmem_st_wait();
}

// head sum over the G consecutive lanes of one token
template <int G>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int off = G >> 1; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// Sums each of the 8 values v[0..7] over the G lanes of a token by recursive
// halving: at every step a lane keeps half of its values and trades the other
// half with its partner, so 8 sums over 16 lanes take 8 shuffles instead of 32.
// On return the lane holds the sums of blocks base .. base + max(1, 8/G) - 1 in
// v[0..]; the return value is base.
template <int G>
__device__ __forceinline__ int group_reduce8(float* v, int lane) {
  int base = 0;
  int n = 8;
#pragma unroll
  for (int off = G >> 1; off >= 1; off >>= 1) {
    if (n > 1) {
      const bool up = (lane & off) != 0;
      const int h = n >> 1;
#pragma unroll
      for (int k = 0; k < h; ++k) {
        const float send = up ? v[k] : v[k + h];
        const float keep = up ? v[k + h] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
      }
      if (up) base += h;
      n = h;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    }
  }
  return base;
}

// Importance of the 8 selection blocks B0 .. B0+7 covered by 32 compressed keys
// (probabilities h[0..31] of one row), summed over the G heads of the token and
// written to imp_row by one lane per block; `cin` is the mass carried into block
// B0 from the previous 32 keys. Returns the mass carried past block B0 + 7.
template <int G>
__device__ __forceinline__ float importance32(const float* h, float cin, int lane, bool write, float* imp_row,
                                              int B0, int jt) {
  float v[8];
#pragma unroll
  for (int qb = 0; qb < 8; ++qb) v[qb] = 2.f * (h[4 * qb] + h[4 * qb + 1] + h[4 * qb + 2]) + h[4 * qb + 3];
#pragma unroll
  for (int qb = 0; qb < 7; ++qb) v[qb + 1] += h[4 * qb + 3];
  const float carry = group_sum<G>(h[31]);
  const int base = group_reduce8<G>(v, lane);
  constexpr int kHeld = G >= 8 ? 1 : 8 / G;
  constexpr int kDup = G > 8 ? G / 8 - 1 : 0;   // lanes holding copies of the same sums
  if (write && (lane & kDup) == 0) {
#pragma unroll
    for (int k = 0; k < kHeld; ++k) {
      const int qb = base + k;
      if (B0 + qb <= jt) imp_row[B0 + qb] = v[k] + (qb == 0 ? cin : 0.f);
    }
  }
  return carry;
}

}  // namespace

// Optional in-kernel timeline (compiled only with -DNSA_PREFILL_TRACE): lane 0
// of every warp of four CTAs (KV head 0, the last query tile of each quarter of the grid)
// records clock64() at fixed points of each tile's life; nsa_prefill_trace_read
// copies the records out. Off in the library build.
#ifdef NSA_PREFILL_TRACE
constexpr int kTrTiles = 320;
__device__ unsigned long long g_trace[4][12][kTrTiles][4];
__device__ unsigned long long g_trace_phase[4][12][8];
#define TR(j, k)                                                                            \
  do {                                                                                      \
    if (tr_cta >= 0 && (threadIdx.x & 31) == 0 && (j) >= 0 && (j) < kTrTiles)                \
      g_trace[tr_cta][threadIdx.x >> 5][(j)][(k)] = clock64();                              \
  } while (0)
#define TRP(k)                                                                              \
  do {                                                                                      \
    if (tr_cta >= 0 && (threadIdx.x & 31) == 0) g_trace_phase[tr_cta][threadIdx.x >> 5][(k)] = clock64(); \
  } while (0)
#else
#define TR(j, k) do {} while (0)
#define TRP(k) do {} while (0)
#endif


// dynamic shared memory: Q [d_k/64][128 rows][128 B] | K ring | V ring | bars | block masks [nb][MW] | union [nb] | importance carries [nb/8 + 2][128/G] f32 |
// (when it fits) importance [128/G][nb] f32 | selections [128/G][32] i32
__host__ __device__ inline size_t fused_fixed_bytes(int nb, int G) {
  const int tok = 128 / G, mw = (tok + 31) / 32;
  return sizeof(FBars) + (size_t)nb * mw * 4 + (size_t)nb * 4 +
         (size_t)(nb / 8 + 2) * tok * 4 + 64;
}

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1) nsa_prefill_kernel(const PrefillArgs a,
                                                                   const __grid_constant__ PrefillMaps mp) {
  constexpr int K_BYTES = kKeys * DK * 2;
  constexpr int V_BYTES = kKeys * DV * 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nks = a.n_stages, nvs = a.n_vstages;
  uint8_t* Qs = smem;                        // Q tile, 128-byte swizzled chunks of 64 columns
  uint8_t* kring = smem + 128 * DK * 2;
  uint8_t* vring = kring + (size_t)nks * K_BYTES;
  FBars* bars = reinterpret_cast<FBars*>(vring + (size_t)nvs * V_BYTES);
  const int G = a.G;
  const int TOK = 128 / G, MW = (TOK + 31) / 32;
  uint32_t* bm = reinterpret_cast<uint32_t*>(bars + 1);            // [nb][MW] token bits per block
  int* uni = reinterpret_cast<int*>(bm + (size_t)a.nb_stride * MW);  // union of selected blocks
  float* cbuf = reinterpret_cast<float*>(uni + a.nb_stride);      // [32-key half][token] carried mass
  float* imp_s = cbuf + (size_t)(a.nb_stride / 8 + 2) * TOK;      // [token][nb] when a.imp_smem
  int32_t* sel_s = reinterpret_cast<int32_t*>(imp_s + (size_t)TOK * a.nb_stride);   // [token][32]
  volatile int* abort_flag = &bars->abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, g = blockIdx.y;
  const int b = seq_of_tile(a.seqs, tile);
  const int L = a.seqs.len[b];
  const int64_t tok0 = a.seqs.tok_off[b];
  const int64_t cmp0 = a.seqs.cmp_off[b];
  const int t0 = (tile - a.seqs.tile_prefix[b]) * TOK;
  const int t_last = min(t0 + TOK - 1, L - 1);
  const int jt_max = t_last / a.ls;
  const int nkc = (cmp_visible_dev(t_last, a.l, a.s) + kKeys - 1) / kKeys;   // compressed tiles per pass
  const int key0w = max(0, t0 - a.window + 1);
  const int nkw = (t_last - key0w) / kKeys + 1;                              // window tiles
  const int first_w = 2 * nkc, first_s = first_w + nkw;
#ifdef NSA_PREFILL_TRACE
  const int tr_q = (int)gridDim.x / 4;
  const int tr_cta = (g == 0 && tr_q > 0 && (tile + 1) % tr_q == 0) ? (tile + 1) / tr_q - 1 : -1;
#endif
  TRP(0);

  for (int i = tid; i < (jt_max + 1) * MW; i += kThreads) bm[i] = 0u;
  if (tid == 0) {
    for (int i = 0; i < nks; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
    }
    for (int i = 0; i < nvs; ++i) {
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
    }
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < kSBuf; ++i) {   // every softmax thread reads (and writes P into) every tile
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], kSmThreads);
      mbar_init(&bars->p_full[i], kSmThreads);
      mbar_init(&bars->pv_done[i], 1);
    }
    mbar_init(&bars->ob_free, kSmThreads);
    mbar_init(&bars->sel_ready, 1);
    mbar_init(&bars->drain, 2);   // one commit per MMA issuer
    mbar_init(&bars->smx, kSmThreads);
    bars->abort = 0;
    bars->nu = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&bars->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------ Q and K producer
    if (lane == 0) {
      prefetch_tmap(&mp.k);
      mbar_arrive_expect_tx(&bars->q_full, (uint32_t)(128 * DK * 2));
#pragma unroll
      for (int kb = 0; kb < DK / 64; ++kb)
        tma_load_3d(Qs + kb * 16384, &mp.q, &bars->q_full, kb * 64, g * G, (int)(tok0 + t0));
      int issued = 0;
      bool ok = true;
      auto load = [&](int j, const CUtensorMap* mk, int row) -> bool {
        const int st = j % nks;
        if (j >= nks && !mbar_wait(&bars->k_empty[st], ((j / nks) - 1) & 1, abort_flag, a.status, 401))
          return false;
        if (j == 0 && NSA_INJECT(a, FAULT_PREFILL_K_TILE)) {   // checking build: withhold the first tile
          issued = 1;
          return true;
        }
        TR(j, 0);
        uint8_t* Ks = kring + (size_t)st * 8192;   // chunk kb of slot st at kb * nks * 8 KB + st * 8 KB
        mbar_arrive_expect_tx(&bars->k_full[st], K_BYTES);
#pragma unroll
        for (int kb = 0; kb < DK / 64; ++kb)
          tma_load_3d(Ks + (size_t)kb * nks * 8192, mk, &bars->k_full[st], kb * 64, g, row);
        issued = j + 1;
        return true;
      };
      int j = 0;
      for (int pass = 0; pass < 2; ++pass)
        for (int i = 0; i < nkc && ok; ++i) ok = load(j++, &mp.kc, (int)(cmp0 + i * kKeys));
      for (int i = 0; i < nkw && ok; ++i) ok = load(j++, &mp.k, (int)(tok0 + key0w + i * kKeys));
      if (ok) ok = mbar_wait(&bars->sel_ready, 0, abort_flag, a.status, 402);
      const int nu = ok ? bars->nu : 0;
      for (int u = 0; u < nu && ok; ++u) {
        if (!NSA_BOUNDS(uni[u] >= 0 && uni[u] <= jt_max, a.status, 501)) {
          *abort_flag = 1;   // stop the other roles; the copies issued so far are drained below
          ok = false;
          break;
        }
        ok = load(j++, &mp.k, (int)(tok0 + (int64_t)uni[u] * a.ls));
      }
      if (!ok) {   // let the copies still in flight land before the CTA exits
        mbar_wait_drain(&bars->q_full, 0);
        for (int v = issued - nks < 0 ? 0 : issued - nks; v < issued; ++v)
          mbar_wait_drain(&bars->k_full[v % nks], (v / nks) & 1);
      }
    }
  } else if (warp == 11) {
    // ------------------------------------------------------------ V producer (tiles with P.V only)
    if (lane == 0) {
      prefetch_tmap(&mp.v);
      int issued = 0;
      bool ok = true;
      auto load = [&](int vi, const CUtensorMap* mv, int row) -> bool {
        const int st = vi % nvs;
        if (vi >= nvs && !mbar_wait(&bars->v_empty[st], ((vi / nvs) - 1) & 1, abort_flag, a.status, 403))
          return false;
        TR(vi, 0);
        uint8_t* Vs = vring + (size_t)st * V_BYTES;
        mbar_arrive_expect_tx(&bars->v_full[st], V_BYTES);
#pragma unroll
        for (int vb = 0; vb < DV / 64; ++vb) tma_load_3d(Vs + vb * 8192, mv, &bars->v_full[st], vb * 64, g, row);
        issued = vi + 1;
        return true;
      };
      int vi = 0;
      for (int i = 0; i < nkc && ok; ++i) ok = load(vi++, &mp.vc, (int)(cmp0 + i * kKeys));
      for (int i = 0; i < nkw && ok; ++i) ok = load(vi++, &mp.v, (int)(tok0 + key0w + i * kKeys));
      if (ok) ok = mbar_wait(&bars->sel_ready, 0, abort_flag, a.status, 404);
      const int nu = ok ? bars->nu : 0;
      for (int u = 0; u < nu && ok; ++u) {
        if (!NSA_BOUNDS(uni[u] >= 0 && uni[u] <= jt_max, a.status, 502)) {
          *abort_flag = 1;   // stop the other roles; the copies issued so far are drained below
          ok = false;
          break;
        }
        ok = load(vi++, &mp.v, (int)(tok0 + (int64_t)uni[u] * a.ls));
      }
      if (!ok)
        for (int v = issued - nvs < 0 ? 0 : issued - nvs; v < issued; ++v)
          mbar_wait_drain(&bars->v_full[v % nvs], (v / nvs) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ S = Q.K^T issuer
    // S(j) goes to buffer j % 4; the buffer is free again once the softmax read
    // S(j - 4) (C1 tiles) or P.V(j - 4) consumed the P written over it. Tiles are
    // taken in pairs (j even): their S buffers are adjacent columns and their K
    // tiles adjacent rows of the ring (chunk-interleaved slots), so one N = 128
    // product computes both.
    if (lane == 0) {
      const uint32_t idesc_64 = umma_idesc_bf16(128, kKeys, false, false);
      const uint32_t idesc_128 = umma_idesc_bf16(128, 2 * kKeys, false, false);
      const uint64_t kdesc0 = umma_desc_sw128(smem_u32(kring), 16, 1024);
      const uint64_t qdesc0 = umma_desc_sw128(smem_u32(Qs), 16, 1024);
      uint64_t qd[DK / 16];   // Q operand descriptors, fixed for the CTA
      uint32_t koff[DK / 16]; // K operand offsets (16-byte units) inside a slot
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk) {
        qd[kk] = qdesc0 + (uint64_t)((((kk >> 2) * 16384) + (kk & 3) * 32) >> 4);
        koff[kk] = (uint32_t)(kk >> 2) * (uint32_t)nks * (8192u >> 4) + (uint32_t)((kk & 3) * 32 >> 4);
      }
      auto buf_free = [&](int jj) -> bool {
        if (jj < kSBuf) return true;
        // s_* barriers complete once per tile, p_full / pv_done once per P.V tile (index >= nkc)
        const int jp = jj - kSBuf, sb = jj & (kSBuf - 1);
        return (jp >= nkc) ? mbar_wait(&bars->pv_done[sb], ((jp - nkc) >> 2) & 1, abort_flag, a.status, 416)
                           : mbar_wait(&bars->s_free[sb], (jp >> 2) & 1, abort_flag, a.status, 418);
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, a.status, 411);
      int total = first_s;
      bool known = false;
      int st = 0;
      uint32_t kph = 0;   // K ring slot of tile j and its phase parity
      for (int j = 0; ok;) {
        if (!known && j + 1 >= first_s) {
          ok = mbar_wait(&bars->sel_ready, 0, abort_flag, a.status, 414);
          if (!ok) break;
          total = first_s + bars->nu;
          known = true;
        }
        if (j >= total) break;
        const bool pair = j + 1 < total;   // j and st are even whenever a pair starts
        const int sb = j & (kSBuf - 1);
        ok = mbar_wait(&bars->k_full[st], kph, abort_flag, a.status, 415) &&
             (!pair || mbar_wait(&bars->k_full[st + 1], kph, abort_flag, a.status, 415)) && buf_free(j) &&
             (!pair || buf_free(j + 1));
        if (!ok) break;
        TR(j, 0);
        tc_fence_after();
        const uint64_t kd = kdesc0 + (uint64_t)((uint32_t)st * (8192u >> 4));
        const uint32_t dcol = tmem + col_s(sb);
        if (pair) {
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk) umma_ss(dcol, qd[kk], kd + koff[kk], idesc_128, kk > 0 ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk) umma_ss(dcol, qd[kk], kd + koff[kk], idesc_64, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full[sb]);
        umma_commit(&bars->k_empty[st]);
        if (pair) {
          umma_commit(&bars->s_full[sb + 1]);
          umma_commit(&bars->k_empty[st + 1]);
        }
        TR(j, 1);
        const int adv = pair ? 2 : 1;
        j += adv;
        st += adv;
        if (st >= nks) {
          st -= nks;
          kph ^= 1u;
        }
      }
      // every product this thread issued has finished before tensor memory is released
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0);
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ O += P.V issuer
    // (P(i) exists only after the softmax read S(i), so Q.K(i) has finished and
    // releasing the stage after P.V(i) also covers the K half)
    if (lane == 0) {
      const uint32_t idesc_pv = umma_idesc_bf16(128, DV, false, true);
      const uint64_t vdesc0 = umma_desc_sw128(smem_u32(vring), 8192, 1024);
      bool ok = true;
      int total = first_s;
      int vs = 0;
      uint32_t vph = 0;   // V ring slot of P.V tile i and its phase parity
      for (int i = nkc; ok; ++i) {
        if (i == first_s) {
          ok = mbar_wait(&bars->sel_ready, 0, abort_flag, a.status, 417);
          if (!ok) break;
          total = first_s + bars->nu;
        }
        if (i >= total) break;
        const int sb = i & (kSBuf - 1);
        ok = mbar_wait(&bars->v_full[vs], vph, abort_flag, a.status, 419) &&
             mbar_wait(&bars->p_full[sb], ((i - nkc) >> 2) & 1, abort_flag, a.status, 412) &&
             (i != first_s || mbar_wait(&bars->ob_free, 0, abort_flag, a.status, 413));
        if (!ok) break;
        TR(i, 2);
        tc_fence_after();
        const bool first = (i == nkc) || (i == first_w) || (i == first_s);
        const uint32_t ocol = i < first_w ? kColOA : kColOB;
        const uint64_t vd = vdesc0 + (uint64_t)((uint32_t)vs * (uint32_t)(V_BYTES >> 4));
        // P (bf16 pairs, 32 columns) sits over the first half of the S columns of its buffer
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          umma_ts(tmem + ocol, tmem + col_s(sb) + (uint32_t)(kk * 8), vd + (uint64_t)(kk * (2048 >> 4)), idesc_pv,
                  (first && kk == 0) ? 0u : 1u);
        umma_commit(&bars->pv_done[sb]);
        umma_commit(&bars->v_empty[vs]);
        TR(i, 3);
        if (++vs == nvs) {
          vs = 0;
          vph ^= 1u;
        }
      }
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    // Warp w owns the 16 rows 32 * (w % 4) + 16 * (w / 4) .. + 15 (tensor-memory
    // lanes; a warp reaches only its own lane quarter w % 4). Lane i holds row
    // i % 16 and key columns 32 * kh .. + 31 of every tile (kh = i / 16): the two
    // half-warps split each tile's keys and trade row maxima and sums by
    // shuffles; each keeps the softmax denominator of its own columns until the
    // end of the phase. A half-warp's P store covers S columns the other half has
    // read, and both reads finish (tcgen05.wait::ld) before either store.
    const int kh = lane >> 4;         // key half
    const int q4 = warp & 3;          // TMEM lane quarter
    const int r = q4 * 32 + (warp >> 2) * 16 + (lane & 15);   // row = TMEM lane
    const int tt = r / G, hh = r % G;
    const int t = t0 + tt;
    const bool valid = t < L;
    const int64_t n = tok0 + t;
    const int hq = g * G + hh;
    const uint32_t lane_base = (uint32_t)(r - (lane & 15)) << 16;
    const uint32_t colh = 32u * (uint32_t)kh;   // this thread's key columns inside a tile
    const float sc = a.scale_log2;    // raw score -> log2 units
    float gc = 0.f, gsl = 0.f, gw = 0.f;
    if (valid) {
      const float* gp = a.gates + ((size_t)n * a.H_q + hq) * 3;
      gc = gp[0];
      gsl = gp[1];
      gw = gp[2];
    }
    const int jt = t / a.ls;
    float* imp_row = a.imp_smem ? imp_s + (size_t)tt * a.nb_stride : a.imp + ((size_t)n * a.H_kv + g) * a.nb_stride;

    bool ok = true;
    // waits give one answer per warp (the tensor-memory accesses after them are warp-wide)
    auto uwait = [&](uint64_t* bar, int parity, uint32_t site) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, (uint32_t)parity, abort_flag, a.status, site));
    };
    // the other key half's value for this row
    auto exchange = [&](float mine) -> float { return __shfl_xor_sync(0xffffffffu, mine, 16); };
    auto pair_max = [&](float mine) -> float { return fmaxf(mine, exchange(mine)); };
    // A thread holds the 32 scores of its row and columns for the current tile.
    float sv[32];
    int cur_j = 0;
    (void)cur_j;
    int cur_b = 0;   // S/P buffer of the tile being processed (tile j uses buffer j % 4)
    auto wait_s = [&](int j) -> bool {
      cur_b = j & (kSBuf - 1);
      cur_j = j;
      if (!uwait(&bars->s_full[cur_b], (j >> 2) & 1, 422)) return false;
      TR(j, 0);
      tc_fence_after();
      return true;
    };
    // raw scores of this warp's 32 keys of the current tile (two loads, one wait)
    auto ld32 = [&]() {
      const uint32_t src = tmem + lane_base + col_s(cur_b);
      tmem_ld16_h<32>(src, sv);
      tmem_ld16_h<32>(src + 16, sv + 16);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 32; ++c) asm volatile("" : "+f"(sv[c]));   // no use before the wait
    };
    // bf16 P (sv * scale) of keys colh .. colh + 31 into columns colh/2 .. colh/2 + 15
    // (P of key pair (2c, 2c+1) sits in column c; the warp's S reads are done)
    auto st32 = [&](float scale) {
#pragma unroll
      for (int c = 0; c < 16; c += 8) {
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(sv[2 * (c + i)] * scale, sv[2 * (c + i) + 1] * scale);
        tmem_st8_h<16>(tmem + lane_base + col_s(cur_b) + c, pk);
      }
    };
    auto st32_zero = [&]() {
      const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
      for (int c = 0; c < 16; c += 8) tmem_st8_h<16>(tmem + lane_base + col_s(cur_b) + c, z);
    };
    // all S reads of the tile are done (and its P written)
    auto tile_done = [&](bool with_p) {
      TR(cur_j, 2);
      if (with_p) tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->s_free[cur_b]);
      if (with_p) mbar_arrive(&bars->p_full[cur_b]);
      TR(cur_j, 3);
    };
    // P.V of tile i (>= nkc) has finished; p_full / pv_done phases count P.V tiles per buffer
    auto wait_pv = [&](int i) -> bool {
      if (!uwait(&bars->pv_done[i & (kSBuf - 1)], ((i - nkc) >> 2) & 1, 424)) return false;
      tc_fence_after();
      return true;
    };

    // ---------------- C1: compressed keys, row max and denominator (per warp, merged)
    const int nvis = valid ? cmp_visible_dev(t, a.l, a.s) : 0;
    float m = -1e30f, lp = 0.f;   // raw units
    for (int j = 0; j < nkc; ++j) {
      if (ok) ok = wait_s(j);
      const int c0 = j * kKeys + (int)colh;
      const bool part = !__all_sync(0xffffffffu, c0 + 32 <= nvis);
      if (ok) {
        ld32();
        tile_done(false);   // S is in registers: the buffer is free again
      }
      if (part) {
#pragma unroll
        for (int c = 0; c < 32; ++c) sv[c] = (c0 + c < nvis) ? sv[c] : -INFINITY;
      }
      const float mn = fmaxf(m, tree_max<32>(sv));
      const float mo = -mn * sc;
#pragma unroll
      for (int c = 0; c < 32; ++c) sv[c] = ex2(fmaf(sv[c], sc, mo));
      lp = lp * ex2((m - mn) * sc) + tree_sum<32>(sv);
      m = mn;
    }
    // p = 2^(s sc - m sc - log2 l): the denominator is folded into the exponent
    // (-inf when no compressed key is visible: p = 0)
    float mo_c = -INFINITY;
    if (nkc > 0) {   // merge the two key halves' (max, sum) in a fixed order
      const float m_o = exchange(m);
      const float l_o = exchange(lp);
      const float m0 = kh == 0 ? m : m_o, m1 = kh == 0 ? m_o : m;
      const float l0 = kh == 0 ? lp : l_o, l1 = kh == 0 ? l_o : lp;
      const float mm = fmaxf(m0, m1);
      const float lc = l0 * ex2((m0 - mm) * sc) + l1 * ex2((m1 - mm) * sc);
      mo_c = lc > 0.f ? -mm * sc - log2f(lc) : -INFINITY;
    }

    TRP(1);
    // ---------------- C2: probabilities, importance, O_A = P.V_cmp (g_cmp applied in the W merge)
    // compressed key i' = 4u' + u spans tokens [16i', 16i' + 32): u in {0,1,2} puts
    // 2p on selection block u', u = 3 puts p on u' and u' + 1 (overlap / stride).
    // The 32 keys of a warp cover 8 selection blocks; the mass its last key
    // carries into the next block is added before the selection.
    for (int i = 0; i < nkc; ++i) {
      const int j = nkc + i;
      if (ok) ok = wait_s(j);
      const int c0 = i * kKeys + (int)colh;
      const bool part = !__all_sync(0xffffffffu, c0 + 32 <= nvis);
      if (ok) ld32();
      if (part) {
#pragma unroll
        for (int c = 0; c < 32; ++c) sv[c] = (c0 + c < nvis) ? sv[c] : -INFINITY;
      }
#pragma unroll
      for (int c = 0; c < 32; ++c) sv[c] = ex2(fmaf(sv[c], sc, mo_c));
      if (ok) st32(1.f);
      TR(j, 1);
      const bool wr = valid && ok;
      const int B0 = 16 * i + 8 * kh;
      float carry;
      switch (G) {
        case 16: carry = importance32<16>(sv, 0.f, lane, wr, imp_row, B0, jt); break;
        case 8: carry = importance32<8>(sv, 0.f, lane, wr, imp_row, B0, jt); break;
        case 4: carry = importance32<4>(sv, 0.f, lane, wr, imp_row, B0, jt); break;
        case 2: carry = importance32<2>(sv, 0.f, lane, wr, imp_row, B0, jt); break;
        default: carry = importance32<1>(sv, 0.f, lane, wr, imp_row, B0, jt); break;
      }
      if (wr && hh == 0) cbuf[(2 * i + kh) * TOK + tt] = carry;
      if (ok) tile_done(true);
    }

    TRP(2);
    // ---------------- top-n per token and the tile's union of selected blocks
    int smx_phase = 0;
    auto sm_sync = [&]() {
      mbar_arrive(&bars->smx);
      if (!uwait(&bars->smx, smx_phase & 1, 425)) ok = false;
      ++smx_phase;
    };
    sm_sync();
    const int nh = 2 * nkc;   // 32-key halves of the compressed tiles
    for (int tk = warp; tk < TOK && ok; tk += 8) {
      const int tq = t0 + tk;
      if (tq >= L) break;
      const int64_t nq = tok0 + tq;
      const int jq = tq / a.ls;
      float* irow = a.imp_smem ? imp_s + (size_t)tk * a.nb_stride : a.imp + ((size_t)nq * a.H_kv + g) * a.nb_stride;
      // mass carried across the 32-key boundaries (written by the warps of the other half)
      for (int h = 1 + lane; h < nh; h += 32)
        if (8 * h <= jq) irow[8 * h] += cbuf[(h - 1) * TOK + tk];
      if (nh > 0) {
        for (int jb = 8 * nh + lane; jb <= jq; jb += 32)
          irow[jb] = (jb == 8 * nh) ? cbuf[(nh - 1) * TOK + tk] : 0.f;
      } else {
        for (int jb = lane; jb <= jq; jb += 32) irow[jb] = 0.f;
      }
      __syncwarp();
      int32_t* gsel = a.sel + ((size_t)nq * a.H_kv + g) * a.top_n;
      int32_t* srow = a.imp_smem ? sel_s + tk * 32 : gsel;
      warp_topn_any(irow, jq, a.top_n, a.force_first, a.force_local, srow, lane);
      __syncwarp();
      if (lane < a.top_n) {
        const int jb = srow[lane];
        if (jb >= 0 && NSA_BOUNDS(jb <= jq && (lane == 0 || srow[lane - 1] < jb), a.status, 503))
          atomicOr(&bm[jb * MW + (tk >> 5)], 1u << (tk & 31));
        if (a.imp_smem && a.want_sel) gsel[lane] = jb;
      }
      if (a.imp_smem && a.want_imp) {
        float* gimp = a.imp + ((size_t)nq * a.H_kv + g) * a.nb_stride;
        for (int jb = lane; jb <= jq; jb += 32) gimp[jb] = irow[jb];
      }
    }
    sm_sync();
    // the union of the tile's selections, ascending: each softmax warp takes a
    // contiguous range of 32-block chunks, counts its blocks, and after a sync
    // writes them at the offset of the warps before it
    {
      const int nch32 = (jt_max + 32) / 32, cpw = (nch32 + 7) / 8;
      const int c_lo = min(nch32, warp * cpw), c_hi = min(nch32, c_lo + cpw);
      auto chunk_bits = [&](int c) -> uint32_t {
        const int jb = c * 32 + lane;
        bool any = false;
        if (jb <= jt_max)
          for (int w = 0; w < MW; ++w) any |= bm[jb * MW + w] != 0u;
        return __ballot_sync(0xffffffffu, any);
      };
      int cnt = 0;
      for (int c = c_lo; c < c_hi; ++c) cnt += __popc(chunk_bits(c));
      if (lane == 0) bars->ucnt[warp] = cnt;
      sm_sync();
      int off = 0;
      for (int w = 0; w < warp; ++w) off += bars->ucnt[w];
      for (int c = c_lo; c < c_hi; ++c) {
        const uint32_t bal = chunk_bits(c);
        if ((bal >> lane) & 1u) uni[off + __popc(bal & ((1u << lane) - 1u))] = c * 32 + lane;
        off += __popc(bal);
      }
      if (warp == 7 && lane == 0) bars->nu = off;   // the total: warp 7's range ends last
    }
    sm_sync();
    TRP(3);
    if (tid == 0) mbar_arrive(&bars->sel_ready);
    const int nu = ok ? bars->nu : 0;

    // ---------------- online phases (window, selected blocks)
    // A tile raises the row's reference max only when its own max exceeds it by
    // more than kRescaleLog2 (rescaling this warp's half of O_B once the previous
    // product has landed); p = 2^(s - ref) stays below 2^kRescaleLog2.
    const float thr = kRescaleLog2 / sc;
    float m_ref = -1e30f;
    // mask32() masks the raw scores of this warp's keys; a row with rowv == false
    // takes no part in the tile (max -inf, p = 0) at no per-key cost
    auto online_tile = [&](int j, bool skip, bool rowv, auto&& mask32) -> bool {
      float tmx = -1e30f;
      if (!skip && ok) {
        ld32();
        mask32();
        tmx = tree_max<32>(sv);
        if (!rowv) tmx = -1e30f;
      }
      tmx = pair_max(tmx);
      TR(j, 1);
      if (!ok) return false;
      float ref = m_ref, alpha = 1.f;
      if (tmx > ref + thr) {
        alpha = ex2((ref - tmx) * sc);
        ref = tmx;
      }
      const bool had = m_ref > -1e29f;
      m_ref = ref;
      if (__any_sync(0xffffffffu, had && alpha != 1.f)) {
        if (!wait_pv(j - 1)) return false;
        tmem_scale_cols<DV / 2>(tmem + lane_base + kColOB, had ? alpha : 1.f);
      }
      lp *= alpha;
      if (skip) {
        st32_zero();
      } else {
        const float mo = rowv ? -ref * sc : -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; ++c) sv[c] = ex2(fmaf(sv[c], sc, mo));
        lp += tree_sum<32>(sv);
        st32(1.f);
      }
      tile_done(true);
      return true;
    };
    // denominator of the phase, both warps' columns summed in a fixed order
    auto phase_sum = [&]() -> float {
      const float other = exchange(lp);
      return kh == 0 ? lp + other : other + lp;
    };

    // ---------------- W: window keys into O_B, then O_A = g_cmp O_A + g_win / l * O_B
    const int wlo = t - a.window + 1;
    lp = 0.f;
    for (int i = 0; i < nkw; ++i) {
      const int j = first_w + i;
      if (ok) ok = wait_s(j);
      const int k0 = key0w + i * kKeys + (int)colh;
      const bool part = !__all_sync(0xffffffffu, valid && k0 >= wlo && k0 + 31 <= t);
      auto mask_w = [&]() {
        if (!part) return;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int tau = k0 + c;
          sv[c] = (valid && tau <= t && tau >= wlo) ? sv[c] : -INFINITY;
        }
      };
      if (!online_tile(j, false, valid, mask_w)) ok = false;
    }
    {
      const float lw = phase_sum();
      if (ok) ok = wait_pv(first_s - 1);
      const float sw = lw > 0.f ? gw / lw : 0.f;
#pragma unroll 1
      for (int c = 0; c < DV / 2; c += 16) {
        const uint32_t cb = lane_base + c;
        float ob[16], oa[16];
        tmem_ld16_h<DV / 2>(tmem + kColOB + cb, ob);
        if (nkc > 0) tmem_ld16_h<DV / 2>(tmem + kColOA + cb, oa);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = __float_as_uint((nkc > 0 ? gc * oa[e] : 0.f) + sw * ob[e]);
        tmem_st8_h<DV / 2>(tmem + kColOA + cb, w);
        tmem_st8_h<DV / 2>(tmem + kColOA + cb + 8, w + 8);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->ob_free);
    }

    TRP(4);
    // ---------------- S: union blocks, each row masked to its token's selection
    m_ref = -1e30f;
    lp = 0.f;
    for (int u = 0; u < nu; ++u) {
      const int j = first_s + u;
      if (ok) ok = wait_s(j);
      const int jb = uni[u];
      const bool mine = valid && ((bm[jb * MW + (tt >> 5)] >> (tt & 31)) & 1u);
      const int k0 = jb * a.ls + (int)colh;
      // no row of this warp selected the block: its P rows are zero
      const bool skip = !__any_sync(0xffffffffu, mine);
      // keys after t exist only in a row's own current block
      const bool part = __any_sync(0xffffffffu, mine && k0 + 31 > t);
      auto mask_s = [&]() {
        if (!part) return;
#pragma unroll
        for (int c = 0; c < 32; ++c) sv[c] = (k0 + c <= t) ? sv[c] : -INFINITY;
      };
      if (!online_tile(j, skip, mine, mask_s)) ok = false;
    }
    {
      const float ls_ = nu > 0 ? phase_sum() : 0.f;
      if (ok && nu > 0) ok = wait_pv(first_s + nu - 1);
      const float ss = ls_ > 0.f ? gsl / ls_ : 0.f;
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + ((size_t)n * a.H_q + hq) * DV + kh * (DV / 2);
#pragma unroll 1
      for (int c = 0; c < DV / 2; c += 16) {
        const uint32_t cb = lane_base + c;
        float ob[16], oa[16];
        tmem_ld16_h<DV / 2>(tmem + kColOB + cb, ob);
        tmem_ld16_h<DV / 2>(tmem + kColOA + cb, oa);
        tmem_ld_wait();
        if (valid && ok) {
          uint4 pk0, pk1;
          pk0.x = pack_bf16x2(fmaf(ss, ob[0], oa[0]), fmaf(ss, ob[1], oa[1]));
          pk0.y = pack_bf16x2(fmaf(ss, ob[2], oa[2]), fmaf(ss, ob[3], oa[3]));
          pk0.z = pack_bf16x2(fmaf(ss, ob[4], oa[4]), fmaf(ss, ob[5], oa[5]));
          pk0.w = pack_bf16x2(fmaf(ss, ob[6], oa[6]), fmaf(ss, ob[7], oa[7]));
          pk1.x = pack_bf16x2(fmaf(ss, ob[8], oa[8]), fmaf(ss, ob[9], oa[9]));
          pk1.y = pack_bf16x2(fmaf(ss, ob[10], oa[10]), fmaf(ss, ob[11], oa[11]));
          pk1.z = pack_bf16x2(fmaf(ss, ob[12], oa[12]), fmaf(ss, ob[13], oa[13]));
          pk1.w = pack_bf16x2(fmaf(ss, ob[14], oa[14]), fmaf(ss, ob[15], oa[15]));
          *reinterpret_cast<uint4*>(dst + c) = pk0;
          *reinterpret_cast<uint4*>(dst + c + 8) = pk1;
        }
      }
    }
  }

  TRP(5);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// K and V ring depths that fit the opt-in shared memory of one CTA (false: none)
static size_t imp_smem_bytes(int nb, int G) { return (size_t)(128 / G) * (nb + 32) * 4; }

bool prefill_fused_stages(PrefillArgs& a) {
  const size_t kb = (size_t)kKeys * a.d_k * 2, vb = (size_t)kKeys * a.d_v * 2;
  size_t budget = 232448 - 1024 - (size_t)128 * a.d_k * 2 - fused_fixed_bytes(a.nb_stride, a.G);
  int n = (int)(budget / (kb + vb));
  if (n > kMaxStages) n = kMaxStages;
  if (n < 2) return false;
  // long sequences: keep the importance on chip by giving up V stages (down to
  // two) before spilling it to the workspace
  const size_t ib = imp_smem_bytes(a.nb_stride, a.G);
  if (budget < (size_t)n * (kb + vb) + ib) {
    for (int nv = n - 1; nv >= 2; --nv)
      if (budget >= (size_t)n * kb + (size_t)nv * vb + ib) {
        a.imp_smem = 1;
        a.n_stages = n & ~1;
        a.n_vstages = nv;
        return true;
      }
  }
  budget -= (size_t)n * (kb + vb);
  // the tile's importance and selections stay on chip when the room is left over
  a.imp_smem = budget >= imp_smem_bytes(a.nb_stride, a.G) ? 1 : 0;
  if (a.imp_smem) budget -= imp_smem_bytes(a.nb_stride, a.G);
  int nk = n + (int)(budget / kb);   // spare room holds extra K tiles
  if (nk > kMaxStages) nk = kMaxStages;
  a.n_stages = nk & ~1;   // even: tiles are computed in pairs of adjacent K slots
  a.n_vstages = n;
  return true;
}

template <int DK, int DV>
static cudaError_t launch_fused_t(const PrefillArgs& a, const PrefillMaps& m, int n_tiles, cudaStream_t st) {
  auto kern = nsa_prefill_kernel<DK, DV>;
  const size_t smem = 1024 + (size_t)128 * DK * 2 + (size_t)a.n_stages * kKeys * DK * 2 +
                     (size_t)a.n_vstages * kKeys * DV * 2 + fused_fixed_bytes(a.nb_stride, a.G) +
                     (a.imp_smem ? imp_smem_bytes(a.nb_stride, a.G) : 0);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(n_tiles, a.H_kv), kThreads, smem, st>>>(a, m);
  return cudaGetLastError();
}

cudaError_t launch_prefill_fused(const PrefillArgs& a, const PrefillMaps& m, int n_tiles, cudaStream_t st) {
  if (n_tiles == 0) return cudaSuccess;
  if (a.n_stages < 2 || a.n_stages > kMaxStages || a.n_vstages < 2 || a.n_vstages > kMaxStages)
    return cudaErrorInvalidValue;
  if (a.d_k == 192 && a.d_v == 128) return launch_fused_t<192, 128>(a, m, n_tiles, st);
  if (a.d_k == 64 && a.d_v == 64) return launch_fused_t<64, 64>(a, m, n_tiles, st);
  if (a.d_k == 128 && a.d_v == 128) return launch_fused_t<128, 128>(a, m, n_tiles, st);
  if (a.d_k == 192 && a.d_v == 64) return launch_fused_t<192, 64>(a, m, n_tiles, st);
  if (a.d_k == 64 && a.d_v == 128) return launch_fused_t<64, 128>(a, m, n_tiles, st);
  if (a.d_k == 128 && a.d_v == 64) return launch_fused_t<128, 64>(a, m, n_tiles, st);
  return cudaErrorInvalidValue;
}

}  // namespace nsa

#ifdef NSA_PREFILL_TRACE
extern "C" int nsa_prefill_trace_read(void* tiles, void* phases) {
  if (cudaMemcpyFromSymbol(tiles, nsa::g_trace, sizeof(nsa::g_trace)) != cudaSuccess) return 1;
  if (cudaMemcpyFromSymbol(phases, nsa::g_trace_phase, sizeof(nsa::g_trace_phase)) != cudaSuccess) return 1;
  return 0;
}
extern "C" int nsa_prefill_trace_clear() {
  static unsigned long long z[4 * 12 * nsa::kTrTiles * 4];
  if (cudaMemcpyToSymbol(nsa::g_trace, z, sizeof(nsa::g_trace)) != cudaSuccess) return 1;
  if (cudaMemcpyToSymbol(nsa::g_trace_phase, z, sizeof(nsa::g_trace_phase)) != cudaSuccess) return 1;
  return 0;
}
#endif
