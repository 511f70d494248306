// Selected-block attention (prefill) and top-n block selection.
//
// Selection ("Native Sparse Attention" lesson, aiengineeringfromscratch.com,
// step 3; "Разреженное внимание — NSA и DSA", ai.flicky.cc, section "NSA: три
// ветви", selection branch): per (token t, KV head g) take every candidate block
// 0..t/l' when they fit in top_n; otherwise force the first `force_first` blocks
// and the `force_local` blocks ending at the one holding t, then fill the
// remaining slots with the highest importance, ties to the lower block index.
// One warp per (t, g): a 32-step radix select on the order-preserving bit
// pattern of the scores finds the threshold, ties are resolved in index order
// with ballots, and the result is compacted in ascending order.
//
// Attention over the selected blocks (same section: exact attention over the
// n*l' raw tokens of the chosen blocks, shared by all heads of the GQA group;
// keys after t inside the current block are masked). One CTA per (t, g): a
// producer thread streams each chosen block of 64 keys once through a 4-stage
// TMA ring; four consumer warps each take every fourth block and run the G
// heads (padded to the 16 rows of an m16n8k16 tile) against it with an online
// softmax, then the four partial states are merged and g_slc * o_slc is added
// to the fp32 accumulator.
#include "common.cuh"
#include "kernels.h"
#include "topn.cuh"
#include "warp_mma.cuh"

namespace nsa {

namespace {

__device__ __forceinline__ int seq_of_tile(const SeqTable& t, int tile) {
  int lo = 0, hi = t.n - 1;
  while (lo < hi) {   // last b with tile_prefix[b] <= tile
    const int mid = (lo + hi + 1) >> 1;
    if (t.tile_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int seq_of_token(const SeqTable& t, int64_t row) {
  int lo = 0, hi = t.n - 1;
  while (lo < hi) {   // last b with tok_off[b] <= row and len > 0 reaching it
    const int mid = (lo + hi + 1) >> 1;
    if (t.tok_off[mid] <= row) lo = mid; else hi = mid - 1;
  }
  while (lo > 0 && row >= t.tok_off[lo] + t.len[lo]) --lo;   // (only for empty sequences)
  return lo;
}

}  // namespace

// ---------------------------------------------------------------------------
// top-n selection
// ---------------------------------------------------------------------------
template <int PER>
__global__ void __launch_bounds__(128) topn_kernel(const PrefillArgs a, int64_t n_tokens) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (wid >= n_tokens * a.H_kv) return;
  const int64_t n = wid / a.H_kv;
  const int g = (int)(wid % a.H_kv);
  const int b = seq_of_token(a.seqs, n);
  const int t = (int)(n - a.seqs.tok_off[b]);
  warp_topn<PER>(a.imp + ((size_t)n * a.H_kv + g) * a.nb_stride, t / a.ls, a.top_n, a.force_first,
                 a.force_local, a.sel + ((size_t)n * a.H_kv + g) * a.top_n, lane);
}

cudaError_t launch_topn(const PrefillArgs& a, int64_t n_tokens, cudaStream_t st) {
  const int64_t warps = n_tokens * a.H_kv;
  if (warps == 0) return cudaSuccess;
  const int blocks = (int)((warps + 3) / 4);
  const int per = (a.nb_stride + 31) / 32;
  if (per <= 4) topn_kernel<4><<<blocks, 128, 0, st>>>(a, n_tokens);
  else if (per <= 8) topn_kernel<8><<<blocks, 128, 0, st>>>(a, n_tokens);
  else if (per <= 16) topn_kernel<16><<<blocks, 128, 0, st>>>(a, n_tokens);
  else if (per <= 32) topn_kernel<32><<<blocks, 128, 0, st>>>(a, n_tokens);
  else if (per <= 64) topn_kernel<64><<<blocks, 128, 0, st>>>(a, n_tokens);
  else if (per <= 128) topn_kernel<128><<<blocks, 128, 0, st>>>(a, n_tokens);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// selected-block attention
//
// CTA = 8 consecutive tokens of one sequence x one KV head; consumer warp w owns
// token t0 + w (its G heads are the 16 MMA rows; Q for the 8 tokens is staged in
// shared memory by one TMA box). The blocks the 8 tokens selected are merged into
// one ascending union; a producer warp streams each union block once through a
// 4-stage TMA ring, and every warp whose token selected it computes on it (the
// forced blocks 0, jt-1, jt are shared by all 8). Warps wait only for their own
// blocks: the producer publishes which union position a stage holds, and a
// stage is refilled once the warps that needed its block released it (the
// producer itself stands in for the warps that did not need it). Each warp adds
// g_slc * o_slc of its own token to the fp32 accumulator from its fragments.
// ---------------------------------------------------------------------------
namespace {
constexpr int kSelStages = 4;
constexpr int kSelTok = 8;                        // tokens (consumer warps) per CTA
constexpr int kSelThreads = (kSelTok + 1) * 32;   // + producer warp
constexpr int kSelMaxUnion = kSelTok * 32;        // top_n <= 32

template <int DK, int DV>
struct SelSmem {
  static constexpr int K_BYTES = 64 * DK * 2;
  static constexpr int V_BYTES = 64 * DV * 2;
  static constexpr int STAGE = K_BYTES + V_BYTES;
  static constexpr int RING = kSelStages * STAGE;
  static constexpr int Q_MAX = kSelTok * 16 * DK * 2;   // 8 tokens x G <= 16 heads
  // Q | ring | barriers | stage tags | union list | union masks | flags | bitmap [nb_stride]
  static constexpr int FIXED = 1024 + Q_MAX + RING + (2 * kSelStages + 1) * 8 + kSelStages * 4 +
                               kSelMaxUnion * 8 + 64;
  static int total(int nb_stride) { return FIXED + nb_stride * 4; }
};
}  // namespace

template <int DK, int DV>
__global__ void __launch_bounds__(kSelThreads, 1) sel_attn_kernel(const PrefillArgs a,
                                                                  const __grid_constant__ PrefillMaps mp) {
  using S = SelSmem<DK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qs = smem;                                            // [DK/64][8*G rows][128 B]
  uint8_t* ring = smem + S::Q_MAX;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + S::RING);
  uint64_t* empty = full + kSelStages;
  uint64_t* q_full = empty + kSelStages;
  volatile int* stage_tag = reinterpret_cast<volatile int*>(q_full + 1);   // union position held
  int* uni = const_cast<int*>(stage_tag) + kSelStages;          // [kSelMaxUnion]
  uint32_t* umask = reinterpret_cast<uint32_t*>(uni + kSelMaxUnion);
  int* nuni = reinterpret_cast<int*>(umask + kSelMaxUnion);
  volatile int* abort_flag = nuni + 1;
  uint32_t* bm = reinterpret_cast<uint32_t*>(nuni + 16);         // [nb_stride] warp bits per block

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G;
  const int TOK = 256 / G, SUB = TOK / kSelTok;   // host tiles hold 2 x 128/G tokens
  const int tile = blockIdx.x / SUB, sub = blockIdx.x % SUB;
  const int g = blockIdx.y;
  const int b = seq_of_tile(a.seqs, tile);
  const int L = a.seqs.len[b];
  const int64_t tok0 = a.seqs.tok_off[b];
  const int t0 = (tile - a.seqs.tile_prefix[b]) * TOK + sub * kSelTok;
  if (t0 >= L) return;   // whole CTA past the end of its sequence (uniform)
  const int t_last = min(t0 + kSelTok - 1, L - 1);
  const int jt_max = t_last / a.ls;
  const uint32_t qchunk = (uint32_t)kSelTok * G * 128;

  for (int j = tid; j <= jt_max; j += kSelThreads) bm[j] = 0u;
  if (tid == 0) {
    for (int i = 0; i < kSelStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kSelTok);
      stage_tag[i] = -1;
    }
    mbar_init(q_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // mark the blocks each token selected
  const int t = t0 + warp;
  const bool has_tok = warp < kSelTok && t < L;
  const int64_t n = tok0 + t;
  if (has_tok && lane < a.top_n) {
    const int j = a.sel[((size_t)n * a.H_kv + g) * a.top_n + lane];
    if (j >= 0 && j <= jt_max) atomicOr(&bm[j], 1u << warp);
  }
  __syncthreads();
  // compact the union in ascending block order (producer warp)
  if (warp == kSelTok) {
    int cnt = 0;
    for (int j0 = 0; j0 <= jt_max; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t m = j <= jt_max ? bm[j] : 0u;
      const uint32_t bal = __ballot_sync(0xffffffffu, m != 0u);
      if (m != 0u) {
        const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
        uni[pos] = j;
        umask[pos] = m;
      }
      cnt += __popc(bal);
    }
    if (lane == 0) *nuni = cnt;
  }
  __syncthreads();
  const int nu = *nuni;

  if (warp == kSelTok) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, (uint32_t)(DK / 64) * qchunk);
      for (int kb = 0; kb < DK / 64; ++kb)
        tma_load_3d(qs + kb * qchunk, &mp.q8, q_full, kb * 64, g * G, (int)(tok0 + t0));
      int issued = 0;
      for (int u = 0; u < nu; ++u) {
        const int st = u % kSelStages;
        if (u >= kSelStages && !mbar_wait(&empty[st], ((u / kSelStages) - 1) & 1, abort_flag, a.status, 301)) break;
        issued = u + 1;
        stage_tag[st] = u;
        uint8_t* Ks = ring + st * S::STAGE;
        const int row = (int)(tok0 + (int64_t)uni[u] * a.ls);
        mbar_arrive_expect_tx(&full[st], S::STAGE);
        for (int kb = 0; kb < DK / 64; ++kb) tma_load_3d(Ks + kb * 8192, &mp.k, &full[st], kb * 64, g, row);
        for (int vb = 0; vb < DV / 64; ++vb)
          tma_load_3d(Ks + S::K_BYTES + vb * 8192, &mp.v, &full[st], vb * 64, g, row);
        const uint32_t others = kSelTok - __popc(umask[u]);   // warps that will not release it
        if (others) mbar_arrive_cnt(&empty[st], others);
      }
      if (*abort_flag) {   // let the copies still in flight land before the CTA exits
        mbar_wait_drain(q_full, 0);
        for (int v = issued - kSelStages < 0 ? 0 : issued - kSelStages; v < issued; ++v)
          mbar_wait_drain(&full[v % kSelStages], (v / kSelStages) & 1);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    RowState<DV> rs;
    rs.init();
    const uint32_t bit = 1u << warp;
    bool ok = true;
    if (has_tok) {
      ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, abort_flag, a.status, 303));
      const uint32_t qbase = smem_u32(qs);
      for (int u = 0; u < nu && ok; ++u) {
        if (!(umask[u] & bit)) continue;
        const int st = u % kSelStages;
        // the stage must hold union position u before its barrier phase is meaningful
        bool w = smem_wait_eq(&stage_tag[st], u, abort_flag, a.status, 304) &&
                 mbar_wait(&full[st], (u / kSelStages) & 1, abort_flag, a.status, 302);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        const uint32_t kb = smem_u32(ring + st * S::STAGE);
        float s[8][4];
        warp_qk_sq<DK>(qbase, qchunk, warp * G, kb, s, lane);
        const int key0 = uni[u] * a.ls + (lane & 3) * 2;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const bool vis = key0 + nt * 8 + e <= t;
            s[nt][e] = vis ? s[nt][e] * a.scale_log2 : -INFINITY;
            s[nt][2 + e] = vis ? s[nt][2 + e] * a.scale_log2 : -INFINITY;
          }
        }
        rs.update(s);
        warp_pv<DV>(s, kb + S::K_BYTES, rs.o, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
      }
    }
    rs.finish();
    if (has_tok && ok) {
      // acc[n, h, :] += g_slc * o / l for the group's heads (rows lane/4, lane/4 + 8)
      const int r0 = lane >> 2, cq = (lane & 3) * 2;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int row = r0 + half * 8;
        if (row < G) {
          const int h = g * G + row;
          const float gs = a.gates[((size_t)n * a.H_q + h) * 3 + 1] / rs.l[half];
          float* dst = a.acc + ((size_t)n * a.H_q + h) * DV;
#pragma unroll
          for (int i = 0; i < DV / 8; ++i) {
            float2* p = reinterpret_cast<float2*>(dst + i * 8 + cq);
            float2 v = *p;
            v.x += gs * rs.o[i][2 * half];
            v.y += gs * rs.o[i][2 * half + 1];
            *p = v;
          }
        }
      }
    }
  }
  __syncthreads();
}

template <int DK, int DV>
static cudaError_t launch_sel_t(const PrefillArgs& a, const PrefillMaps& m, int n_tiles, cudaStream_t st) {
  using S = SelSmem<DK, DV>;
  auto kern = sel_attn_kernel<DK, DV>;
  const int smem = S::total(a.nb_stride);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int sub = (256 / a.G) / kSelTok;
  kern<<<dim3(n_tiles * sub, a.H_kv), kSelThreads, smem, st>>>(a, m);
  return cudaGetLastError();
}

cudaError_t launch_sel_attn(const PrefillArgs& a, const PrefillMaps& m, int n_tiles, cudaStream_t st) {
  if (n_tiles == 0) return cudaSuccess;
  if (a.d_k == 192 && a.d_v == 128) return launch_sel_t<192, 128>(a, m, n_tiles, st);
  if (a.d_k == 64 && a.d_v == 64) return launch_sel_t<64, 64>(a, m, n_tiles, st);
  if (a.d_k == 128 && a.d_v == 128) return launch_sel_t<128, 128>(a, m, n_tiles, st);
  if (a.d_k == 192 && a.d_v == 64) return launch_sel_t<192, 64>(a, m, n_tiles, st);
  if (a.d_k == 64 && a.d_v == 128) return launch_sel_t<64, 128>(a, m, n_tiles, st);
  if (a.d_k == 128 && a.d_v == 64) return launch_sel_t<128, 64>(a, m, n_tiles, st);
  return cudaErrorInvalidValue;
}

}  // namespace nsa
