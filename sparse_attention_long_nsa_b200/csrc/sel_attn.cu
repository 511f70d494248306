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
// ---------------------------------------------------------------------------
namespace {
constexpr int kSelStages = 4;
constexpr int kSelConsumers = 4;
constexpr int kSelThreads = (kSelConsumers + 1) * 32;

template <int DK, int DV>
struct SelSmem {
  static constexpr int K_BYTES = 64 * DK * 2;
  static constexpr int V_BYTES = 64 * DV * 2;
  static constexpr int STAGE = K_BYTES + V_BYTES;
  static constexpr int MERGE = kSelConsumers * 16 * (DV + 2) * 4;
  static constexpr int RING = kSelStages * STAGE;
  static constexpr int TOTAL = 1024 + (RING > MERGE ? RING : MERGE) + 1024;
};
}  // namespace

template <int DK, int DV>
__global__ void __launch_bounds__(kSelThreads, 1) sel_attn_kernel(const PrefillArgs a,
                                                                  const __grid_constant__ PrefillMaps mp) {
  using S = SelSmem<DK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (S::RING > S::MERGE ? S::RING : S::MERGE));
  uint64_t* empty = full + kSelStages;
  int* sel_s = reinterpret_cast<int*>(empty + kSelStages);     // [32]
  volatile int* abort_flag = sel_s + 32;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n = blockIdx.x / a.H_kv;
  const int g = blockIdx.x % a.H_kv;
  const int b = seq_of_token(a.seqs, n);
  const int t = (int)(n - a.seqs.tok_off[b]);
  const int64_t tok0 = a.seqs.tok_off[b];
  const int G = a.G;

  if (tid < 32) sel_s[tid] = tid < a.top_n ? a.sel[((size_t)n * a.H_kv + g) * a.top_n + tid] : -1;
  if (tid == 0) {
    for (int i = 0; i < kSelStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  int nsel = 0;
  while (nsel < a.top_n && sel_s[nsel] >= 0) ++nsel;

  if (warp == kSelConsumers) {
    if (lane == 0) {
      for (int i = 0; i < nsel; ++i) {
        const int st = i % kSelStages;
        if (i >= kSelStages && !mbar_wait(&empty[st], ((i / kSelStages) - 1) & 1, abort_flag, a.status, 301)) break;
        uint8_t* Ks = ring + st * S::STAGE;
        uint8_t* Vs = Ks + S::K_BYTES;
        const int row = (int)(tok0 + (int64_t)sel_s[i] * a.ls);
        mbar_arrive_expect_tx(&full[st], S::STAGE);
        for (int kb = 0; kb < DK / 64; ++kb) tma_load_3d(Ks + kb * 8192, &mp.k, &full[st], kb * 64, g, row);
        for (int vb = 0; vb < DV / 64; ++vb) tma_load_3d(Vs + vb * 8192, &mp.v, &full[st], vb * 64, g, row);
      }
    }
  } else {
    uint32_t qa[DK / 16][4];
    RowState<DV> rs;
    rs.init();
    const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(a.q) + ((size_t)n * a.H_q + (size_t)g * G) * DK;
    load_q_frags<DK>(qa, qp, G, lane);
    for (int i = warp; i < nsel; i += kSelConsumers) {
      const int st = i % kSelStages;
      if (!mbar_wait(&full[st], (i / kSelStages) & 1, abort_flag, a.status, 302)) break;
      const uint32_t kb = smem_u32(ring + st * S::STAGE);
      float s[8][4];
      warp_qk<DK>(qa, kb, s, lane);
      const int key0 = sel_s[i] * a.ls + (lane & 3) * 2;
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
    rs.finish();
    // publish the partial state once every consumer is done with the ring
    named_bar_sync(1, kSelConsumers * 32);
    rs.stage(reinterpret_cast<float*>(ring) + warp * 16 * (DV + 2), lane);
    named_bar_sync(1, kSelConsumers * 32);
    // merge: thread handles (row, dv range)
    const float* base = reinterpret_cast<const float*>(ring);
    const int per_row = (kSelConsumers * 32) / 16;   // threads per row
    const int row = tid / per_row;
    const int part = tid % per_row;
    if (row < G) {
      float M = -1e30f;
      for (int w = 0; w < kSelConsumers; ++w) M = fmaxf(M, base[(w * 16 + row) * (DV + 2) + DV]);
      float wsc[kSelConsumers], Lsum = 0.f;
      for (int w = 0; w < kSelConsumers; ++w) {
        const float* rw = base + (w * 16 + row) * (DV + 2);
        wsc[w] = rw[DV + 1] > 0.f ? exp2f(rw[DV] - M) : 0.f;
        Lsum += wsc[w] * rw[DV + 1];
      }
      const int h = g * G + row;
      const float gs = a.gates[((size_t)n * a.H_q + h) * 3 + 1] / Lsum;
      float* dst = a.acc + ((size_t)n * a.H_q + h) * DV;
      const int span = DV / per_row;
      for (int c = part * span; c < (part + 1) * span; ++c) {
        float v = 0.f;
        for (int w = 0; w < kSelConsumers; ++w) v += wsc[w] * base[(w * 16 + row) * (DV + 2) + c];
        dst[c] += gs * v;
      }
    }
  }
  __syncthreads();
}

template <int DK, int DV>
static cudaError_t launch_sel_t(const PrefillArgs& a, const PrefillMaps& m, int64_t n_tokens, cudaStream_t st) {
  using S = SelSmem<DK, DV>;
  auto kern = sel_attn_kernel<DK, DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::TOTAL);
  if (e != cudaSuccess) return e;
  const int64_t grid = n_tokens * a.H_kv;
  if (grid > 0x7fffffff) return cudaErrorInvalidValue;
  kern<<<(unsigned)grid, kSelThreads, S::TOTAL, st>>>(a, m);
  return cudaGetLastError();
}

cudaError_t launch_sel_attn(const PrefillArgs& a, const PrefillMaps& m, int64_t n_tokens, cudaStream_t st) {
  if (n_tokens == 0) return cudaSuccess;
  if (a.d_k == 192 && a.d_v == 128) return launch_sel_t<192, 128>(a, m, n_tokens, st);
  if (a.d_k == 64 && a.d_v == 64) return launch_sel_t<64, 64>(a, m, n_tokens, st);
  if (a.d_k == 128 && a.d_v == 128) return launch_sel_t<128, 128>(a, m, n_tokens, st);
  if (a.d_k == 192 && a.d_v == 64) return launch_sel_t<192, 64>(a, m, n_tokens, st);
  if (a.d_k == 64 && a.d_v == 128) return launch_sel_t<64, 128>(a, m, n_tokens, st);
  if (a.d_k == 128 && a.d_v == 64) return launch_sel_t<128, 64>(a, m, n_tokens, st);
  return cudaErrorInvalidValue;
}

}  // namespace nsa
