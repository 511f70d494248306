// Block compression: k_cmp[i] = vec(x[i*s : i*s+l] + pe) . W  (per KV head).
//
// "Разреженное внимание — NSA и DSA" (ai.flicky.cc), section "NSA: три ветви",
// compression branch: overlapping blocks of l tokens with stride s, each mapped
// to one key and one value by a learned map. The map here is one linear layer W
// [l*d_in, d_out] of the token-major flattened block plus a position embedding
// pe [l, d_in] added to every token; by linearity the embedding contributes the
// constant row vec(pe).W, which the prep kernel computes once in fp32.
//
// The GEMM runs on the 5th-generation tensor cores: M = 128 compressed rows of
// one KV head, N = d_out, K = l*d_in, bf16 operands staged in 128-byte-swizzled
// shared memory, fp32 accumulator in tensor memory (tcgen05.mma issued by one
// thread), read back with tcgen05.ld for the bias-add + bf16 epilogue. When the
// rows give too few CTAs to fill the GPU, the K = l*d_in reduction is split over
// grid.z into fp32 partial sums that a small kernel adds in a fixed order.
// The A rows are a strided gather (row i starts at token i*s): one TMA box over a
// (channel, token mod s, token div s) view of the packed tokens, or cp.async rows
// (paged input, last partial group of s tokens); the B tile (64 columns of W^T)
// is one TMA box.
#include "common.cuh"
#include "kernels.h"

namespace nsa {

// ---------------------------------------------------------------------------
// prep: wt[n][k] = bf16(w[k][n]); partial[kt][n] = sum over the 32 rows of tile
// kt of pe_flat[k] * w[k][n]; bias[n] = sum_kt partial[kt][n] (fixed order)
// ---------------------------------------------------------------------------
__global__ void compress_transpose_kernel(const float* __restrict__ w, const float* __restrict__ pe,
                                          int K, int N, __nv_bfloat16* __restrict__ wt,
                                          float* __restrict__ partial) {
  __shared__ float tile[32][33];
  const int k0 = blockIdx.y * 32, n0 = blockIdx.x * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;   // 32 x 8
  for (int r = ty; r < 32; r += 8) {
    const int k = k0 + r, n = n0 + tx;
    tile[r][tx] = (k < K && n < N) ? w[(size_t)k * N + n] : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int n = n0 + r, k = k0 + tx;
    if (n < N && k < K) wt[(size_t)n * K + k] = __float2bfloat16_rn(tile[tx][r]);
  }
  if (ty == 0) {
    const int n = n0 + tx;
    float s = 0.f;
    for (int r = 0; r < 32; ++r) {
      const int k = k0 + r;
      if (k < K) s = fmaf(pe[k], tile[r][tx], s);
    }
    if (n < N) partial[(size_t)blockIdx.y * N + n] = s;
  }
}

// 32 columns per CTA of 32 x 8 threads: thread (x, y) adds the tiles
// y, y + 8, ... of column x, then the 8 partial sums are added in order y = 0..7
__global__ void compress_bias_kernel(const float* __restrict__ partial, int KT, int N,
                                     float* __restrict__ bias) {
  __shared__ float acc[8][33];
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int n = blockIdx.x * 32 + tx;
  float s = 0.f;
  if (n < N)
    for (int kt = ty; kt < KT; kt += 8) s += partial[(size_t)kt * N + n];
  acc[ty][tx] = s;
  __syncthreads();
  if (ty == 0 && n < N) {
    float t = acc[0][tx];
#pragma unroll
    for (int y = 1; y < 8; ++y) t += acc[y][tx];
    bias[n] = t;
  }
}

cudaError_t launch_compress_prep(const float* w, const float* pe, int K, int N, void* wt_bf16,
                                 float* partial, float* bias, cudaStream_t st) {
  dim3 grid((N + 31) / 32, (K + 31) / 32);
  compress_transpose_kernel<<<grid, dim3(32, 8), 0, st>>>(
      w, pe, K, N, static_cast<__nv_bfloat16*>(wt_bf16), partial);
  compress_bias_kernel<<<(N + 31) / 32, dim3(32, 8), 0, st>>>(partial, (K + 31) / 32, N, bias);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// GEMM
// ---------------------------------------------------------------------------
constexpr int kCmpStages = 4;
constexpr int kTileM = 128;

template <int D_OUT>
struct CompressSmem {
  static constexpr int A_BYTES = kTileM * 128;            // 128 rows x 64 bf16
  static constexpr int B_BYTES = D_OUT * 128;             // D_OUT rows x 64 bf16
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int TOTAL = kCmpStages * STAGE + 1024 /*align*/ + 256 /*barriers*/;
};

__device__ __forceinline__ int find_seq(const SeqTable& t, int tile) {
  int b = 0;
  while (b + 1 < t.n && t.tile_prefix[b + 1] <= tile) ++b;
  return b;
}

// one map (m = 0 keys, 1 values) of KV head g
template <int D_IN, int D_OUT>
__device__ __forceinline__ void compress_gemm_body(const CompressArgs& a, const CompressMaps& mp, int m, int g) {
  using S = CompressSmem<D_OUT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* mma_done = reinterpret_cast<uint64_t*>(smem + kCmpStages * S::STAGE);
  uint64_t* b_full = mma_done + kCmpStages + 1;   // the B tile of a stage has landed (TMA)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(b_full + kCmpStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x;
  const int b = find_seq(a.seqs, tile);
  const int L = a.seqs.len[b];
  const int ncmp = n_cmp_of(L, a.l, a.s);
  const int i0 = (tile - a.seqs.tile_prefix[b]) * kTileM;
  const int64_t tok0 = a.seqs.tok_off[b];
  const int K = a.l * D_IN;
  const int kb0 = blockIdx.z * a.kb_per_split[m];              // this CTA's share of K
  const int nkb = min(K / 64 - kb0, a.kb_per_split[m]);
  constexpr uint32_t TM_COLS = D_OUT <= 64 ? 64 : (D_OUT <= 128 ? 128 : 256);

  if (tid == 0) {
    for (int i = 0; i <= kCmpStages; ++i) mbar_init(&mma_done[i], 1);
    for (int i = 0; i < kCmpStages; ++i) mbar_init(&b_full[i], 1);
    prefetch_tmap(&mp.w[m]);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, TM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;

  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(a.x[m]);
  const size_t row_stride = (size_t)a.H_kv * D_IN;   // elements between tokens

  // The A tile of a K block (token offset r) is rows i0 .. i0+127 of the view
  // (channel, token mod s, token div s) of the packed tokens: one TMA box when
  // every row this CTA writes lies in whole groups of s tokens inside the view
  // (rows past its end read zeros and are never written out); otherwise (paged
  // input, or a last partial group) one cp.async row per thread.
  const int64_t last_tok = tok0 + (int64_t)(min(i0 + kTileM, ncmp) - 1) * a.s + a.l - 1;
  const bool a_tma = a.x_chunks > 0 && !a.x_pt.table && last_tok < (int64_t)a.x_chunks * a.s;
  auto load_stage = [&](int st, int kb) {
    uint8_t* A = smem + st * S::STAGE;
    uint8_t* Bm = A + S::A_BYTES;
    const int f0 = (kb0 + kb) * 64;
    const int r = f0 / D_IN, e0 = f0 % D_IN;
    if (a_tma) {
      if (tid == 0) {
        const int64_t t_row0 = tok0 + (int64_t)i0 * a.s + r;   // token of row i0
        mbar_arrive_expect_tx(&b_full[st], (uint32_t)(S::A_BYTES + S::B_BYTES));
        tma_load_3d(A, &mp.x[m], &b_full[st], g * D_IN + e0, (int)(t_row0 % a.s), (int)(t_row0 / a.s));
        tma_load_3d(Bm, &mp.w[m], &b_full[st], f0, 0, 0);
      }
      return;
    }
    {  // A: one 128-byte row per thread
      const int row = tid;
      const int ci = i0 + row;
      bool ok = ci < ncmp;
      int64_t xr = tok0 + (int64_t)(ok ? ci : 0) * a.s + r;   // token row (paged: index in the sequence)
      if (a.x_pt.table) {
        const int pg = a.x_pt.table[(int64_t)b * a.x_pt.max_pages + (int)(xr / a.x_pt.page_size)];
        if (pg < 0 || pg >= a.x_pt.n_pages) {   // invalid page: zeros, and the error is recorded
          if (ok) atomicOr(a.status, DEV_ERR_BOUNDS);
          ok = false;
          xr = 0;
        } else {
          xr = (int64_t)pg * a.x_pt.page_size + xr % a.x_pt.page_size;
        }
      }
      const __nv_bfloat16* src = x + (size_t)xr * row_stride + (size_t)g * D_IN + e0;
#pragma unroll
      for (int c = 0; c < 8; ++c) cp_async16_zfill(A + sw128(row, c), src + c * 8, ok);
    }
    // B: the 64 columns of all D_OUT rows of W^T, one TMA box (128-byte swizzle)
    if (tid == 0) {
      mbar_arrive_expect_tx(&b_full[st], (uint32_t)S::B_BYTES);
      tma_load_3d(Bm, &mp.w[m], &b_full[st], f0, 0, 0);
    }
  };

  const uint32_t idesc = umma_idesc_bf16(kTileM, D_OUT, false, false);
  bool ok = true;
  int loaded = 0;   // K blocks whose loads were issued
  for (int kb = 0; kb < nkb + kCmpStages - 1; ++kb) {
    if (kb < nkb) {
      const int st = kb % kCmpStages;
      if (kb >= kCmpStages) {
        if (!mbar_wait(&mma_done[st], ((kb / kCmpStages) - 1) & 1, abort_flag, a.status, 101)) {
          ok = false;
        }
      }
      if (ok) {
        load_stage(st, kb);
        loaded = kb + 1;
      }
    }
    cp_async_commit();
    const int c = kb - (kCmpStages - 1);
    if (c >= 0) {
      cp_async_wait<kCmpStages - 1>();
      fence_proxy_async_smem();
      __syncthreads();
      if (*abort_flag) { ok = false; break; }
      if (tid == 0) {
        const int st = c % kCmpStages;
        if (!mbar_wait(&b_full[st], (c / kCmpStages) & 1, abort_flag, a.status, 104)) ok = false;
      }
      if (__syncthreads_or(!ok)) { ok = false; break; }
      if (tid == 0) {
        tc_fence_after();
        const int st = c % kCmpStages;
        const uint32_t a_addr = smem_u32(smem + st * S::STAGE);
        const uint32_t b_addr = a_addr + S::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t da = umma_desc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t db = umma_desc_sw128(b_addr + kk * 32, 16, 1024);
          umma_ss(tmem_d, da, db, idesc, (c > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&mma_done[st]);
      }
    }
  }
  cp_async_wait<0>();
  // all MMAs done: commit a final barrier (also on the abort path, so that no
  // product is still running when tensor memory is released); the B tiles still
  // in flight land first
  if (tid == 0) {
    for (int v = loaded - kCmpStages < 0 ? 0 : loaded - kCmpStages; v < loaded; ++v)
      mbar_wait_drain(&b_full[v % kCmpStages], (v / kCmpStages) & 1);
    umma_commit(&mma_done[kCmpStages]);
  }
  __syncthreads();
  if (ok && !*abort_flag) ok = mbar_wait(&mma_done[kCmpStages], 0, abort_flag, a.status, 102);
  else if (tid == 0) mbar_wait_drain(&mma_done[kCmpStages], 0);
  tc_fence_after();

  if (ok) {
    // epilogue: warp w owns accumulator rows 32w .. 32w+31 (TMEM lanes)
    const int row = warp * 32 + lane;
    const int ci = i0 + row;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out[m]);
    int64_t oe = a.seqs.cmp_off[b] + ci;   // output row (paged: entry index in the sequence)
    bool oval = true;
    if (a.out_pt.table && ci < ncmp) {
      const int pg = a.out_pt.table[(int64_t)b * a.out_pt.max_pages + (int)(oe / a.out_pt.page_size)];
      oval = pg >= 0 && pg < a.out_pt.n_pages;
      if (!oval) atomicOr(a.status, DEV_ERR_BOUNDS);
      oe = oval ? (int64_t)pg * a.out_pt.page_size + oe % a.out_pt.page_size : 0;
    }
    const size_t orow = ((size_t)oe * a.H_kv + g) * D_OUT;
#pragma unroll 1
    for (int c0 = 0; c0 < D_OUT; c0 += 16) {
      float v[16];
      tmem_ld16(tmem_d + ((uint32_t)(warp * 32) << 16) + c0, v);
      tmem_ld_wait();
      if (ci < ncmp && oval) {
        if (a.ksplit[m] == 1) {
          uint32_t pk[8];
#pragma unroll
          for (int j = 0; j < 8; ++j)
            pk[j] = pack_bf16x2(v[2 * j] + a.bias[m][c0 + 2 * j], v[2 * j + 1] + a.bias[m][c0 + 2 * j + 1]);
          uint4* dst = reinterpret_cast<uint4*>(out + orow + c0);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        } else {
          float4* dst = reinterpret_cast<float4*>(a.part[m] + (size_t)blockIdx.z * a.rows_total * a.H_kv * D_OUT + orow + c0);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem_d, TM_COLS);
}

// keys and values of every KV head in one launch (grid.y = 2 H_kv); a CTA whose
// split index is beyond its map's split count has nothing to do
template <int DK, int DV>
__global__ void __launch_bounds__(128, 1) compress_gemm_kernel(const CompressArgs a,
                                                                const __grid_constant__ CompressMaps mp) {
  const int m = blockIdx.y >= a.H_kv ? 1 : 0;
  if ((int)blockIdx.z >= a.ksplit[m]) return;
  if (m == 0) compress_gemm_body<DK, DK>(a, mp, 0, blockIdx.y);
  else compress_gemm_body<DV, DV>(a, mp, 1, blockIdx.y - a.H_kv);
}

template <int DK, int DV>
static cudaError_t launch_gemm_t(const CompressArgs& a, const CompressMaps& mp, int n_tiles, cudaStream_t st) {
  constexpr int smem = CompressSmem<DK>::TOTAL > CompressSmem<DV>::TOTAL ? CompressSmem<DK>::TOTAL
                                                                        : CompressSmem<DV>::TOTAL;
  auto kern = compress_gemm_kernel<DK, DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(n_tiles, 2 * a.H_kv, a.ksplit[0] > a.ksplit[1] ? a.ksplit[0] : a.ksplit[1]);
  kern<<<grid, 128, smem, st>>>(a, mp);
  return cudaGetLastError();
}

// out[r, :] = bf16(sum_z part[z, r, :] + bias) over the packed output rows of
// both maps (float4 indices [0, n4k) keys, then [n4k, n4k + n4v) values), the
// partial sums added in a fixed order (deterministic)
__global__ void compress_finalize_kernel(const CompressArgs a, int64_t n4k, int64_t n4v, int dk, int dv) {
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // float4 index
  if (i >= n4k + n4v) return;
  const int m = i < n4k ? 0 : 1;
  if (m == 1) i -= n4k;
  const int64_t n4 = m == 0 ? n4k : n4v;
  const int d_out = m == 0 ? dk : dv;
  const float4* part = reinterpret_cast<const float4*>(a.part[m]);
  float4 acc = part[i];
  for (int z = 1; z < a.ksplit[m]; ++z) {
    const float4 v = part[(size_t)z * n4 + i];
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  const int c = (int)((i * 4) % d_out);
  const float* bias = a.bias[m];
  uint2 pk;
  pk.x = pack_bf16x2(acc.x + bias[c], acc.y + bias[c + 1]);
  pk.y = pack_bf16x2(acc.z + bias[c + 2], acc.w + bias[c + 3]);
  reinterpret_cast<uint2*>(a.out[m])[i] = pk;
}

cudaError_t launch_compress_finalize(int d_k, int d_v, const CompressArgs& a, cudaStream_t st) {
  const int64_t n4k = a.ksplit[0] > 1 ? a.rows_total * a.H_kv * d_k / 4 : 0;
  const int64_t n4v = a.ksplit[1] > 1 ? a.rows_total * a.H_kv * d_v / 4 : 0;
  if (n4k + n4v <= 0) return cudaSuccess;
  compress_finalize_kernel<<<(unsigned)((n4k + n4v + 255) / 256), 256, 0, st>>>(a, n4k, n4v, d_k, d_v);
  return cudaGetLastError();
}

cudaError_t launch_compress_gemm(int d_k, int d_v, const CompressArgs& a, const CompressMaps& mp, int n_tiles,
                                 cudaStream_t st) {
  if (n_tiles <= 0) return cudaSuccess;
#define NSA_CMP_CASE(DK, DV) \
  if (d_k == DK && d_v == DV) return launch_gemm_t<DK, DV>(a, mp, n_tiles, st);
  NSA_CMP_CASE(192, 128) NSA_CMP_CASE(64, 64) NSA_CMP_CASE(128, 128) NSA_CMP_CASE(192, 64)
  NSA_CMP_CASE(64, 128) NSA_CMP_CASE(128, 64)
#undef NSA_CMP_CASE
  return cudaErrorInvalidValue;
}

}  // namespace nsa
