// Internal launch interface between the C-ABI host layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nsa {

constexpr int kMaxBatch = 128;

// Opt-in per-kernel timing: CUDA events recorded on the launching stream around
// each launch (see nsa_profile_enable / nsa_profile_read in include/nsa.h).
enum ProfSlot {
  P_COMPRESS_PREP = 0, P_COMPRESS_GEMM, P_PREFILL_ATTN, P_DEC_CMP, P_DEC_FINE, P_BWD_INDEX, P_BWD_QUERY,
  P_BWD_KEYS, P_BWD_COMPRESS, P_DSA_INDEX, P_DSA_TOPK, P_DSA_ATTN, P_COUNT
};
void prof_begin(int slot, cudaStream_t st);
void set_error_detail(const char* msg);   // text returned by nsa_last_error_detail()
int test_fault_site();                    // checking build: site set by nsa_test_set_fault (else 0)
void prof_end(int slot, cudaStream_t st, int launches);

// Per-launch sequence table, passed by value as a kernel parameter.
struct SeqTable {
  int32_t n;                         // sequences
  int32_t tile_prefix[kMaxBatch + 1];// first tile id of each sequence
  int64_t tok_off[kMaxBatch];        // first token row
  int64_t cmp_off[kMaxBatch];        // first compressed row
  int32_t len[kMaxBatch];            // tokens
};

__host__ __device__ inline int n_cmp_of(int L, int l, int s) { return L >= l ? (L - l) / s + 1 : 0; }

// Paged caches: token (or compressed entry) e of sequence b lives in physical page
// table[b * max_pages + e / page_size] at row e % page_size of the pool
// [n_pages * page_size, H_kv, d]. A null table means the contiguous batched
// layout. Page ids outside [0, n_pages) are recorded as DEV_ERR_BOUNDS in the
// status word and replaced by page 0 (the result is then not valid).
struct PageTable {
  const int32_t* table;   // device int32 [B, max_pages] or null
  int page_size, max_pages, n_pages;
};
__device__ __forceinline__ int64_t paged_row(const PageTable& pt, int b, int e, uint32_t* status) {
  int p = pt.table[(int64_t)b * pt.max_pages + e / pt.page_size];
  if (p < 0 || p >= pt.n_pages) {
    atomicOr(status, 2u);   // DEV_ERR_BOUNDS
    p = 0;
  }
  return (int64_t)p * pt.page_size + e % pt.page_size;
}

// ----- compression (block summaries) -----
// Both maps in one launch: index 0 = keys (d = d_k), 1 = values (d = d_v);
// grid.y = 2 H_kv (y < H_kv: keys of KV head y, else values of head y - H_kv).
struct CompressArgs {
  const void* x[2];       // bf16 [*, H_kv, d]
  const void* wt[2];      // bf16 [d, l*d] (W transposed, rounded)
  const float* bias[2];   // fp32 [d] = vec(pe) . W
  void* out[2];           // bf16 [*, H_kv, d]
  int H_kv, l, s;
  int ksplit[2];          // split of the K = l*d reduction over grid.z (1: no split)
  int kb_per_split[2];    // 64-wide K blocks per split
  float* part[2];         // fp32 [ksplit][rows_total][H_kv][d] partial sums (ksplit > 1)
  int64_t rows_total;     // output rows (packed: sum of n_cmp)
  int x_chunks;           // whole groups of s tokens in the x view (0: no view, cp.async rows)
  uint32_t* status;
  // paged caches (x_pt.table non-null): seqs.tok_off / cmp_off are then token and
  // entry indices within sequence b, mapped through the tables
  PageTable x_pt, out_pt;
  SeqTable seqs;
};
cudaError_t launch_compress_prep(const float* w, const float* pe, int K, int N, void* wt_bf16,
                                 float* partial, float* bias, cudaStream_t st);
struct CompressMaps {
  CUtensorMap w[2];   // W^T of both maps: boxes of 64 columns x all d rows (128-byte swizzle)
  CUtensorMap x[2];   // keys / values as (channel, token mod s, token div s): boxes of 64 channels x 128 rows
};
cudaError_t launch_compress_gemm(int d_k, int d_v, const CompressArgs& a, const CompressMaps& mp, int n_tiles,
                                 cudaStream_t st);
cudaError_t launch_compress_finalize(int d_k, int d_v, const CompressArgs& a, cudaStream_t st);

// ----- prefill -----
struct PrefillArgs {
  const void* q;          // bf16 [N, H_q, d_k]
  const void* k;          // bf16 [N, H_kv, d_k]
  const void* v;          // bf16 [N, H_kv, d_v]
  const void* kc;         // bf16 [Nc, H_kv, d_k]
  const void* vc;         // bf16 [Nc, H_kv, d_v]
  const float* gates;     // fp32 [N, H_q, 3]
  float* imp;             // fp32 [N, H_kv, nb_stride]
  int32_t* sel;           // int32 [N, H_kv, top_n]
  void* out;              // bf16 [N, H_q, d_v]
  int H_q, H_kv, G, d_k, d_v;
  int l, s, ls, top_n, window, force_first, force_local;
  int nb_stride;
  int n_stages;           // K ring depth of the fused kernel
  int n_vstages;          // V ring depth
  int imp_smem;           // importance and selections of the query tile kept in shared memory
  int want_imp, want_sel; // caller asked for the importance / selection rows
  float scale_log2;       // softmax scale * log2(e)
  uint32_t* status;
  int fault_site;         // checking build only: injected failure (FAULT_*), 0 = none
  SeqTable seqs;          // tile_prefix counts query tiles of 128/G tokens
};
struct PrefillMaps {
  CUtensorMap k, v, kc, vc;   // boxes of 64 rows x 1 head x 64 elements
  CUtensorMap q;              // box of 128/G tokens x G heads x 64 elements (one query tile)
};
bool prefill_fused_stages(PrefillArgs& a);   // sets the ring depths; false: does not fit
cudaError_t launch_prefill_fused(const PrefillArgs& a, const PrefillMaps& m, int n_tiles, cudaStream_t st);

// ----- decode -----
struct DecodeArgs {
  const void* q;          // bf16 [B, H_q, d_k]
  const void* kcache;     // bf16 [B, Lmax, H_kv, d_k]
  const void* vcache;     // bf16 [B, Lmax, H_kv, d_v]
  const void* kc;         // bf16 [B, Lmax_cmp, H_kv, d_k]
  const void* vc;         // bf16 [B, Lmax_cmp, H_kv, d_v]
  const int32_t* lens;    // int32 [B]
  const float* gates;     // fp32 [B, H_q, 3]
  void* out;              // bf16 [B, H_q, d_v]
  int32_t* sel;           // int32 [B, H_kv, top_n]
  float* imp;             // fp32 [B, H_kv, nb_stride]
  float* part;            // split partials (workspace)
  float* ocmp;            // fp32 [B, H_q, d_v] g_cmp * o_cmp (workspace)
  int B, Lmax, Lmax_cmp, max_len;
  int H_q, H_kv, G, d_k, d_v;
  int l, s, ls, top_n, window, force_first, force_local;
  int nb_stride;
  int n_cmp_chunks;              // D1 splits per (b, g), 512 compressed keys each
  int n_sw_chunks;               // D3 splits per (b, g), 4 blocks of l_sel keys each
  float scale_log2;
  uint32_t* status;
  int fault_site;         // checking build only: injected failure (FAULT_*), 0 = none
  PageTable kv_pt;        // paged raw cache (table null: [B, Lmax] rows)
  PageTable cmp_pt;       // paged compressed cache (table null: [B, Lmax_cmp] rows)
};
struct DecodeMaps {
  CUtensorMap k, v, kc, vc;
  CUtensorMap q;   // q [B, H_q, d_k] with a box of one sequence's G heads
};
// ----- backward (prefill) -----
struct BackwardArgs {
  const void* q;          // bf16 [N, H_q, d_k]
  const void* dout;       // bf16 [N, H_q, d_v]
  const float* gates;     // fp32 [N, H_q, 3]
  const int32_t* sel;     // int32 [N, H_kv, top_n] (the forward's selection)
  float* dq;              // fp32 [N, H_q, d_k]
  float* dk;              // fp32 [N, H_kv, d_k] (zeroed; raw branches add into it, then the compression's share)
  float* dv;              // fp32 [N, H_kv, d_v]
  float* dkc;             // fp32 [Nc, H_kv, d_k] (zeroed; compressed-key pass adds into it)
  float* dvc;             // fp32 [Nc, H_kv, d_v]
  float* dgates;          // fp32 [N, H_q, 3]
  float* lse;             // fp32 [N, H_q, 3] per-branch log-sum-exp (log2 units), gate order
  float* dd;              // fp32 [N, H_q, 3] per-branch <dout, O_b>, gate order
  const int32_t* inv_off; // [n_lists + 1]: list (blk_prefix[b] + j) * H_kv + g
  const int32_t* inv_tok; // tokens (index within the sequence) of every list
  int H_q, H_kv, G, d_k, d_v;
  int l, s, ls, top_n, window;
  int nb_stride;          // selection blocks of the longest sequence
  int tok_chunk;          // key passes: query tokens per CTA (grid.z splits)
  float scale, scale_log2;
  uint32_t* status;
  SeqTable seqs;                        // tile_prefix: query tiles of 8 tokens
  int32_t blk_prefix[kMaxBatch + 1];    // 64-key raw blocks per sequence (prefix)
  int32_t cblk_prefix[kMaxBatch + 1];   // 64-entry compressed tiles per sequence (prefix)
};
struct BackwardMaps {
  CUtensorMap k32, v32, kc32, vc32;     // 32-row boxes (query-side key tiles)
  CUtensorMap k64, v64, kc64, vc64;     // 64-row boxes (key-side resident tiles)
  CUtensorMap qg, dog;                  // one token's G heads of q / dout
};
size_t backward_query_smem(int d_k, int d_v, int nb);
cudaError_t launch_backward_attn(const BackwardArgs& a, const BackwardMaps& m, int q_tiles, int raw_blocks,
                                 int raw_z, int cmp_tiles, int cmp_z, cudaStream_t st);
cudaError_t launch_inverted_index(const BackwardArgs& a, int64_t n_ent, int n_lists, int32_t* cnt, int32_t* off,
                                  int32_t* cur, int32_t* slot, int32_t* tok, cudaStream_t st);
cudaError_t launch_compress_backward(const float* dc, const void* x, const float* W, const float* pe, int d_in,
                                     int d_out, int H_kv, int l, int s, const SeqTable& seqs,
                                     const int32_t* ncmp_prefix, int64_t n_cmp_total, float* dx, float* dW,
                                     float* dpe, float* colsum, cudaStream_t st);

// ----- DSA variant (lightning indexer + token top-k + attention) -----
struct DsaArgs {
  const void* q;          // bf16 [*, H_q, d_k]
  const void* k;          // bf16 rows of the raw keys: token s of a query's sequence at row base + s
  const void* v;
  const void* qi;         // fp8 e4m3 [*, H_I, d_I] (row = the query row)
  const void* ki;         // fp8 e4m3 [*, d_I] (row base + s)
  const float* wi;        // fp32 [*, H_I]
  void* out;              // bf16 [*, H_q, d_v]
  float* scores;          // fp32 [slots, ld_scores] indexer scores of this chunk of queries
  int32_t* idx;           // int32 [slots, top_k] kept tokens (ascending, -1 padded)
  int64_t ld_scores;
  int64_t q0;             // first query of this chunk
  const int32_t* lens;    // decode: device int32 [B] (query b at len - 1, base b * Lmax); null for prefill
  int Lmax, max_len;
  SeqTable seqs;          // prefill: packed sequences (query n = token n)
  int H_q, H_kv, G, H_I, top_k;
  float scale_log2;
  uint32_t* status;
};
cudaError_t launch_dsa(const DsaArgs& a, int n_slots, int max_keys, int d_k, int d_v, int d_i, cudaStream_t st);

size_t decode_partials_floats(const DecodeArgs& a);
cudaError_t launch_decode(const DecodeArgs& a, const DecodeMaps& m, cudaStream_t st);

}  // namespace nsa
