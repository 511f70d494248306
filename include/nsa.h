/*
 * nsa.h — C ABI of libnsa.so: Native Sparse Attention (NSA) forward on one
 * NVIDIA B200 (sm_100a), causal prefill and KV-cache decode.
 *
 * The method (sources, cited by page title and section):
 *   "Native Sparse Attention" lesson, aiengineeringfromscratch.com (Phase 10,
 *   lesson 17), sections "Concept / three parallel branches" and "Compute budget";
 *   "Разреженное внимание — NSA и DSA", ai.flicky.cc (stage 5.5, lesson 02),
 *   section "NSA: три ветви" (equation for o_t), "Ветвь отбора", "Практика".
 *
 * For each query position t and query head h (KV head g = h / G, G = H_q/H_kv):
 *   o_t = g_cmp * Attn(q, K_cmp, V_cmp) + g_slc * Attn(q, K_slc, V_slc)
 *       + g_win * Attn(q, K_win, V_win)
 * where K_cmp/V_cmp are compressed block summaries (blocks of l tokens, stride s),
 * K_slc/V_slc are the raw tokens of the top-n selection blocks (size l') chosen
 * per GQA group from the compressed-attention probabilities, and K_win/V_win are
 * the last w tokens. Softmax scale 1/sqrt(d_k) unless `scale` is set.
 *
 * Conventions shared by every entry point:
 *  - Memory: every pointer argument is DEVICE memory unless its comment says
 *    HOST. The caller allocates and owns all buffers, including the workspace;
 *    the library allocates no memory and keeps no state between calls (except
 *    the opt-in profiler's CUDA events, see nsa_profile_enable).
 *  - Layout: row-major, contiguous, 16-byte aligned base pointers. bf16 is
 *    IEEE bfloat16 (2 bytes); fp32 is IEEE binary32.
 *  - Asynchrony: work is enqueued on `stream` (a cudaStream_t; NULL = legacy
 *    default stream). Returns once enqueued.
 *  - Errors: arguments are validated on the host before anything is launched;
 *    on any error nothing is written and nothing is launched.
 *    NSA_ERR_INVALID_ARG: null/misaligned pointer, non-positive size,
 *    inconsistent lengths. NSA_ERR_UNSUPPORTED: valid but not built (head dims,
 *    group size, block parameters; see below). NSA_ERR_WORKSPACE: ws_bytes below
 *    nsa_workspace_size(). NSA_ERR_CUDA: a CUDA launch or driver call failed.
 *    NSA_ERR_DEVICE_CHECK: returned only by nsa_check_device_status() when a
 *    kernel recorded a failure (a bounded wait ran out).
 *  - Supported: d_k in {64, 128, 192}, d_v in {64, 128}, G in {1, 2, 4, 8, 16},
 *    l_cmp = 32, stride = 16, l_sel = 64, 1 <= top_n <= 32, window >= 1,
 *    force_first + force_local <= top_n, batch <= NSA_MAX_BATCH.
 *  - Workspace: the first 256 bytes hold a device status word and the work
 *    counters of the decode pass (back to 0 at the end of every decode call).
 *    Call nsa_workspace_init() once on a new workspace before its first use.
 *    A workspace serves one call at a time: calls that share one must be
 *    ordered (same stream, or events between streams).
 */
#ifndef NSA_H_
#define NSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define NSA_MAX_BATCH 128

typedef enum {
  NSA_OK = 0,
  NSA_ERR_INVALID_ARG = 1,
  NSA_ERR_UNSUPPORTED = 2,
  NSA_ERR_WORKSPACE = 3,
  NSA_ERR_CUDA = 4,
  NSA_ERR_DEVICE_CHECK = 5
} nsa_status_t;

/* Method parameters (NSA-ru "NSA: три ветви"): compression block l_cmp with
 * stride `stride`; selection block l_sel; top_n selected blocks per GQA group,
 * of which force_first initial blocks and force_local local blocks (the block
 * holding t and the ones just before it) are always taken; sliding window of
 * `window` keys ending at t; scale = softmax scale, 0 means 1/sqrt(d_k). */
typedef struct {
  int32_t l_cmp, stride, l_sel, top_n, window, force_first, force_local;
  float scale;
} nsa_params_t;

/* Head geometry: H_q query heads share H_kv key/value heads (GQA, G = H_q/H_kv). */
typedef struct {
  int32_t H_q, H_kv, d_k, d_v;
} nsa_heads_t;

enum { NSA_OP_COMPRESS = 0, NSA_OP_PREFILL = 1, NSA_OP_DECODE = 2, NSA_OP_BACKWARD = 3 };

/* Bytes of workspace `op` needs. `batch` = number of sequences;
 * `total_tokens` = sum of sequence lengths (prefill; for NSA_OP_COMPRESS it sizes
 * optional room that lets nsa_compress split its reduction across more SMs when
 * the output rows are packed; 0 gives the minimum, which is always valid);
 * `max_len` = longest sequence (prefill) or upper bound of the cache lengths
 * (decode). Returns 0 for invalid arguments. */
size_t nsa_workspace_size(int op, const nsa_heads_t* heads, const nsa_params_t* params,
                          int32_t batch, int64_t total_tokens, int32_t max_len);

/* Zero the workspace header (status word) on `stream`. */
nsa_status_t nsa_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/* Synchronise `stream`, read and clear the device status word. Returns NSA_OK,
 * NSA_ERR_DEVICE_CHECK (a kernel recorded a failed bounded wait; its outputs are
 * not valid) or NSA_ERR_CUDA. */
nsa_status_t nsa_check_device_status(void* workspace, void* stream);

/* Block compression (NSA-ru "Сжатая ветвь"; NSA-lesson "Concept"): for every
 * sequence b and every whole block i (i*stride + l_cmp <= len_b):
 *   k_cmp[i] = sum_{r<l} sum_e (k[i*stride + r, g, e] + pe_k[r, e]) * w_ck[r*d_k + e, :]
 * and the same for v with w_cv, pe_v. The flattened block is token-major.
 * Arithmetic: k, v and W rounded to bf16 once, fp32 accumulation; the position
 * term sum(pe*W) is added in fp32; outputs rounded to bf16.
 *   k        bf16, token t of sequence b at row tok_offset[b] + t: [*, H_kv, d_k]
 *   v        bf16, same rows: [*, H_kv, d_v]
 *   w_ck     fp32 [l_cmp*d_k, d_k];  pe_k fp32 [l_cmp, d_k]
 *   w_cv     fp32 [l_cmp*d_v, d_v];  pe_v fp32 [l_cmp, d_v]
 *   tok_offset HOST int64 [batch]: first row of each sequence in k / v
 *   seq_len    HOST int32 [batch]: tokens of each sequence (>= 0)
 *   cmp_offset HOST int64 [batch]: first output row of each sequence
 *   k_cmp    bf16 out: rows cmp_offset[b] .. + n_cmp(len_b) - 1 of [*, H_kv, d_k]
 *   v_cmp    bf16 out: same rows of [*, H_kv, d_v]
 * n_cmp(L) = (L - l_cmp)/stride + 1 for L >= l_cmp, else 0. Packed prefill uses
 * tok_offset = cu_seqlens[b], cmp_offset = running sum of n_cmp; a batched
 * cache [B, Lmax, H_kv, d] uses tok_offset = b*Lmax, cmp_offset = b*Lmax_cmp. */
nsa_status_t nsa_compress(const void* k, const void* v, const float* w_ck, const float* pe_k,
                          const float* w_cv, const float* pe_v, const int64_t* tok_offset,
                          const int32_t* seq_len, const int64_t* cmp_offset, int32_t batch,
                          const nsa_heads_t* heads, const nsa_params_t* params, void* k_cmp,
                          void* v_cmp, void* workspace, size_t ws_bytes, void* stream);

/* The compression's weights in the form the GEMM reads (NSA-ru "NSA: три
 * ветви", compression branch): W^T of both maps rounded to bf16 and the fp32
 * position terms sum(pe * W). nsa_compress forms them from the fp32 weights on
 * every call; a caller whose weights stay fixed across calls (inference, or
 * training between optimizer steps) forms them once with nsa_compress_prepare
 * and passes them to nsa_compress_prepared, which then runs only the GEMM. The
 * results are identical.
 * nsa_compress_weights_size: bytes of the prepared form (0 for invalid
 * arguments). */
size_t nsa_compress_weights_size(const nsa_heads_t* heads, const nsa_params_t* params);

/* Fill `prepared` (device, 256-byte aligned, prepared_bytes >=
 * nsa_compress_weights_size) from w_ck, pe_k, w_cv, pe_v (the layouts of
 * nsa_compress). The caller owns `prepared`; it holds no pointer to the inputs.
 * NSA_ERR_INVALID_ARG for null or misaligned pointers, NSA_ERR_WORKSPACE when
 * prepared_bytes is too small, NSA_ERR_UNSUPPORTED for head sizes the GEMM is
 * not built for. */
nsa_status_t nsa_compress_prepare(const float* w_ck, const float* pe_k, const float* w_cv, const float* pe_v,
                                  const nsa_heads_t* heads, const nsa_params_t* params, void* prepared,
                                  size_t prepared_bytes, void* stream);

/* nsa_compress with weights from nsa_compress_prepare (same heads and params):
 * the same outputs, arguments and errors, without the per-call conversion. */
nsa_status_t nsa_compress_prepared(const void* k, const void* v, const void* prepared,
                                   const int64_t* tok_offset, const int32_t* seq_len, const int64_t* cmp_offset,
                                   int32_t batch, const nsa_heads_t* heads, const nsa_params_t* params,
                                   void* k_cmp, void* v_cmp, void* workspace, size_t ws_bytes, void* stream);

/* Incremental decode (NSA-ru "NSA: три ветви", compression branch: a summary
 * exists for every whole block of l_cmp tokens at stride `stride`; the cache
 * grows one token, or several, at a time). When sequence b of a batched cache
 * [batch, Lmax, H_kv, d] grows from lens_prev[b] to lens[b] tokens, the blocks
 * i with n_cmp(lens_prev[b]) <= i < n_cmp(lens[b]) are completed; their tokens
 * form one segment starting at row b*Lmax + i0*stride. HOST-only planning:
 *   lens_prev  HOST int32 [batch] or NULL (NULL: lens[b] - 1, one new token)
 *   lens       HOST int32 [batch], lens_prev[b] <= lens[b] <= Lmax
 *   tok_offset, seq_len, cmp_offset  HOST out [batch]: the arguments of the
 *              nsa_compress call that writes the new summaries into rows
 *              b*Lmax_cmp + i of a compressed cache [batch, Lmax_cmp, H_kv, d]
 *              (seq_len 0 for sequences that completed no block)
 *   n_blocks   HOST out or NULL: number of summaries to write
 * NSA_ERR_INVALID_ARG for inconsistent lengths or Lmax_cmp < n_cmp(Lmax). Any
 * l_cmp that is a multiple of `stride` is planned (only `l_cmp`, `stride` of
 * params are read); nsa_compress_append checks what the kernels support. */
nsa_status_t nsa_compress_append_plan(const int32_t* lens_prev, const int32_t* lens, int32_t batch, int32_t Lmax,
                                      int32_t Lmax_cmp, const nsa_params_t* params, int64_t* tok_offset,
                                      int32_t* seq_len, int64_t* cmp_offset, int32_t* n_blocks);

/* Plans as nsa_compress_append_plan and writes the new summaries in place with
 * one nsa_compress call on `stream` (no launch when no block was completed).
 * k_cache/v_cache: bf16 [batch, Lmax, H_kv, d_k / d_v]; k_cmp_cache/v_cmp_cache:
 * bf16 [batch, Lmax_cmp, H_kv, d_k / d_v]; n_blocks: HOST out or NULL. The
 * workspace is that of nsa_compress (nsa_workspace_size(NSA_OP_COMPRESS, ...,
 * batch, 0, 0) suffices). */
nsa_status_t nsa_compress_append(const void* k_cache, const void* v_cache, const float* w_ck, const float* pe_k,
                                 const float* w_cv, const float* pe_v, const int32_t* lens_prev, const int32_t* lens,
                                 int32_t batch, int32_t Lmax, int32_t Lmax_cmp, const nsa_heads_t* heads,
                                 const nsa_params_t* params, void* k_cmp_cache, void* v_cmp_cache,
                                 int32_t* n_blocks, void* workspace, size_t ws_bytes, void* stream);

/* nsa_compress without a workspace argument, for callers that cannot allocate
 * device memory where they compress: code that runs while a CUDA graph is being
 * captured, engines that fix their memory plan ahead of time and forbid
 * allocation on the serving path, plugins inside a framework that owns every
 * device allocation. There is no counterpart in the pages describing NSA: this
 * is an interface convenience. Same arguments, layouts, arithmetic and results
 * as nsa_compress, minus workspace/ws_bytes.
 *  - Scratch: a file-scope device array of NSA_NOALLOC_SCRATCH_BYTES (4 MiB)
 *    inside libnsa.so; every GPU that loads the library keeps it reserved until
 *    the process exits. Calls that would need more scratch than that return
 *    NSA_ERR_WORKSPACE (with a message in nsa_last_error_detail()); no supported
 *    head size needs more (d_k = 192, d_v = 128 needs 3.6 MB).
 *  - Allocates nothing: no cudaMalloc/cudaFree or allocating library call.
 *  - Set-up: the first call on a device looks up the array's device address for
 *    the current device (cudaGetSymbolAddress); make that first call before any
 *    stream capture.
 *  - Sharing: every call on a device uses the same array, which keeps the last
 *    call's contents (each call clears the status word it needs zeroed). Calls
 *    whose work overlaps on the GPU (different streams, or different host
 *    threads) race on the array and must be serialised by the caller.
 *  - Device errors: nsa_check_device_status() does not apply (the status word
 *    is inside the array); nsa_noalloc_check_status() reads and clears it. */
#define NSA_NOALLOC_SCRATCH_BYTES 4194304
nsa_status_t nsa_compress_noalloc(const void* k, const void* v, const float* w_ck, const float* pe_k,
                                  const float* w_cv, const float* pe_v, const int64_t* tok_offset,
                                  const int32_t* seq_len, const int64_t* cmp_offset, int32_t batch,
                                  const nsa_heads_t* heads, const nsa_params_t* params, void* k_cmp,
                                  void* v_cmp, void* stream);

/* The status word of nsa_compress_noalloc's built-in scratch on the current
 * device: synchronises `stream`, reads the word and clears it. Returns NSA_OK,
 * NSA_ERR_DEVICE_CHECK (a kernel of the last call on this device recorded a
 * failed bounded wait or index check; its outputs are not valid) or
 * NSA_ERR_CUDA. It synchronises, so it cannot run during stream capture; call
 * it after the captured work has run. Allocates nothing. */
nsa_status_t nsa_noalloc_check_status(void* stream);

/* Causal NSA prefill over packed variable-length sequences (NSA-ru "NSA: три
 * ветви"; NSA-lesson "Concept"). Positions restart at 0 in every sequence.
 *   q        bf16 [N, H_q, d_k], N = cu_seqlens[batch]
 *   k, v     bf16 [N, H_kv, d_k], [N, H_kv, d_v]
 *   k_cmp, v_cmp bf16 [sum_b n_cmp(len_b), H_kv, d_k / d_v], packed in sequence
 *            order (as written by nsa_compress with cmp_offset = running sum)
 *   gates    fp32 [N, H_q, 3] in the order (cmp, slc, win)
 *   cu_seqlens HOST int32 [batch + 1], non-decreasing, cu_seqlens[0] = 0
 *   out      bf16 out [N, H_q, d_v]
 *   sel_out  int32 out or NULL: [N, H_kv, top_n] selected block indices per
 *            (token, KV head), ascending, padded with -1
 *   imp_out  fp32 out or NULL: [N, H_kv, n_blk(max_len)] selection-block
 *            importance (entries beyond the token's own block are unspecified)
 * The workspace (nsa_workspace_size(NSA_OP_PREFILL, ...)) must not overlap any
 * argument. Selection ties go to the lower block index. */
nsa_status_t nsa_prefill(const void* q, const void* k, const void* v, const void* k_cmp,
                         const void* v_cmp, const float* gates, const int32_t* cu_seqlens,
                         int32_t batch, const nsa_heads_t* heads, const nsa_params_t* params,
                         void* out, int32_t* sel_out, float* imp_out, void* workspace,
                         size_t ws_bytes, void* stream);

/* NSA decode: one new query per sequence against a KV cache that already holds
 * the new token, so the query sits at position cache_lens[b] - 1.
 *   q            bf16 [batch, H_q, d_k]
 *   k_cache      bf16 [batch, Lmax, H_kv, d_k];  v_cache bf16 [batch, Lmax, H_kv, d_v]
 *   k_cmp_cache  bf16 [batch, Lmax_cmp, H_kv, d_k]; v_cmp_cache likewise with d_v;
 *                entries 0 .. n_cmp(cache_lens[b]) - 1 must be valid
 *   cache_lens   DEVICE int32 [batch], 1 <= cache_lens[b] <= max_len <= Lmax
 *   gates        fp32 [batch, H_q, 3] (cmp, slc, win)
 *   out          bf16 out [batch, H_q, d_v]
 *   sel_out      int32 out or NULL: [batch, H_kv, top_n], ascending, -1 padded
 *   imp_out      fp32 out or NULL: [batch, H_kv, n_blk(max_len)]
 * `max_len` (HOST) bounds the lengths and sizes the launch; lengths above it
 * are an error recorded in the device status word (the sequence is skipped).
 * max_len above 262144 tokens returns NSA_ERR_UNSUPPORTED. */
nsa_status_t nsa_decode(const void* q, const void* k_cache, const void* v_cache,
                        const void* k_cmp_cache, const void* v_cmp_cache,
                        const int32_t* cache_lens, int32_t batch, int32_t Lmax, int32_t Lmax_cmp,
                        int32_t max_len, const float* gates, const nsa_heads_t* heads,
                        const nsa_params_t* params, void* out, int32_t* sel_out, float* imp_out,
                        void* workspace, size_t ws_bytes, void* stream);

/* Paged KV cache (the same decode as nsa_decode; NSA-lesson introduction: at
 * long context decode is dominated by reading the KV cache, which serving
 * systems keep in fixed-size pages). Raw keys/values live in pools of pages:
 *   k_pool       bf16 [n_pages, page_size, H_kv, d_k]; v_pool likewise with d_v
 *   block_table  DEVICE int32 [batch, max_pages]: token t of sequence b is row
 *                t % page_size of page block_table[b][t / page_size]
 * and the compressed summaries in pools of their own pages:
 *   k_cmp_pool   bf16 [n_cmp_pages, cmp_page_size, H_kv, d_k]; v_cmp_pool with d_v
 *   cmp_block_table DEVICE int32 [batch, max_cmp_pages]: summary i of sequence b
 *                is row i % cmp_page_size of page cmp_block_table[b][i / cmp_page_size]
 * page_size must be a multiple of 64 (a selection block and a 32-key tile never
 * straddle pages) and cmp_page_size a multiple of 32 (nor does a tile of 32
 * summaries). Only the pages a sequence's length reaches are read. Page ids
 * outside [0, n_pages) are recorded in the status word (nsa_check_device_status
 * then reports NSA_ERR_DEVICE_CHECK) and read as page 0. Other arguments as in
 * nsa_decode; max_len <= max_pages * page_size. Results are identical to
 * nsa_decode on the same contents laid out contiguously. */
nsa_status_t nsa_decode_paged(const void* q, const void* k_pool, const void* v_pool, int32_t n_pages,
                              int32_t page_size, const int32_t* block_table, int32_t max_pages,
                              const void* k_cmp_pool, const void* v_cmp_pool, int32_t n_cmp_pages,
                              int32_t cmp_page_size, const int32_t* cmp_block_table, int32_t max_cmp_pages,
                              const int32_t* cache_lens, int32_t batch, int32_t max_len, const float* gates,
                              const nsa_heads_t* heads, const nsa_params_t* params, void* out, int32_t* sel_out,
                              float* imp_out, void* workspace, size_t ws_bytes, void* stream);

/* Compression into paged caches (layouts as in nsa_decode_paged): writes the
 * summaries of the blocks completed while the sequences grew from lens_prev to
 * lens tokens (HOST int32 [batch]; lens_prev NULL means lens - 1; all zeros
 * builds the whole compressed cache), reading the raw tokens through
 * block_table and writing through cmp_block_table. n_blocks: HOST out or NULL.
 * Results are identical to nsa_compress on the same contents laid out
 * contiguously. Invalid page ids are recorded in the status word (the rows they
 * would read are taken as zeros, the rows they would write are skipped). */
nsa_status_t nsa_compress_paged(const void* k_pool, const void* v_pool, int32_t n_pages, int32_t page_size,
                                const int32_t* block_table, int32_t max_pages, const float* w_ck, const float* pe_k,
                                const float* w_cv, const float* pe_v, const int32_t* lens_prev, const int32_t* lens,
                                int32_t batch, void* k_cmp_pool, void* v_cmp_pool, int32_t n_cmp_pages,
                                int32_t cmp_page_size, const int32_t* cmp_block_table, int32_t max_cmp_pages,
                                const nsa_heads_t* heads, const nsa_params_t* params, int32_t* n_blocks,
                                void* workspace, size_t ws_bytes, void* stream);

/* Backward of the causal NSA prefill ("Native Sparse Attention" lesson, section
 * on native trainability: the top-n step is not differentiable and only decides
 * which blocks are loaded; gradients flow through the compressed branch and the
 * selected and window contributions). Gradients of L with dL/dout = dout with the
 * selection held at `sel` (the forward's sel_out):
 *   q, k, v, k_cmp, v_cmp, gates, cu_seqlens (HOST), batch, heads, params:
 *            as given to nsa_compress / nsa_prefill (k_cmp/v_cmp its outputs)
 *   dout     bf16 [N, H_q, d_v]
 *   sel      int32 [N, H_kv, top_n], ascending, -1 padded (nsa_prefill sel_out)
 *   w_ck, pe_k, w_cv, pe_v: the compression weights given to nsa_compress
 *   dq       fp32 out [N, H_q, d_k];   dk fp32 out [N, H_kv, d_k]; dv [N, H_kv, d_v]
 *   dgates   fp32 out [N, H_q, 3] (cmp, slc, win)
 *   dw_ck, dw_cv  fp32 out [l_cmp*d, d];  dpe_k, dpe_v fp32 out [l_cmp, d]
 * dk/dv include the compressed branch's share through the compression. The
 * compressed-key gradients and dW are accumulated with atomic additions, so the
 * low-order bits of dk, dv and dW may differ between calls. Workspace:
 * nsa_workspace_size(NSA_OP_BACKWARD, heads, params, batch, N, max_len). */
nsa_status_t nsa_prefill_backward(const void* q, const void* k, const void* v, const void* k_cmp,
                                  const void* v_cmp, const float* gates, const void* dout, const int32_t* sel,
                                  const float* w_ck, const float* pe_k, const float* w_cv, const float* pe_v,
                                  const int32_t* cu_seqlens, int32_t batch, const nsa_heads_t* heads,
                                  const nsa_params_t* params, float* dq, float* dk, float* dv, float* dgates,
                                  float* dw_ck, float* dpe_k, float* dw_cv, float* dpe_v, void* workspace,
                                  size_t ws_bytes, void* stream);

/* DSA variant ("Разреженное внимание — NSA и DSA", section "DSA: молниеносный
 * индексатор"): a lightning indexer scores every past token s <= t of query t,
 *   I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s])   (H_I heads of size d_I, FP8)
 * the top_k tokens by I are kept (ties to the lower index; every token when
 * t + 1 <= top_k) and each query head attends to the raw keys/values of the kept
 * tokens (GQA: head h uses KV head h / G; scale as in nsa_params_t; one
 * selection serves all heads). Supported: H_I <= 16, d_I in {32, 64, 128},
 * top_k <= 65536, the head dims of the NSA entry points. */
typedef struct {
  int32_t H_I, d_I, top_k;
  float scale;   /* 0 => 1/sqrt(d_k) */
} nsa_dsa_params_t;

enum { NSA_OP_DSA_DECODE = 4, NSA_OP_DSA_PREFILL = 5 };

/* Workspace bytes of nsa_dsa_decode (batch sequences, caches up to max_len) or
 * nsa_dsa_prefill (total_tokens packed tokens, longest sequence max_len; the
 * queries run in chunks whose score rows fill at most 2^26 floats). 0 for
 * invalid arguments. */
size_t nsa_dsa_workspace_size(int op, const nsa_heads_t* heads, const nsa_dsa_params_t* dsa, int32_t batch,
                              int64_t total_tokens, int32_t max_len);

/* DSA decode: one query per sequence at position cache_lens[b] - 1.
 *   q          bf16 [batch, H_q, d_k]
 *   k_cache    bf16 [batch, Lmax, H_kv, d_k]; v_cache bf16 [batch, Lmax, H_kv, d_v]
 *   qi         fp8 e4m3 [batch, H_I, d_I];  wi fp32 [batch, H_I]
 *   ki_cache   fp8 e4m3 [batch, Lmax, d_I] (the indexer's key of every cached token)
 *   cache_lens DEVICE int32 [batch], 1 <= len <= max_len <= Lmax (others are
 *              recorded in the status word and skipped)
 *   out        bf16 out [batch, H_q, d_v]
 *   idx_out    int32 out or NULL: [batch, top_k] kept tokens, ascending, -1 padded
 *   score_out  fp32 out or NULL: [batch, max_len] indexer scores (entries past the
 *              query's own position are unspecified) */
nsa_status_t nsa_dsa_decode(const void* q, const void* k_cache, const void* v_cache, const void* qi, const float* wi,
                            const void* ki_cache, const int32_t* cache_lens, int32_t batch, int32_t Lmax,
                            int32_t max_len, const nsa_dsa_params_t* dsa, const nsa_heads_t* heads, void* out,
                            int32_t* idx_out, float* score_out, void* workspace, size_t ws_bytes, void* stream);

/* DSA causal prefill over packed sequences (positions restart at 0 per sequence).
 *   q bf16 [N, H_q, d_k]; k, v bf16 [N, H_kv, d_k / d_v]; qi fp8 [N, H_I, d_I];
 *   wi fp32 [N, H_I]; ki fp8 [N, d_I]; cu_seqlens HOST int32 [batch + 1];
 *   out bf16 out [N, H_q, d_v]; idx_out int32 out or NULL [N, top_k];
 *   score_out fp32 out or NULL [N, max_len] (max_len = longest sequence). */
nsa_status_t nsa_dsa_prefill(const void* q, const void* k, const void* v, const void* qi, const float* wi,
                             const void* ki, const int32_t* cu_seqlens, int32_t batch, const nsa_dsa_params_t* dsa,
                             const nsa_heads_t* heads, void* out, int32_t* idx_out, float* score_out,
                             void* workspace, size_t ws_bytes, void* stream);

/* Opt-in per-kernel timing (no compute change). While enabled, every entry point
 * records a CUDA event pair on its stream around each of its kernel launches.
 * nsa_profile_read() waits for the recorded events, writes for each of the
 * first n_slots kernel slots the accumulated milliseconds and launch count since
 * the previous read, and resets them. Slot names: nsa_profile_slot_name(). The
 * events are created on first use and reused; this is the only state the
 * library keeps between calls. Returns NSA_ERR_CUDA if an event query fails. */
#define NSA_PROFILE_SLOTS 12
nsa_status_t nsa_profile_enable(int32_t enable);
nsa_status_t nsa_profile_read(double* ms_out, int64_t* launches_out, int32_t n_slots);
const char* nsa_profile_slot_name(int32_t slot);

/* Human-readable name of a status code (static string). */
const char* nsa_status_string(nsa_status_t status);

/* Text of the last CUDA error seen by this thread's calls (static per thread). */
const char* nsa_last_error_detail(void);

#ifdef __cplusplus
}
#endif

#endif /* NSA_H_ */
