// C-ABI host layer of libnsa.so: argument validation, workspace carving,
// tensor-map encoding and the launch sequence of each entry point.
// See include/nsa.h for the contract of every function.
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/nsa.h"
#include "common.cuh"
#include "kernels.h"

using namespace nsa;

namespace {

thread_local char g_detail[256] = "";

nsa_status_t cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_detail, sizeof(g_detail), "%s: %s", where, cudaGetErrorString(e));
  return NSA_ERR_CUDA;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool heads_supported(const nsa_heads_t* h) {
  const int G = h->H_kv > 0 ? h->H_q / h->H_kv : 0;
  const bool dk = h->d_k == 64 || h->d_k == 128 || h->d_k == 192;
  const bool dv = h->d_v == 64 || h->d_v == 128;
  const bool g = G == 1 || G == 2 || G == 4 || G == 8 || G == 16;
  return dk && dv && g;
}

nsa_status_t check_heads(const nsa_heads_t* h) {
  if (!h || h->H_q <= 0 || h->H_kv <= 0 || h->d_k <= 0 || h->d_v <= 0) return NSA_ERR_INVALID_ARG;
  if (h->H_q % h->H_kv != 0) return NSA_ERR_INVALID_ARG;
  if (!heads_supported(h)) return NSA_ERR_UNSUPPORTED;
  return NSA_OK;
}

nsa_status_t check_params(const nsa_params_t* p, bool need_selection) {
  if (!p) return NSA_ERR_INVALID_ARG;
  if (p->l_cmp <= 0 || p->stride <= 0 || p->l_sel <= 0) return NSA_ERR_INVALID_ARG;
  if (p->l_cmp % p->stride != 0 || p->l_sel % p->stride != 0) return NSA_ERR_INVALID_ARG;
  if (!(p->scale >= 0.f)) return NSA_ERR_INVALID_ARG;
  if (need_selection) {
    if (p->top_n <= 0 || p->window <= 0 || p->force_first < 0 || p->force_local < 0)
      return NSA_ERR_INVALID_ARG;
    if (p->force_first + p->force_local > p->top_n) return NSA_ERR_INVALID_ARG;
    if (p->top_n > 32) return NSA_ERR_UNSUPPORTED;
  }
  if (p->l_cmp != 32 || p->stride != 16 || (need_selection && p->l_sel != 64))
    return NSA_ERR_UNSUPPORTED;
  return NSA_OK;
}

// blocks of the decode fine pass: the selected ones plus those the window touches
int max_union_blocks(const nsa_params_t* p) { return p->top_n + (p->window + p->l_sel - 1) / p->l_sel + 1; }

float softmax_scale(const nsa_params_t* p, int d_k) {
  return p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)d_k);
}

int n_blk_of(int L, int ls) { return (L + ls - 1) / ls; }

// ---- workspace layouts ----
constexpr int kMaxKSplit = 4;   // more splits cost more in partial sums than they gain in CTAs
struct CompressWs {
  size_t wt_k, wt_v, part_k, part_v, bias_k, bias_v, ksum, total;
};
// `rows` bounds the packed compressed rows; it sizes the split-K partial sums
// (none when 0). Everything before `ksum` is the fixed minimum.
CompressWs compress_ws(const nsa_heads_t* h, const nsa_params_t* p, int64_t rows) {
  CompressWs w{};
  size_t off = 256;
  const size_t Kk = (size_t)p->l_cmp * h->d_k, Kv = (size_t)p->l_cmp * h->d_v;
  w.wt_k = off; off = align256(off + Kk * h->d_k * 2);
  w.wt_v = off; off = align256(off + Kv * h->d_v * 2);
  w.part_k = off; off = align256(off + ((Kk + 31) / 32) * h->d_k * 4);
  w.part_v = off; off = align256(off + ((Kv + 31) / 32) * h->d_v * 4);
  w.bias_k = off; off = align256(off + (size_t)h->d_k * 4);
  w.bias_v = off; off = align256(off + (size_t)h->d_v * 4);
  w.ksum = off;   // split-K partial sums of both maps: [ksplit][rows][H_kv][d_k], then the same with d_v
  if (rows > 0) off = align256(off + (size_t)kMaxKSplit * (size_t)rows * h->H_kv * (h->d_k + h->d_v) * 4);
  w.total = off;
  return w;
}

struct PrefillWs {
  size_t imp, sel, total;
  int nb;
};
PrefillWs prefill_ws(const nsa_heads_t* h, const nsa_params_t* p, int64_t N, int max_len) {
  PrefillWs w{};
  size_t off = 256;
  w.nb = n_blk_of(max_len, p->l_sel);
  w.imp = off; off = align256(off + (size_t)N * h->H_kv * w.nb * 4);
  w.sel = off; off = align256(off + (size_t)N * h->H_kv * p->top_n * 4);
  w.total = off;
  return w;
}

// backward workspace: per-branch lse and <dout, O_b>, fp32 gradients of the
// compressed keys/values, the inverted selection index, column sums
struct BackwardWs {
  size_t lse, dd, dkc, dvc, cnt, off, cur, slot, tok, colsum, total;
  int64_t n_lists, n_ent, ncmp;
};
BackwardWs backward_ws(const nsa_heads_t* h, const nsa_params_t* p, int batch, int64_t N, int64_t ncmp,
                       int64_t nblk) {
  BackwardWs w{};
  w.n_lists = nblk * h->H_kv;
  w.n_ent = N * h->H_kv * p->top_n;
  w.ncmp = ncmp;
  size_t off = 256;
  w.lse = off; off = align256(off + (size_t)N * h->H_q * 3 * 4);
  w.dd = off; off = align256(off + (size_t)N * h->H_q * 3 * 4);
  w.dkc = off; off = align256(off + (size_t)ncmp * h->H_kv * h->d_k * 4);
  w.dvc = off; off = align256(off + (size_t)ncmp * h->H_kv * h->d_v * 4);
  w.cnt = off; off = align256(off + (size_t)w.n_lists * 4);
  w.off = off; off = align256(off + (size_t)(w.n_lists + 1) * 4);
  w.cur = off; off = align256(off + (size_t)w.n_lists * 4);
  w.slot = off; off = align256(off + (size_t)w.n_ent * 4);
  w.tok = off; off = align256(off + (size_t)w.n_ent * 4);
  w.colsum = off; off = align256(off + 256 * 4);
  w.total = off;
  (void)batch;
  return w;
}

void fill_decode_args(DecodeArgs& a, const nsa_heads_t* h, const nsa_params_t* p, int B, int Lmax,
                      int Lmax_cmp, int max_len) {
  a.B = B; a.Lmax = Lmax; a.Lmax_cmp = Lmax_cmp; a.max_len = max_len;
  a.H_q = h->H_q; a.H_kv = h->H_kv; a.G = h->H_q / h->H_kv; a.d_k = h->d_k; a.d_v = h->d_v;
  a.l = p->l_cmp; a.s = p->stride; a.ls = p->l_sel; a.top_n = p->top_n; a.window = p->window;
  a.force_first = p->force_first; a.force_local = p->force_local;
  a.nb_stride = n_blk_of(max_len, p->l_sel);
  a.n_cmp_chunks = (n_cmp_of(max_len, p->l_cmp, p->stride) + 511) / 512;
  if (a.n_cmp_chunks < 1) a.n_cmp_chunks = 1;
  a.n_sw_chunks = (max_union_blocks(p) + 3) / 4;
  a.scale_log2 = softmax_scale(p, h->d_k) * 1.4426950408889634f;
}

struct DecodeWs {
  size_t part, ocmp, sel, imp, total;
};
DecodeWs decode_ws(const DecodeArgs& a) {
  DecodeWs w{};
  size_t off = 256;
  w.part = off; off = align256(off + decode_partials_floats(a) * 4);
  w.ocmp = off; off = align256(off + (size_t)a.B * a.H_q * a.d_v * 4);
  w.sel = off; off = align256(off + (size_t)a.B * a.H_kv * a.top_n * 4);
  w.imp = off; off = align256(off + (size_t)a.B * a.H_kv * a.nb_stride * 4);
  w.total = off;
  return w;
}

// ---- tensor maps ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D bf16 map over a [rows, heads, dim] tensor; box = (64 elements, bh heads, br rows),
// 128-byte swizzle. Coordinates: (element, head, row).
bool make_map_3d(CUtensorMap* m, const void* base, int dim, int heads, int64_t rows, int bh, int br) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t gdim[3] = {(cuuint64_t)dim, (cuuint64_t)heads, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t gstride[2] = {(cuuint64_t)dim * 2, (cuuint64_t)dim * heads * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)bh, (cuuint32_t)br};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstride, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The packed tokens [rows, heads, dim] viewed as (channel, token mod s, token
// div s) over the first `chunks` whole groups of s tokens: a box of 64 channels
// x 1 x 128 groups holds 128 rows that start s tokens apart (128-byte swizzle).
bool make_map_xview(CUtensorMap* m, const void* base, int dim, int heads, int s, int64_t chunks) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t c = (cuuint64_t)dim * heads;
  cuuint64_t gdim[3] = {c, (cuuint64_t)s, (cuuint64_t)chunks};
  cuuint64_t gstride[2] = {c * 2, c * 2 * (cuuint64_t)s};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstride, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---- opt-in profiler ----
struct ProfRec {
  int slot, launches;
  cudaEvent_t a, b;
};
struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> pool;
  std::vector<ProfRec> recs;
  cudaEvent_t open[P_COUNT] = {};
  double total_ms[P_COUNT] = {};
  int64_t launches[P_COUNT] = {};
  cudaEvent_t get() {
    if (!pool.empty()) { cudaEvent_t e = pool.back(); pool.pop_back(); return e; }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
};
Profiler& prof() {
  static Profiler p;
  return p;
}

const char* kSlotNames[P_COUNT] = {"compress_prep", "compress_gemm", "prefill_attn", "dec_cmp", "dec_fine",
                                   "bwd_index", "bwd_query", "bwd_keys", "bwd_compress", "dsa_index", "dsa_topk",
                                   "dsa_attn"};

}  // namespace

namespace nsa {
void set_error_detail(const char* msg) { snprintf(g_detail, sizeof(g_detail), "%s", msg); }

#ifdef NSA_FAULT_INJECT
static int g_test_fault = 0;
int test_fault_site() { return g_test_fault; }
#else
int test_fault_site() { return 0; }
#endif

void prof_begin(int slot, cudaStream_t st) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (!p.on) return;
  cudaEvent_t e = p.get();
  cudaEventRecord(e, st);
  p.open[slot] = e;
}
void prof_end(int slot, cudaStream_t st, int launches) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (!p.on || !p.open[slot]) return;
  cudaEvent_t e = p.get();
  cudaEventRecord(e, st);
  p.recs.push_back({slot, launches, p.open[slot], e});
  p.open[slot] = nullptr;
}
}  // namespace nsa

extern "C" {

#ifdef NSA_FAULT_INJECT
nsa_status_t nsa_test_set_fault(int32_t site) {
  if (site < FAULT_NONE || site > FAULT_PREFILL_K_TILE) return NSA_ERR_INVALID_ARG;
  nsa::g_test_fault = site;
  return NSA_OK;
}
#endif

nsa_status_t nsa_profile_enable(int32_t enable) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  p.on = enable != 0;
  return NSA_OK;
}

nsa_status_t nsa_profile_read(double* ms_out, int64_t* launches_out, int32_t n_slots) {
  if (n_slots < 0 || (n_slots > 0 && (!ms_out || !launches_out))) return NSA_ERR_INVALID_ARG;
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  for (const ProfRec& r : p.recs) {
    float ms = 0.f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess) return cuda_fail(e, "nsa_profile_read");
    p.total_ms[r.slot] += ms;
    p.launches[r.slot] += r.launches;
    p.pool.push_back(r.a);
    p.pool.push_back(r.b);
  }
  p.recs.clear();
  for (int i = 0; i < n_slots; ++i) {
    ms_out[i] = i < P_COUNT ? p.total_ms[i] : 0.0;
    launches_out[i] = i < P_COUNT ? p.launches[i] : 0;
  }
  for (int i = 0; i < P_COUNT; ++i) { p.total_ms[i] = 0.0; p.launches[i] = 0; }
  return NSA_OK;
}

const char* nsa_profile_slot_name(int32_t slot) {
  return (slot >= 0 && slot < P_COUNT) ? kSlotNames[slot] : "";
}


const char* nsa_status_string(nsa_status_t s) {
  switch (s) {
    case NSA_OK: return "NSA_OK";
    case NSA_ERR_INVALID_ARG: return "NSA_ERR_INVALID_ARG";
    case NSA_ERR_UNSUPPORTED: return "NSA_ERR_UNSUPPORTED";
    case NSA_ERR_WORKSPACE: return "NSA_ERR_WORKSPACE";
    case NSA_ERR_CUDA: return "NSA_ERR_CUDA";
    case NSA_ERR_DEVICE_CHECK: return "NSA_ERR_DEVICE_CHECK";
  }
  return "NSA_UNKNOWN_STATUS";
}

const char* nsa_last_error_detail(void) { return g_detail; }

size_t nsa_workspace_size(int op, const nsa_heads_t* heads, const nsa_params_t* params, int32_t batch,
                          int64_t total_tokens, int32_t max_len) {
  if (check_heads(heads) != NSA_OK) return 0;
  if (batch <= 0 || batch > NSA_MAX_BATCH) return 0;
  switch (op) {
    case NSA_OP_COMPRESS: {
      if (check_params(params, false) != NSA_OK || total_tokens < 0) return 0;
      // packed rows are at most total_tokens / stride (+1 per sequence)
      const int64_t rows = total_tokens > 0 ? total_tokens / params->stride + batch : 0;
      return compress_ws(heads, params, rows).total;
    }
    case NSA_OP_PREFILL:
      if (check_params(params, true) != NSA_OK || total_tokens < 0 || max_len < 0) return 0;
      return prefill_ws(heads, params, total_tokens, max_len).total;
    case NSA_OP_BACKWARD: {
      if (check_params(params, true) != NSA_OK || total_tokens < 0) return 0;
      // bounds of the packed compressed rows and selection blocks of any split
      // of total_tokens into `batch` sequences
      const int64_t ncmp = total_tokens / params->stride + batch;
      const int64_t nblk = total_tokens / params->l_sel + batch;
      return backward_ws(heads, params, batch, total_tokens, ncmp, nblk).total;
    }
    case NSA_OP_DECODE: {
      if (check_params(params, true) != NSA_OK || max_len <= 0 || max_union_blocks(params) > 64) return 0;
      DecodeArgs a{};
      fill_decode_args(a, heads, params, batch, max_len, n_cmp_of(max_len, params->l_cmp, params->stride),
                       max_len);
      if (a.n_cmp_chunks > 32) return 0;
      return decode_ws(a).total;
    }
  }
  return 0;
}

nsa_status_t nsa_workspace_init(void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace || ws_bytes < 256 || !aligned16(workspace)) return NSA_ERR_INVALID_ARG;
  cudaError_t e = cudaMemsetAsync(workspace, 0, 256, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NSA_OK : cuda_fail(e, "nsa_workspace_init");
}

nsa_status_t nsa_check_device_status(void* workspace, void* stream) {
  if (!workspace) return NSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t h[2] = {0, 0};
  cudaError_t e = cudaMemcpyAsync(h, workspace, sizeof(h), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "nsa_check_device_status");
  if (h[0] != 0) {
    snprintf(g_detail, sizeof(g_detail), "device status 0x%x at site %u", h[0], h[1]);
    e = cudaMemsetAsync(workspace, 0, 256, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "nsa_check_device_status(clear)");
    return NSA_ERR_DEVICE_CHECK;
  }
  return NSA_OK;
}

}  // extern "C"

namespace {
// bf16 W^T and the position terms of both maps at base + (the offsets of w) - shift
// (shift 0: a workspace; 256: a prepared blob, which has no workspace header)
cudaError_t prepare_weights(const float* w_ck, const float* pe_k, const float* w_cv, const float* pe_v,
                            const nsa_heads_t* heads, const nsa_params_t* params, uint8_t* base, size_t shift,
                            const CompressWs& w, cudaStream_t st) {
  const int Kk = params->l_cmp * heads->d_k, Kv = params->l_cmp * heads->d_v;
  cudaError_t e = launch_compress_prep(w_ck, pe_k, Kk, heads->d_k, base + (w.wt_k - shift),
                                       (float*)(base + (w.part_k - shift)), (float*)(base + (w.bias_k - shift)), st);
  if (e == cudaSuccess)
    e = launch_compress_prep(w_cv, pe_v, Kv, heads->d_v, base + (w.wt_v - shift),
                             (float*)(base + (w.part_v - shift)), (float*)(base + (w.bias_v - shift)), st);
  return e;
}

// nsa_compress with optional page tables for the input tokens and the output
// summaries (both null: the plain layouts of nsa_compress) and optional prepared
// weights (null: formed from the fp32 weights into the workspace)
nsa_status_t compress_common(const void* k, const void* v, const float* w_ck, const float* pe_k, const float* w_cv,
                             const float* pe_v, const int64_t* tok_offset, const int32_t* seq_len,
                             const int64_t* cmp_offset, int32_t batch, const nsa_heads_t* heads,
                             const nsa_params_t* params, void* k_cmp, void* v_cmp, void* workspace, size_t ws_bytes,
                             void* stream, const PageTable& x_pt, const PageTable& out_pt,
                             const uint8_t* prepared = nullptr) {
  nsa_status_t s = check_heads(heads);
  if (s != NSA_OK) return s;
  if ((s = check_params(params, false)) != NSA_OK) return s;
  if (heads->d_k != 64 && heads->d_k != 128 && heads->d_k != 192) return NSA_ERR_UNSUPPORTED;
  if (batch <= 0 || batch > NSA_MAX_BATCH) return batch <= 0 ? NSA_ERR_INVALID_ARG : NSA_ERR_UNSUPPORTED;
  if (!k || !v || !tok_offset || !seq_len || !cmp_offset || !k_cmp || !v_cmp || !workspace) return NSA_ERR_INVALID_ARG;
  if (!prepared && (!w_ck || !pe_k || !w_cv || !pe_v)) return NSA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cmp) || !aligned16(v_cmp) || !aligned16(workspace))
    return NSA_ERR_INVALID_ARG;
  const CompressWs w = compress_ws(heads, params, 0);
  if (ws_bytes < w.total) return NSA_ERR_WORKSPACE;

  SeqTable t{};
  t.n = batch;
  int tiles = 0;
  int64_t rows_total = 0;   // packed output rows; -1 when the rows are not packed
  for (int b = 0; b < batch; ++b) {
    if (seq_len[b] < 0 || tok_offset[b] < 0 || cmp_offset[b] < 0) return NSA_ERR_INVALID_ARG;
    t.tile_prefix[b] = tiles;
    t.tok_off[b] = tok_offset[b];
    t.cmp_off[b] = cmp_offset[b];
    t.len[b] = seq_len[b];
    const int nc = n_cmp_of(seq_len[b], params->l_cmp, params->stride);
    tiles += (nc + 127) / 128;
    if (rows_total >= 0) rows_total = (cmp_offset[b] == rows_total) ? rows_total + nc : -1;
  }
  t.tile_prefix[batch] = tiles;
  if (out_pt.table) rows_total = -1;   // paged output rows are not packed: no split of K

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // the prepared weights: in the workspace (formed now) or the caller's blob,
  // whose offsets are the workspace's less its 256-byte header
  const uint8_t* wbase = prepared ? prepared : ws;
  const size_t wshift = prepared ? 256 : 0;
  cudaError_t e = cudaSuccess;
  if (!prepared) {
    prof_begin(P_COMPRESS_PREP, st);
    e = prepare_weights(w_ck, pe_k, w_cv, pe_v, heads, params, ws, 0, w, st);
    prof_end(P_COMPRESS_PREP, st, 4);
    if (e != cudaSuccess) return cuda_fail(e, "compress prep");
  }
  if (tiles == 0) return NSA_OK;

  CompressArgs a{};
  a.H_kv = heads->H_kv; a.l = params->l_cmp; a.s = params->stride;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.x_pt = x_pt;
  a.out_pt = out_pt;
  a.seqs = t;
  a.rows_total = rows_total > 0 ? rows_total : 0;
  a.x[0] = k; a.wt[0] = wbase + (w.wt_k - wshift); a.bias[0] = (const float*)(wbase + (w.bias_k - wshift));
  a.x[1] = v; a.wt[1] = wbase + (w.wt_v - wshift); a.bias[1] = (const float*)(wbase + (w.bias_v - wshift));
  a.out[0] = k_cmp;
  a.out[1] = v_cmp;
  // split K when the row tiles alone leave SMs idle, the rows are packed and the
  // workspace has room for the partial sums of both maps
  int ks = 1;
  if (rows_total > 0) {
    const int ctas = tiles * heads->H_kv * 2;
    ks = (2 * 148 + ctas - 1) / ctas;
    if (ks > kMaxKSplit) ks = kMaxKSplit;
    const size_t dsum = (size_t)(heads->d_k + heads->d_v);
    while (ks > 1 && w.ksum + (size_t)ks * rows_total * heads->H_kv * dsum * 4 > ws_bytes) ks >>= 1;
  }
  const int dm[2] = {heads->d_k, heads->d_v};
  bool split = false;
  for (int m = 0; m < 2; ++m) {
    const int nkb = params->l_cmp * dm[m] / 64;
    a.kb_per_split[m] = (nkb + ks - 1) / ks;
    a.ksplit[m] = (nkb + a.kb_per_split[m] - 1) / a.kb_per_split[m];
    split |= a.ksplit[m] > 1;
  }
  a.part[0] = (float*)(ws + w.ksum);
  a.part[1] = a.part[0] + (size_t)a.ksplit[0] * a.rows_total * heads->H_kv * heads->d_k;
  // W^T of both maps in boxes of 64 columns x d rows; k and v as views of whole
  // groups of s tokens up to the end of the last sequence (contiguous input only)
  CompressMaps mp;
  memset(&mp, 0, sizeof(mp));
  if (!make_map_3d(&mp.w[0], a.wt[0], params->l_cmp * heads->d_k, 1, heads->d_k, 1, heads->d_k) ||
      !make_map_3d(&mp.w[1], a.wt[1], params->l_cmp * heads->d_v, 1, heads->d_v, 1, heads->d_v)) {
    snprintf(g_detail, sizeof(g_detail), "cuTensorMapEncodeTiled failed (compression)");
    return NSA_ERR_CUDA;
  }
  a.x_chunks = 0;
  if (!x_pt.table) {
    int64_t rows_x = 0;
    for (int bb = 0; bb < batch; ++bb)
      if (tok_offset[bb] + seq_len[bb] > rows_x) rows_x = tok_offset[bb] + seq_len[bb];
    const int64_t chunks = rows_x / params->stride;
    if (chunks > 0 && chunks < (int64_t)1 << 31 &&
        make_map_xview(&mp.x[0], k, heads->d_k, heads->H_kv, params->stride, chunks) &&
        make_map_xview(&mp.x[1], v, heads->d_v, heads->H_kv, params->stride, chunks))
      a.x_chunks = (int)chunks;
  }
  prof_begin(P_COMPRESS_GEMM, st);
  e = launch_compress_gemm(heads->d_k, heads->d_v, a, mp, tiles, st);
  if (e == cudaSuccess && split) e = launch_compress_finalize(heads->d_k, heads->d_v, a, st);
  prof_end(P_COMPRESS_GEMM, st, split ? 2 : 1);
  if (e != cudaSuccess) return cuda_fail(e, "compress gemm");
  return NSA_OK;
}
}  // namespace

extern "C" {

nsa_status_t nsa_compress(const void* k, const void* v, const float* w_ck, const float* pe_k, const float* w_cv,
                          const float* pe_v, const int64_t* tok_offset, const int32_t* seq_len,
                          const int64_t* cmp_offset, int32_t batch, const nsa_heads_t* heads,
                          const nsa_params_t* params, void* k_cmp, void* v_cmp, void* workspace, size_t ws_bytes,
                          void* stream) {
  const PageTable none{};
  return compress_common(k, v, w_ck, pe_k, w_cv, pe_v, tok_offset, seq_len, cmp_offset, batch, heads, params, k_cmp,
                         v_cmp, workspace, ws_bytes, stream, none, none);
}

size_t nsa_compress_weights_size(const nsa_heads_t* heads, const nsa_params_t* params) {
  if (check_heads(heads) != NSA_OK || check_params(params, false) != NSA_OK) return 0;
  return compress_ws(heads, params, 0).ksum - 256;
}

nsa_status_t nsa_compress_prepare(const float* w_ck, const float* pe_k, const float* w_cv, const float* pe_v,
                                  const nsa_heads_t* heads, const nsa_params_t* params, void* prepared,
                                  size_t prepared_bytes, void* stream) {
  nsa_status_t s = check_heads(heads);
  if (s != NSA_OK) return s;
  if ((s = check_params(params, false)) != NSA_OK) return s;
  if (heads->d_k != 64 && heads->d_k != 128 && heads->d_k != 192) return NSA_ERR_UNSUPPORTED;
  if (!w_ck || !pe_k || !w_cv || !pe_v || !prepared || (reinterpret_cast<uintptr_t>(prepared) & 255u) != 0)
    return NSA_ERR_INVALID_ARG;
  const CompressWs w = compress_ws(heads, params, 0);
  if (prepared_bytes < w.ksum - 256) return NSA_ERR_WORKSPACE;
  cudaError_t e = prepare_weights(w_ck, pe_k, w_cv, pe_v, heads, params, static_cast<uint8_t*>(prepared), 256, w,
                                  static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "nsa_compress_prepare");
  return NSA_OK;
}

nsa_status_t nsa_compress_prepared(const void* k, const void* v, const void* prepared,
                                   const int64_t* tok_offset, const int32_t* seq_len, const int64_t* cmp_offset,
                                   int32_t batch, const nsa_heads_t* heads, const nsa_params_t* params,
                                   void* k_cmp, void* v_cmp, void* workspace, size_t ws_bytes, void* stream) {
  if (!prepared || (reinterpret_cast<uintptr_t>(prepared) & 255u) != 0) return NSA_ERR_INVALID_ARG;
  const PageTable none{};
  return compress_common(k, v, nullptr, nullptr, nullptr, nullptr, tok_offset, seq_len, cmp_offset, batch, heads,
                         params, k_cmp, v_cmp, workspace, ws_bytes, stream, none, none,
                         static_cast<const uint8_t*>(prepared));
}

nsa_status_t nsa_compress_paged(const void* k_pool, const void* v_pool, int32_t n_pages, int32_t page_size,
                                const int32_t* block_table, int32_t max_pages, const float* w_ck, const float* pe_k,
                                const float* w_cv, const float* pe_v, const int32_t* lens_prev, const int32_t* lens,
                                int32_t batch, void* k_cmp_pool, void* v_cmp_pool, int32_t n_cmp_pages,
                                int32_t cmp_page_size, const int32_t* cmp_block_table, int32_t max_cmp_pages,
                                const nsa_heads_t* heads, const nsa_params_t* params, int32_t* n_blocks,
                                void* workspace, size_t ws_bytes, void* stream) {
  nsa_status_t s = check_heads(heads);
  if (s != NSA_OK) return s;
  if ((s = check_params(params, false)) != NSA_OK) return s;
  if (batch <= 0 || batch > NSA_MAX_BATCH) return batch <= 0 ? NSA_ERR_INVALID_ARG : NSA_ERR_UNSUPPORTED;
  if (!block_table || !cmp_block_table || n_pages <= 0 || n_cmp_pages <= 0 || max_pages <= 0 ||
      max_cmp_pages <= 0)
    return NSA_ERR_INVALID_ARG;
  if (page_size <= 0 || page_size % 64 != 0 || cmp_page_size <= 0 || cmp_page_size % 32 != 0)
    return NSA_ERR_INVALID_ARG;
  const int64_t cap = (int64_t)max_pages * page_size, ccap = (int64_t)max_cmp_pages * cmp_page_size;
  if (cap > INT32_MAX || ccap < n_cmp_of((int)cap, params->l_cmp, params->stride)) return NSA_ERR_INVALID_ARG;
  // plan the new blocks as nsa_compress_append_plan does, but with offsets inside
  // each sequence (token index i0 * stride, entry index i0): the tables map them
  int64_t tok[NSA_MAX_BATCH], coff[NSA_MAX_BATCH];
  int32_t len[NSA_MAX_BATCH], n = 0;
  s = nsa_compress_append_plan(lens_prev, lens, batch, (int32_t)cap, (int32_t)ccap, params, tok, len, coff, &n);
  if (s != NSA_OK) return s;
  for (int b = 0; b < batch; ++b) {
    tok[b] -= (int64_t)b * cap;
    coff[b] -= (int64_t)b * ccap;
  }
  if (n_blocks) *n_blocks = n;
  if (n == 0) return NSA_OK;
  const PageTable x_pt{block_table, page_size, max_pages, n_pages};
  const PageTable out_pt{cmp_block_table, cmp_page_size, max_cmp_pages, n_cmp_pages};
  return compress_common(k_pool, v_pool, w_ck, pe_k, w_cv, pe_v, tok, len, coff, batch, heads, params, k_cmp_pool,
                         v_cmp_pool, workspace, ws_bytes, stream, x_pt, out_pt);
}

nsa_status_t nsa_compress_append_plan(const int32_t* lens_prev, const int32_t* lens, int32_t batch, int32_t Lmax,
                                      int32_t Lmax_cmp, const nsa_params_t* params, int64_t* tok_offset,
                                      int32_t* seq_len, int64_t* cmp_offset, int32_t* n_blocks) {
  // host-only planning works for any block / stride pair (l a multiple of s);
  // nsa_compress_append then checks what the kernels support
  if (!params || params->l_cmp <= 0 || params->stride <= 0 || params->l_cmp % params->stride != 0)
    return NSA_ERR_INVALID_ARG;
  if (batch <= 0 || batch > NSA_MAX_BATCH) return batch <= 0 ? NSA_ERR_INVALID_ARG : NSA_ERR_UNSUPPORTED;
  if (!lens || !tok_offset || !seq_len || !cmp_offset || Lmax <= 0 || Lmax_cmp < 0) return NSA_ERR_INVALID_ARG;
  if (Lmax_cmp < n_cmp_of(Lmax, params->l_cmp, params->stride)) return NSA_ERR_INVALID_ARG;
  int32_t total = 0;
  for (int b = 0; b < batch; ++b) {
    const int L = lens[b];
    const int P = lens_prev ? lens_prev[b] : L - 1;
    if (L < 0 || L > Lmax || P < -1 || P > L) return NSA_ERR_INVALID_ARG;
    // blocks i with n_cmp(P) <= i < n_cmp(L) were completed by the growth; their
    // tokens [i0*s, (i1-1)*s + l) form one segment of the batched cache
    const int i0 = n_cmp_of(P > 0 ? P : 0, params->l_cmp, params->stride);
    const int i1 = n_cmp_of(L, params->l_cmp, params->stride);
    if (i1 > i0) {
      tok_offset[b] = (int64_t)b * Lmax + (int64_t)i0 * params->stride;
      seq_len[b] = (i1 - 1 - i0) * params->stride + params->l_cmp;
      cmp_offset[b] = (int64_t)b * Lmax_cmp + i0;
      total += i1 - i0;
    } else {
      tok_offset[b] = (int64_t)b * Lmax;
      seq_len[b] = 0;
      cmp_offset[b] = (int64_t)b * Lmax_cmp;
    }
  }
  if (n_blocks) *n_blocks = total;
  return NSA_OK;
}

nsa_status_t nsa_compress_append(const void* k_cache, const void* v_cache, const float* w_ck, const float* pe_k,
                                 const float* w_cv, const float* pe_v, const int32_t* lens_prev, const int32_t* lens,
                                 int32_t batch, int32_t Lmax, int32_t Lmax_cmp, const nsa_heads_t* heads,
                                 const nsa_params_t* params, void* k_cmp_cache, void* v_cmp_cache,
                                 int32_t* n_blocks, void* workspace, size_t ws_bytes, void* stream) {
  nsa_status_t s = check_heads(heads);
  if (s != NSA_OK) return s;
  if (batch <= 0 || batch > NSA_MAX_BATCH) return batch <= 0 ? NSA_ERR_INVALID_ARG : NSA_ERR_UNSUPPORTED;
  int64_t tok[NSA_MAX_BATCH], coff[NSA_MAX_BATCH];
  int32_t len[NSA_MAX_BATCH], n = 0;
  s = nsa_compress_append_plan(lens_prev, lens, batch, Lmax, Lmax_cmp, params, tok, len, coff, &n);
  if (s != NSA_OK) return s;
  if (n_blocks) *n_blocks = n;
  if (n == 0) return NSA_OK;   // no block completed: nothing is launched
  return nsa_compress(k_cache, v_cache, w_ck, pe_k, w_cv, pe_v, tok, len, coff, batch, heads, params, k_cmp_cache,
                      v_cmp_cache, workspace, ws_bytes, stream);
}

nsa_status_t nsa_prefill(const void* q, const void* k, const void* v, const void* k_cmp, const void* v_cmp,
                         const float* gates, const int32_t* cu_seqlens, int32_t batch, const nsa_heads_t* heads,
                         const nsa_params_t* params, void* out, int32_t* sel_out, float* imp_out, void* workspace,
                         size_t ws_bytes, void* stream) {
  nsa_status_t s = check_heads(heads);
  if (s != NSA_OK) return s;
  if ((s = check_params(params, true)) != NSA_OK) return s;
  if (batch <= 0 || batch > NSA_MAX_BATCH) return batch <= 0 ? NSA_ERR_INVALID_ARG : NSA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !gates || !cu_seqlens || !out || !workspace) return NSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(workspace) ||
      !aligned16(gates))
    return NSA_ERR_INVALID_ARG;
  if (cu_seqlens[0] != 0) return NSA_ERR_INVALID_ARG;
  int max_len = 0;
  int64_t ncmp_total = 0;
  for (int b = 0; b < batch; ++b) {
    const int L = cu_seqlens[b + 1] - cu_seqlens[b];
    if (L < 0) return NSA_ERR_INVALID_ARG;
    if (L > max_len) max_len = L;
    ncmp_total += n_cmp_of(L, params->l_cmp, params->stride);
  }
  const int64_t N = cu_seqlens[batch];
  if (ncmp_total > 0 && (!k_cmp || !v_cmp || !aligned16(k_cmp) || !aligned16(v_cmp))) return NSA_ERR_INVALID_ARG;
  const PrefillWs w = prefill_ws(heads, params, N, max_len);
  if (ws_bytes < w.total) return NSA_ERR_WORKSPACE;
  if (N == 0) return NSA_OK;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  PrefillArgs a{};
  a.q = q; a.k = k; a.v = v; a.kc = k_cmp; a.vc = v_cmp; a.gates = gates;
  a.imp = imp_out ? imp_out : (float*)(ws + w.imp);
  a.sel = sel_out ? sel_out : (int32_t*)(ws + w.sel);
  a.want_imp = imp_out != nullptr;
  a.want_sel = sel_out != nullptr;
  a.out = out;
  a.H_q = heads->H_q; a.H_kv = heads->H_kv; a.G = heads->H_q / heads->H_kv;
  a.d_k = heads->d_k; a.d_v = heads->d_v;
  a.l = params->l_cmp; a.s = params->stride; a.ls = params->l_sel; a.top_n = params->top_n;
  a.window = params->window; a.force_first = params->force_first; a.force_local = params->force_local;
  a.nb_stride = w.nb;
  a.scale_log2 = softmax_scale(params, heads->d_k) * 1.4426950408889634f;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.fault_site = test_fault_site();
  if (!prefill_fused_stages(a)) {
    snprintf(g_detail, sizeof(g_detail), "sequence too long for the fused prefill kernel (%d blocks)", w.nb);
    return NSA_ERR_UNSUPPORTED;
  }

  const int tok_per_tile = 128 / a.G;   // one 128-row query tile per CTA
  SeqTable t{};
  t.n = batch;
  int tiles = 0;
  int64_t coff = 0;
  for (int b = 0; b < batch; ++b) {
    const int L = cu_seqlens[b + 1] - cu_seqlens[b];
    t.tile_prefix[b] = tiles;
    t.tok_off[b] = cu_seqlens[b];
    t.cmp_off[b] = coff;
    t.len[b] = L;
    tiles += (L + tok_per_tile - 1) / tok_per_tile;
    coff += n_cmp_of(L, params->l_cmp, params->stride);
  }
  t.tile_prefix[batch] = tiles;
  a.seqs = t;

  PrefillMaps m;
  memset(&m, 0, sizeof(m));
  const void* kc_base = ncmp_total > 0 ? k_cmp : k;
  const void* vc_base = ncmp_total > 0 ? v_cmp : v;
  if (!make_map_3d(&m.q, q, heads->d_k, heads->H_q, N, a.G, 128 / a.G) ||
      !make_map_3d(&m.k, k, heads->d_k, heads->H_kv, N, 1, 64) ||
      !make_map_3d(&m.v, v, heads->d_v, heads->H_kv, N, 1, 64) ||
      !make_map_3d(&m.kc, kc_base, heads->d_k, heads->H_kv, ncmp_total > 0 ? ncmp_total : N, 1, 64) ||
      !make_map_3d(&m.vc, vc_base, heads->d_v, heads->H_kv, ncmp_total > 0 ? ncmp_total : N, 1, 64)) {
    snprintf(g_detail, sizeof(g_detail), "cuTensorMapEncodeTiled failed");
    return NSA_ERR_CUDA;
  }

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  prof_begin(P_PREFILL_ATTN, st);
  cudaError_t e = launch_prefill_fused(a, m, tiles, st);
  prof_end(P_PREFILL_ATTN, st, 1);
  if (e != cudaSuccess) return cuda_fail(e, "prefill attention");
  return NSA_OK;
}

}  // extern "C"

namespace {
// nsa_decode with optional page tables; `rows` / `crows` are the rows of the raw
// and compressed tensors the maps cover (batch * Lmax or the pool's rows)
nsa_status_t decode_common(const void* q, const void* k_cache, const void* v_cache, const void* k_cmp_cache,
                           const void* v_cmp_cache, const int32_t* cache_lens, int32_t batch, int32_t Lmax,
                           int32_t Lmax_cmp, int32_t max_len, const float* gates, const nsa_heads_t* heads,
                           const nsa_params_t* params, void* out, int32_t* sel_out, float* imp_out, void* workspace,
                           size_t ws_bytes, void* stream, const PageTable& kv_pt, const PageTable& cmp_pt,
                           int64_t rows, int64_t crows) {
  nsa_status_t s = check_heads(heads);
  if (s != NSA_OK) return s;
  if ((s = check_params(params, true)) != NSA_OK) return s;
  if (batch <= 0 || batch > NSA_MAX_BATCH) return batch <= 0 ? NSA_ERR_INVALID_ARG : NSA_ERR_UNSUPPORTED;
  if (!q || !k_cache || !v_cache || !cache_lens || !gates || !out || !workspace) return NSA_ERR_INVALID_ARG;
  if (max_len <= 0 || Lmax < max_len) return NSA_ERR_INVALID_ARG;
  if (Lmax_cmp < n_cmp_of(max_len, params->l_cmp, params->stride)) return NSA_ERR_INVALID_ARG;
  if (Lmax_cmp > 0 && (!k_cmp_cache || !v_cmp_cache)) return NSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned16(workspace) ||
      (k_cmp_cache && !aligned16(k_cmp_cache)) || (v_cmp_cache && !aligned16(v_cmp_cache)))
    return NSA_ERR_INVALID_ARG;
  if (max_union_blocks(params) > 64) return NSA_ERR_UNSUPPORTED;
  DecodeArgs a{};
  fill_decode_args(a, heads, params, batch, Lmax, Lmax_cmp, max_len);
  if (a.n_cmp_chunks > 32) {   // the chunk merge holds one chunk per lane
    snprintf(g_detail, sizeof(g_detail), "decode cache longer than 262144 tokens");
    return NSA_ERR_UNSUPPORTED;
  }
  const DecodeWs w = decode_ws(a);
  if (ws_bytes < w.total) return NSA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.q = q; a.kcache = k_cache; a.vcache = v_cache; a.kc = k_cmp_cache; a.vc = v_cmp_cache;
  a.lens = cache_lens; a.gates = gates; a.out = out;
  a.sel = sel_out ? sel_out : (int32_t*)(ws + w.sel);
  a.imp = imp_out ? imp_out : (float*)(ws + w.imp);
  a.part = (float*)(ws + w.part);
  a.ocmp = (float*)(ws + w.ocmp);
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.fault_site = test_fault_site();
  a.kv_pt = kv_pt;
  a.cmp_pt = cmp_pt;
  DecodeMaps m;
  memset(&m, 0, sizeof(m));
  // decode streams 32-key tiles
  if (!make_map_3d(&m.k, k_cache, heads->d_k, heads->H_kv, rows, 1, 32) ||
      !make_map_3d(&m.v, v_cache, heads->d_v, heads->H_kv, rows, 1, 32) ||
      !make_map_3d(&m.kc, crows > 0 ? k_cmp_cache : k_cache, heads->d_k, heads->H_kv, crows > 0 ? crows : rows, 1, 32) ||
      !make_map_3d(&m.vc, crows > 0 ? v_cmp_cache : v_cache, heads->d_v, heads->H_kv, crows > 0 ? crows : rows, 1, 32) ||
      !make_map_3d(&m.q, q, heads->d_k, heads->H_q, batch, heads->H_q / heads->H_kv, 1)) {
    snprintf(g_detail, sizeof(g_detail), "cuTensorMapEncodeTiled failed");
    return NSA_ERR_CUDA;
  }
  cudaError_t e = launch_decode(a, m, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode");
  return NSA_OK;
}
}  // namespace

extern "C" {

nsa_status_t nsa_decode(const void* q, const void* k_cache, const void* v_cache, const void* k_cmp_cache,
                        const void* v_cmp_cache, const int32_t* cache_lens, int32_t batch, int32_t Lmax,
                        int32_t Lmax_cmp, int32_t max_len, const float* gates, const nsa_heads_t* heads,
                        const nsa_params_t* params, void* out, int32_t* sel_out, float* imp_out, void* workspace,
                        size_t ws_bytes, void* stream) {
  const PageTable none{};
  return decode_common(q, k_cache, v_cache, k_cmp_cache, v_cmp_cache, cache_lens, batch, Lmax, Lmax_cmp, max_len,
                       gates, heads, params, out, sel_out, imp_out, workspace, ws_bytes, stream, none, none,
                       (int64_t)batch * Lmax, (int64_t)batch * Lmax_cmp);
}

nsa_status_t nsa_decode_paged(const void* q, const void* k_pool, const void* v_pool, int32_t n_pages,
                              int32_t page_size, const int32_t* block_table, int32_t max_pages,
                              const void* k_cmp_pool, const void* v_cmp_pool, int32_t n_cmp_pages,
                              int32_t cmp_page_size, const int32_t* cmp_block_table, int32_t max_cmp_pages,
                              const int32_t* cache_lens, int32_t batch, int32_t max_len, const float* gates,
                              const nsa_heads_t* heads, const nsa_params_t* params, void* out, int32_t* sel_out,
                              float* imp_out, void* workspace, size_t ws_bytes, void* stream) {
  if (!block_table || !cmp_block_table || n_pages <= 0 || n_cmp_pages <= 0 || max_pages <= 0 || max_cmp_pages <= 0)
    return NSA_ERR_INVALID_ARG;
  if (page_size <= 0 || page_size % 64 != 0 || cmp_page_size <= 0 || cmp_page_size % 32 != 0)
    return NSA_ERR_INVALID_ARG;
  const int64_t cap = (int64_t)max_pages * page_size, ccap = (int64_t)max_cmp_pages * cmp_page_size;
  const int64_t rows = (int64_t)n_pages * page_size, crows = (int64_t)n_cmp_pages * cmp_page_size;
  if (cap > INT32_MAX || ccap > INT32_MAX || rows > INT32_MAX || crows > INT32_MAX) return NSA_ERR_UNSUPPORTED;
  const PageTable kv_pt{block_table, page_size, max_pages, n_pages};
  const PageTable cmp_pt{cmp_block_table, cmp_page_size, max_cmp_pages, n_cmp_pages};
  return decode_common(q, k_pool, v_pool, k_cmp_pool, v_cmp_pool, cache_lens, batch, (int32_t)cap, (int32_t)ccap,
                       max_len, gates, heads, params, out, sel_out, imp_out, workspace, ws_bytes, stream, kv_pt,
                       cmp_pt, rows, crows);
}

nsa_status_t nsa_prefill_backward(const void* q, const void* k, const void* v, const void* k_cmp,
                                  const void* v_cmp, const float* gates, const void* dout, const int32_t* sel,
                                  const float* w_ck, const float* pe_k, const float* w_cv, const float* pe_v,
                                  const int32_t* cu_seqlens, int32_t batch, const nsa_heads_t* heads,
                                  const nsa_params_t* params, float* dq, float* dk, float* dv, float* dgates,
                                  float* dw_ck, float* dpe_k, float* dw_cv, float* dpe_v, void* workspace,
                                  size_t ws_bytes, void* stream) {
  nsa_status_t s = check_heads(heads);
  if (s != NSA_OK) return s;
  if ((s = check_params(params, true)) != NSA_OK) return s;
  if (batch <= 0 || batch > NSA_MAX_BATCH) return batch <= 0 ? NSA_ERR_INVALID_ARG : NSA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !gates || !dout || !sel || !w_ck || !pe_k || !w_cv || !pe_v || !cu_seqlens || !dq ||
      !dk || !dv || !dgates || !dw_ck || !dpe_k || !dw_cv || !dpe_v || !workspace)
    return NSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(workspace) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return NSA_ERR_INVALID_ARG;
  if (cu_seqlens[0] != 0) return NSA_ERR_INVALID_ARG;
  int max_len = 0;
  int64_t ncmp = 0, nblk = 0;
  for (int b = 0; b < batch; ++b) {
    const int L = cu_seqlens[b + 1] - cu_seqlens[b];
    if (L < 0) return NSA_ERR_INVALID_ARG;
    if (L > max_len) max_len = L;
    ncmp += n_cmp_of(L, params->l_cmp, params->stride);
    nblk += n_blk_of(L, params->l_sel);
  }
  const int64_t N = cu_seqlens[batch];
  if (ncmp > 0 && (!k_cmp || !v_cmp || !aligned16(k_cmp) || !aligned16(v_cmp))) return NSA_ERR_INVALID_ARG;
  const BackwardWs w = backward_ws(heads, params, batch, N, ncmp, nblk);
  if (ws_bytes < w.total) return NSA_ERR_WORKSPACE;
  const int nb = n_blk_of(max_len, params->l_sel);
  if (backward_query_smem(heads->d_k, heads->d_v, nb) > 232448) {
    snprintf(g_detail, sizeof(g_detail), "sequence too long for the backward query kernel (%d blocks)", nb);
    return NSA_ERR_UNSUPPORTED;
  }
  if (N == 0) return NSA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  BackwardArgs a{};
  a.q = q; a.dout = dout; a.gates = gates; a.sel = sel;
  a.dq = dq; a.dk = dk; a.dv = dv; a.dgates = dgates;
  a.dkc = (float*)(ws + w.dkc); a.dvc = (float*)(ws + w.dvc);
  a.lse = (float*)(ws + w.lse); a.dd = (float*)(ws + w.dd);
  a.inv_off = (const int32_t*)(ws + w.off); a.inv_tok = (const int32_t*)(ws + w.tok);
  a.H_q = heads->H_q; a.H_kv = heads->H_kv; a.G = heads->H_q / heads->H_kv; a.d_k = heads->d_k; a.d_v = heads->d_v;
  a.l = params->l_cmp; a.s = params->stride; a.ls = params->l_sel; a.top_n = params->top_n;
  a.window = params->window;
  a.nb_stride = nb;
  a.tok_chunk = 256;
  a.scale = softmax_scale(params, heads->d_k);
  a.scale_log2 = a.scale * 1.4426950408889634f;
  a.status = reinterpret_cast<uint32_t*>(ws);
  SeqTable t{};
  t.n = batch;
  int q_tiles = 0, raw = 0, ctile = 0;
  int64_t coff = 0;
  int32_t ncmp_prefix[NSA_MAX_BATCH + 1];
  for (int b = 0; b < batch; ++b) {
    const int L = cu_seqlens[b + 1] - cu_seqlens[b];
    const int nc = n_cmp_of(L, params->l_cmp, params->stride);
    t.tile_prefix[b] = q_tiles;
    t.tok_off[b] = cu_seqlens[b];
    t.cmp_off[b] = coff;
    t.len[b] = L;
    a.blk_prefix[b] = raw;
    a.cblk_prefix[b] = ctile;
    ncmp_prefix[b] = (int32_t)coff;
    q_tiles += (L + 7) / 8;
    raw += n_blk_of(L, params->l_sel);
    ctile += (nc + 63) / 64;
    coff += nc;
  }
  t.tile_prefix[batch] = q_tiles;
  a.blk_prefix[batch] = raw;
  a.cblk_prefix[batch] = ctile;
  ncmp_prefix[batch] = (int32_t)coff;
  a.seqs = t;
  // grid.z of the key passes: the longest token sequence of a block (raw: the
  // window range plus every token of the sequence, as block 0 is chosen by all)
  const int cmp_z = (max_len + a.tok_chunk - 1) / a.tok_chunk;
  const int raw_z = (max_len + 64 + params->window + a.tok_chunk - 1) / a.tok_chunk;

  BackwardMaps m;
  memset(&m, 0, sizeof(m));
  const void* kcb = ncmp > 0 ? k_cmp : k;
  const void* vcb = ncmp > 0 ? v_cmp : v;
  const int64_t crows = ncmp > 0 ? ncmp : N;
  const int G = a.G;
  if (!make_map_3d(&m.k32, k, heads->d_k, heads->H_kv, N, 1, 32) ||
      !make_map_3d(&m.v32, v, heads->d_v, heads->H_kv, N, 1, 32) ||
      !make_map_3d(&m.kc32, kcb, heads->d_k, heads->H_kv, crows, 1, 32) ||
      !make_map_3d(&m.vc32, vcb, heads->d_v, heads->H_kv, crows, 1, 32) ||
      !make_map_3d(&m.k64, k, heads->d_k, heads->H_kv, N, 1, 64) ||
      !make_map_3d(&m.v64, v, heads->d_v, heads->H_kv, N, 1, 64) ||
      !make_map_3d(&m.kc64, kcb, heads->d_k, heads->H_kv, crows, 1, 64) ||
      !make_map_3d(&m.vc64, vcb, heads->d_v, heads->H_kv, crows, 1, 64) ||
      !make_map_3d(&m.qg, q, heads->d_k, heads->H_q, N, G, 1) ||
      !make_map_3d(&m.dog, dout, heads->d_v, heads->H_q, N, G, 1)) {
    snprintf(g_detail, sizeof(g_detail), "cuTensorMapEncodeTiled failed");
    return NSA_ERR_CUDA;
  }
  cudaError_t e = cudaMemsetAsync(dk, 0, (size_t)N * heads->H_kv * heads->d_k * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, (size_t)N * heads->H_kv * heads->d_v * 4, st);
  if (e != cudaSuccess) return cuda_fail(e, "backward memset");
  if (ncmp > 0) {
    e = cudaMemsetAsync(ws + w.dkc, 0, (size_t)ncmp * heads->H_kv * heads->d_k * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ws + w.dvc, 0, (size_t)ncmp * heads->H_kv * heads->d_v * 4, st);
    if (e != cudaSuccess) return cuda_fail(e, "backward memset");
  }
  prof_begin(P_BWD_INDEX, st);
  e = launch_inverted_index(a, w.n_ent, (int)w.n_lists, (int32_t*)(ws + w.cnt), (int32_t*)(ws + w.off),
                            (int32_t*)(ws + w.cur), (int32_t*)(ws + w.slot), (int32_t*)(ws + w.tok), st);
  prof_end(P_BWD_INDEX, st, 3);
  if (e != cudaSuccess) return cuda_fail(e, "backward index");
  prof_begin(P_BWD_QUERY, st);
  e = launch_backward_attn(a, m, q_tiles, 0, 0, 0, 0, st);
  prof_end(P_BWD_QUERY, st, 1);
  if (e != cudaSuccess) return cuda_fail(e, "backward query pass");
  prof_begin(P_BWD_KEYS, st);
  e = launch_backward_attn(a, m, 0, raw, raw_z, ctile, cmp_z, st);
  prof_end(P_BWD_KEYS, st, ctile > 0 ? 2 : 1);
  if (e != cudaSuccess) return cuda_fail(e, "backward key passes");
  prof_begin(P_BWD_COMPRESS, st);
  float* colsum = (float*)(ws + w.colsum);
  e = launch_compress_backward(a.dkc, k, w_ck, pe_k, heads->d_k, heads->d_k, heads->H_kv, params->l_cmp,
                               params->stride, t, ncmp_prefix, ncmp, dk, dw_ck, dpe_k, colsum, st);
  if (e == cudaSuccess)
    e = launch_compress_backward(a.dvc, v, w_cv, pe_v, heads->d_v, heads->d_v, heads->H_kv, params->l_cmp,
                                 params->stride, t, ncmp_prefix, ncmp, dv, dw_cv, dpe_v, colsum, st);
  prof_end(P_BWD_COMPRESS, st, 10);
  if (e != cudaSuccess) return cuda_fail(e, "backward compression");
  return NSA_OK;
}

// ---- DSA variant ----
static nsa_status_t check_dsa(const nsa_heads_t* heads, const nsa_dsa_params_t* dp) {
  nsa_status_t s = check_heads(heads);
  if (s != NSA_OK) return s;
  if (!dp || dp->H_I <= 0 || dp->d_I <= 0 || dp->top_k <= 0 || !(dp->scale >= 0.f)) return NSA_ERR_INVALID_ARG;
  if (dp->H_I > 16 || (dp->d_I != 32 && dp->d_I != 64 && dp->d_I != 128) || dp->top_k > 65536)
    return NSA_ERR_UNSUPPORTED;
  return NSA_OK;
}

// queries per chunk of a prefill: the score rows of a chunk fill at most 2^26 floats
static int64_t dsa_chunk(int64_t n_queries, int max_len) {
  const int64_t c = (int64_t(1) << 26) / (max_len > 0 ? max_len : 1);
  return n_queries < c ? n_queries : (c > 0 ? c : 1);
}

struct DsaWs {
  size_t scores, idx, total;
};
static DsaWs dsa_ws(int64_t slots, int max_len, int top_k) {
  DsaWs w{};
  size_t off = 256;
  w.scores = off; off = align256(off + (size_t)slots * max_len * 4);
  w.idx = off; off = align256(off + (size_t)slots * top_k * 4);
  w.total = off;
  return w;
}

size_t nsa_dsa_workspace_size(int op, const nsa_heads_t* heads, const nsa_dsa_params_t* dp, int32_t batch,
                              int64_t total_tokens, int32_t max_len) {
  if (check_dsa(heads, dp) != NSA_OK || batch <= 0 || batch > NSA_MAX_BATCH || max_len <= 0) return 0;
  if (op == NSA_OP_DSA_DECODE) return dsa_ws(batch, max_len, dp->top_k).total;
  if (op == NSA_OP_DSA_PREFILL) {
    if (total_tokens < 0) return 0;
    return dsa_ws(dsa_chunk(total_tokens, max_len), max_len, dp->top_k).total;
  }
  return 0;
}

static void fill_dsa(DsaArgs& a, const void* q, const void* k, const void* v, const void* qi, const float* wi,
                     const void* ki, void* out, const nsa_heads_t* heads, const nsa_dsa_params_t* dp, void* ws) {
  a.q = q; a.k = k; a.v = v; a.qi = qi; a.wi = wi; a.ki = ki; a.out = out;
  a.H_q = heads->H_q; a.H_kv = heads->H_kv; a.G = heads->H_q / heads->H_kv; a.H_I = dp->H_I; a.top_k = dp->top_k;
  a.scale_log2 = (dp->scale > 0.f ? dp->scale : 1.0f / sqrtf((float)heads->d_k)) * 1.4426950408889634f;
  a.status = reinterpret_cast<uint32_t*>(ws);
}

nsa_status_t nsa_dsa_decode(const void* q, const void* k_cache, const void* v_cache, const void* qi, const float* wi,
                            const void* ki_cache, const int32_t* cache_lens, int32_t batch, int32_t Lmax,
                            int32_t max_len, const nsa_dsa_params_t* dp, const nsa_heads_t* heads, void* out,
                            int32_t* idx_out, float* score_out, void* workspace, size_t ws_bytes, void* stream) {
  nsa_status_t s = check_dsa(heads, dp);
  if (s != NSA_OK) return s;
  if (batch <= 0 || batch > NSA_MAX_BATCH) return batch <= 0 ? NSA_ERR_INVALID_ARG : NSA_ERR_UNSUPPORTED;
  if (!q || !k_cache || !v_cache || !qi || !wi || !ki_cache || !cache_lens || !out || !workspace)
    return NSA_ERR_INVALID_ARG;
  if (max_len <= 0 || Lmax < max_len) return NSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(qi) || !aligned16(ki_cache) ||
      !aligned16(out) || !aligned16(workspace))
    return NSA_ERR_INVALID_ARG;
  const DsaWs w = dsa_ws(batch, max_len, dp->top_k);
  if (ws_bytes < w.total) return NSA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DsaArgs a{};
  fill_dsa(a, q, k_cache, v_cache, qi, wi, ki_cache, out, heads, dp, ws);
  a.scores = score_out ? score_out : (float*)(ws + w.scores);
  a.idx = idx_out ? idx_out : (int32_t*)(ws + w.idx);
  a.ld_scores = max_len;
  a.q0 = 0;
  a.lens = cache_lens;
  a.Lmax = Lmax;
  a.max_len = max_len;
  cudaError_t e = launch_dsa(a, batch, max_len, heads->d_k, heads->d_v, dp->d_I, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NSA_OK : cuda_fail(e, "dsa decode");
}

nsa_status_t nsa_dsa_prefill(const void* q, const void* k, const void* v, const void* qi, const float* wi,
                             const void* ki, const int32_t* cu_seqlens, int32_t batch, const nsa_dsa_params_t* dp,
                             const nsa_heads_t* heads, void* out, int32_t* idx_out, float* score_out, void* workspace,
                             size_t ws_bytes, void* stream) {
  nsa_status_t s = check_dsa(heads, dp);
  if (s != NSA_OK) return s;
  if (batch <= 0 || batch > NSA_MAX_BATCH) return batch <= 0 ? NSA_ERR_INVALID_ARG : NSA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !qi || !wi || !ki || !cu_seqlens || !out || !workspace) return NSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(qi) || !aligned16(ki) || !aligned16(out) ||
      !aligned16(workspace))
    return NSA_ERR_INVALID_ARG;
  if (cu_seqlens[0] != 0) return NSA_ERR_INVALID_ARG;
  SeqTable t{};
  t.n = batch;
  int max_len = 0;
  for (int b = 0; b < batch; ++b) {
    const int L = cu_seqlens[b + 1] - cu_seqlens[b];
    if (L < 0) return NSA_ERR_INVALID_ARG;
    if (L > max_len) max_len = L;
    t.tok_off[b] = cu_seqlens[b];
    t.len[b] = L;
  }
  const int64_t N = cu_seqlens[batch];
  if (N == 0) return NSA_OK;
  const int64_t chunk = dsa_chunk(N, max_len);
  const DsaWs w = dsa_ws(chunk, max_len, dp->top_k);
  if (ws_bytes < w.total) return NSA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DsaArgs a{};
  fill_dsa(a, q, k, v, qi, wi, ki, out, heads, dp, ws);
  a.scores = (float*)(ws + w.scores);
  a.ld_scores = max_len;
  a.seqs = t;
  a.max_len = max_len;
  for (int64_t q0 = 0; q0 < N; q0 += chunk) {
    const int n = (int)(N - q0 < chunk ? N - q0 : chunk);
    a.q0 = q0;
    a.idx = idx_out ? idx_out + q0 * dp->top_k : (int32_t*)(ws + w.idx);
    a.scores = score_out ? score_out + q0 * max_len : (float*)(ws + w.scores);
    cudaError_t e = launch_dsa(a, n, max_len, heads->d_k, heads->d_v, dp->d_I, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dsa prefill");
  }
  return NSA_OK;
}

}  // extern "C"
