// nsa_compress_noalloc: block compression for callers that cannot allocate.
//
// Some callers may not call cudaMalloc (or any allocating routine) at the point
// where they run the compression: code running while a CUDA graph is being
// captured on the same device, engines whose memory plan is fixed ahead of time
// and which forbid allocation on the serving path, or plugins that live inside a
// framework that owns every device allocation. For them this entry point takes
// no workspace argument: its scratch (the bf16 copies of the two weight
// matrices, the fp32 position terms and the status word) lives in a file-scope
// device array of NSA_NOALLOC_SCRATCH_BYTES, which every GPU that loads the
// library keeps reserved until the process exits.
#include <cstdio>
#include <mutex>

#include "../../include/nsa.h"
#include "kernels.h"

namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[NSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, resolved once per
// device (the name is only a host-side stand-in; kernels need this address).
nsa_status_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    nsa::set_error_detail("nsa_compress_noalloc: cudaGetDevice failed");
    return NSA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    nsa::set_error_detail("nsa_compress_noalloc: device index out of range");
    return NSA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> g(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      char msg[160];
      snprintf(msg, sizeof(msg), "nsa_compress_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
      nsa::set_error_detail(msg);
      return NSA_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return NSA_OK;
}

}  // namespace

extern "C" nsa_status_t nsa_compress_noalloc(const void* k, const void* v, const float* w_ck, const float* pe_k,
                                             const float* w_cv, const float* pe_v, const int64_t* tok_offset,
                                             const int32_t* seq_len, const int64_t* cmp_offset, int32_t batch,
                                             const nsa_heads_t* heads, const nsa_params_t* params, void* k_cmp,
                                             void* v_cmp, void* stream) {
  const size_t need = nsa_workspace_size(NSA_OP_COMPRESS, heads, params, batch, 0, 0);
  if (need == 0) {
    // invalid or unsupported arguments: let nsa_compress name the exact status
    return nsa_compress(k, v, w_ck, pe_k, w_cv, pe_v, tok_offset, seq_len, cmp_offset, batch, heads, params,
                        k_cmp, v_cmp, nullptr, 0, stream);
  }
  if (need > (size_t)NSA_NOALLOC_SCRATCH_BYTES) {
    char msg[160];
    snprintf(msg, sizeof(msg), "nsa_compress_noalloc: needs %zu bytes of scratch, the built-in maximum is %d",
             need, NSA_NOALLOC_SCRATCH_BYTES);
    nsa::set_error_detail(msg);
    return NSA_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  nsa_status_t s = scratch_address(&scratch);
  if (s != NSA_OK) return s;
  // the array keeps the previous call's contents: clear the status word
  cudaError_t e = cudaMemsetAsync(scratch, 0, 256, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    nsa::set_error_detail("nsa_compress_noalloc: clearing the scratch header failed");
    return NSA_ERR_CUDA;
  }
  return nsa_compress(k, v, w_ck, pe_k, w_cv, pe_v, tok_offset, seq_len, cmp_offset, batch, heads, params, k_cmp,
                      v_cmp, scratch, (size_t)NSA_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" nsa_status_t nsa_noalloc_check_status(void* stream) {
  void* scratch = nullptr;
  nsa_status_t s = scratch_address(&scratch);
  if (s != NSA_OK) return s;
  // the array's header is the status word of an ordinary workspace
  return nsa_check_device_status(scratch, stream);
}
