"""Python binding of libnsa.so — NSA (Native Sparse Attention) forward on B200.

Thin ctypes layer over the C ABI declared in include/nsa.h: every function here
only checks and marshals arguments (torch tensors -> device pointers, the
current CUDA stream) and calls the entry point of the same name. All compute
runs in the library's sm_100a kernels; there is no fallback: if the shared
library is missing or cannot be loaded, every call raises.

Convenience helpers at the bottom (`compress`, `prefill`, `decode`) allocate
outputs and the workspace with torch and then call the entry points.
"""
from __future__ import annotations

import contextlib
import ctypes
import math
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnsa.so")
# checking build (index checks, test fault injection; include/nsa_check.h): tests only
CHECK_LIB_PATH = os.path.join(_PKG, "libnsa_check.so")

NSA_OK, NSA_ERR_INVALID_ARG, NSA_ERR_UNSUPPORTED, NSA_ERR_WORKSPACE, NSA_ERR_CUDA, NSA_ERR_DEVICE_CHECK = range(6)
NSA_OP_COMPRESS, NSA_OP_PREFILL, NSA_OP_DECODE, NSA_OP_BACKWARD = 0, 1, 2, 3
NSA_MAX_BATCH = 128
NSA_NOALLOC_SCRATCH_BYTES = 4194304

# every symbol include/nsa.h declares
EXPORTED = ("nsa_workspace_size", "nsa_workspace_init", "nsa_check_device_status", "nsa_compress",
            "nsa_compress_append_plan", "nsa_compress_append", "nsa_compress_paged", "nsa_compress_noalloc",
            "nsa_noalloc_check_status", "nsa_compress_weights_size", "nsa_compress_prepare", "nsa_compress_prepared",
            "nsa_decode_paged", "nsa_prefill_backward", "nsa_dsa_workspace_size", "nsa_dsa_decode",
            "nsa_dsa_prefill", "nsa_prefill", "nsa_decode", "nsa_profile_enable", "nsa_profile_read", "nsa_profile_slot_name",
            "nsa_status_string", "nsa_last_error_detail")
NSA_PROFILE_SLOTS = 12
NSA_OP_DSA_DECODE, NSA_OP_DSA_PREFILL = 4, 5
# the checking build exports one more symbol (include/nsa_check.h)
CHECK_EXPORTED = EXPORTED + ("nsa_test_set_fault",)
FAULT_NONE, FAULT_DECODE_FINE_TILE, FAULT_PREFILL_K_TILE = 0, 1, 2


class NSAError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {status_name(status)}" + (f" ({detail})" if detail else ""))


class Params(ctypes.Structure):
    """nsa_params_t"""
    _fields_ = [("l_cmp", ctypes.c_int32), ("stride", ctypes.c_int32), ("l_sel", ctypes.c_int32),
                ("top_n", ctypes.c_int32), ("window", ctypes.c_int32), ("force_first", ctypes.c_int32),
                ("force_local", ctypes.c_int32), ("scale", ctypes.c_float)]


class Heads(ctypes.Structure):
    """nsa_heads_t"""
    _fields_ = [("H_q", ctypes.c_int32), ("H_kv", ctypes.c_int32), ("d_k", ctypes.c_int32),
                ("d_v", ctypes.c_int32)]


class DsaParams(ctypes.Structure):
    """nsa_dsa_params_t"""
    _fields_ = [("H_I", ctypes.c_int32), ("d_I", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("scale", ctypes.c_float)]


def make_params(l_cmp=32, stride=16, l_sel=64, top_n=16, window=512, force_first=1, force_local=2,
                scale=0.0) -> Params:
    return Params(l_cmp, stride, l_sel, top_n, window, force_first, force_local, float(scale))


_lib = None
_loaded = {}


def lib() -> ctypes.CDLL:
    """Load libnsa.so once. Raises if it is missing (no CPU fallback exists)."""
    global _lib
    if _lib is not None:
        return _lib
    _lib = _load(LIB_PATH)
    return _lib


@contextlib.contextmanager
def checking_library():
    """Route every entry point of this module through libnsa_check.so (the
    checking build) inside the `with` block; the library build is restored after."""
    global _lib
    prev = lib()
    _lib = _load(CHECK_LIB_PATH)
    try:
        yield _lib
    finally:
        _lib = prev


def nsa_test_set_fault(site: int):
    """Checking build only (include/nsa_check.h): make a producer withhold a tile."""
    L = lib()
    if not hasattr(L, "nsa_test_set_fault"):
        raise RuntimeError("nsa_test_set_fault exists only in the checking build (use checking_library())")
    _check(L.nsa_test_set_fault(int(site)), "nsa_test_set_fault")


def _load(path: str) -> ctypes.CDLL:
    if path in _loaded:
        return _loaded[path]
    if not os.path.exists(path):
        raise ImportError(f"{os.path.basename(path)} not built at {path}; run python -m sparse_attention_long_nsa_b200.build")
    L = ctypes.CDLL(path)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    L.nsa_workspace_size.restype = SZ
    L.nsa_workspace_size.argtypes = [ctypes.c_int, ctypes.POINTER(Heads), ctypes.POINTER(Params), I32, I64, I32]
    L.nsa_workspace_init.restype = ctypes.c_int
    L.nsa_workspace_init.argtypes = [P, SZ, P]
    L.nsa_check_device_status.restype = ctypes.c_int
    L.nsa_check_device_status.argtypes = [P, P]
    L.nsa_compress.restype = ctypes.c_int
    L.nsa_compress.argtypes = [P, P, P, P, P, P, P, P, P, I32, ctypes.POINTER(Heads), ctypes.POINTER(Params),
                               P, P, P, SZ, P]
    L.nsa_compress_weights_size.restype = SZ
    L.nsa_compress_weights_size.argtypes = [ctypes.POINTER(Heads), ctypes.POINTER(Params)]
    L.nsa_compress_prepare.restype = ctypes.c_int
    L.nsa_compress_prepare.argtypes = [P, P, P, P, ctypes.POINTER(Heads), ctypes.POINTER(Params), P, SZ, P]
    L.nsa_compress_prepared.restype = ctypes.c_int
    L.nsa_compress_prepared.argtypes = [P, P, P, P, P, P, I32, ctypes.POINTER(Heads), ctypes.POINTER(Params),
                                        P, P, P, SZ, P]
    L.nsa_compress_append_plan.restype = ctypes.c_int
    L.nsa_compress_append_plan.argtypes = [P, P, I32, I32, I32, ctypes.POINTER(Params), P, P, P, P]
    L.nsa_compress_append.restype = ctypes.c_int
    L.nsa_compress_append.argtypes = [P, P, P, P, P, P, P, P, I32, I32, I32, ctypes.POINTER(Heads),
                                      ctypes.POINTER(Params), P, P, P, P, SZ, P]
    L.nsa_compress_paged.restype = ctypes.c_int
    L.nsa_compress_paged.argtypes = [P, P, I32, I32, P, I32, P, P, P, P, P, P, I32, P, P, I32, I32, P, I32,
                                     ctypes.POINTER(Heads), ctypes.POINTER(Params), P, P, SZ, P]
    L.nsa_decode_paged.restype = ctypes.c_int
    L.nsa_decode_paged.argtypes = [P, P, P, I32, I32, P, I32, P, P, I32, I32, P, I32, P, I32, I32, P,
                                   ctypes.POINTER(Heads), ctypes.POINTER(Params), P, P, P, P, SZ, P]
    L.nsa_prefill_backward.restype = ctypes.c_int
    L.nsa_prefill_backward.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, I32, ctypes.POINTER(Heads),
                                       ctypes.POINTER(Params), P, P, P, P, P, P, P, P, P, SZ, P]
    L.nsa_dsa_workspace_size.restype = SZ
    L.nsa_dsa_workspace_size.argtypes = [ctypes.c_int, ctypes.POINTER(Heads), ctypes.POINTER(DsaParams), I32, I64,
                                         I32]
    L.nsa_dsa_decode.restype = ctypes.c_int
    L.nsa_dsa_decode.argtypes = [P, P, P, P, P, P, P, I32, I32, I32, ctypes.POINTER(DsaParams),
                                 ctypes.POINTER(Heads), P, P, P, P, SZ, P]
    L.nsa_dsa_prefill.restype = ctypes.c_int
    L.nsa_dsa_prefill.argtypes = [P, P, P, P, P, P, P, I32, ctypes.POINTER(DsaParams), ctypes.POINTER(Heads), P, P,
                                  P, P, SZ, P]
    L.nsa_noalloc_check_status.restype = ctypes.c_int
    L.nsa_noalloc_check_status.argtypes = [P]
    L.nsa_compress_noalloc.restype = ctypes.c_int
    L.nsa_compress_noalloc.argtypes = [P, P, P, P, P, P, P, P, P, I32, ctypes.POINTER(Heads),
                                       ctypes.POINTER(Params), P, P, P]
    L.nsa_prefill.restype = ctypes.c_int
    L.nsa_prefill.argtypes = [P, P, P, P, P, P, P, I32, ctypes.POINTER(Heads), ctypes.POINTER(Params), P, P, P,
                              P, SZ, P]
    L.nsa_decode.restype = ctypes.c_int
    L.nsa_decode.argtypes = [P, P, P, P, P, P, I32, I32, I32, I32, P, ctypes.POINTER(Heads),
                             ctypes.POINTER(Params), P, P, P, P, SZ, P]
    L.nsa_profile_enable.restype = ctypes.c_int
    L.nsa_profile_enable.argtypes = [I32]
    L.nsa_profile_read.restype = ctypes.c_int
    L.nsa_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64), I32]
    L.nsa_profile_slot_name.restype = ctypes.c_char_p
    L.nsa_profile_slot_name.argtypes = [I32]
    L.nsa_status_string.restype = ctypes.c_char_p
    L.nsa_status_string.argtypes = [ctypes.c_int]
    L.nsa_last_error_detail.restype = ctypes.c_char_p
    L.nsa_last_error_detail.argtypes = []
    if hasattr(L, "nsa_test_set_fault"):
        L.nsa_test_set_fault.restype = ctypes.c_int
        L.nsa_test_set_fault.argtypes = [I32]
    _loaded[path] = L
    return L


def status_name(s: int) -> str:
    try:
        return lib().nsa_status_string(s).decode()
    except Exception:
        return f"status {s}"


def _check(s: int, where: str):
    if s != NSA_OK:
        detail = lib().nsa_last_error_detail().decode() if s == NSA_ERR_CUDA or s == NSA_ERR_DEVICE_CHECK else ""
        raise NSAError(s, where, detail)


def _ptr(t: Optional[torch.Tensor], dtype=None, device_kind="cuda") -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    if device_kind == "cuda" and t.device.type != "cuda":
        raise ValueError("expected a CUDA tensor")
    if device_kind == "cpu" and t.device.type != "cpu":
        raise ValueError("expected a host tensor")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ---------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ---------------------------------------------------------------------------

def nsa_workspace_size(op: int, heads: Heads, params: Params, batch: int, total_tokens: int, max_len: int) -> int:
    return int(lib().nsa_workspace_size(op, ctypes.byref(heads), ctypes.byref(params), batch, total_tokens,
                                        max_len))


def nsa_workspace_init(ws: torch.Tensor, stream=None):
    _check(lib().nsa_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "nsa_workspace_init")


def nsa_check_device_status(ws: torch.Tensor, stream=None):
    _check(lib().nsa_check_device_status(_ptr(ws), _stream(stream)), "nsa_check_device_status")


def nsa_compress(k, v, w_ck, pe_k, w_cv, pe_v, tok_offset, seq_len, cmp_offset, heads: Heads, params: Params,
                 k_cmp, v_cmp, ws, stream=None):
    """tok_offset/cmp_offset: host int64 [B]; seq_len: host int32 [B]."""
    B = int(seq_len.numel())
    s = lib().nsa_compress(_ptr(k, torch.bfloat16), _ptr(v, torch.bfloat16), _ptr(w_ck, torch.float32),
                           _ptr(pe_k, torch.float32), _ptr(w_cv, torch.float32), _ptr(pe_v, torch.float32),
                           _ptr(tok_offset, torch.int64, "cpu"), _ptr(seq_len, torch.int32, "cpu"),
                           _ptr(cmp_offset, torch.int64, "cpu"), B, ctypes.byref(heads), ctypes.byref(params),
                           _ptr(k_cmp, torch.bfloat16), _ptr(v_cmp, torch.bfloat16), _ptr(ws),
                           ws.numel() * ws.element_size(), _stream(stream))
    _check(s, "nsa_compress")


def nsa_compress_weights_size(heads: Heads, params: Params) -> int:
    return int(lib().nsa_compress_weights_size(ctypes.byref(heads), ctypes.byref(params)))


def nsa_compress_prepare(w_ck, pe_k, w_cv, pe_v, heads: Heads, params: Params, prepared, stream=None):
    s = lib().nsa_compress_prepare(_ptr(w_ck, torch.float32), _ptr(pe_k, torch.float32), _ptr(w_cv, torch.float32),
                                   _ptr(pe_v, torch.float32), ctypes.byref(heads), ctypes.byref(params),
                                   _ptr(prepared), prepared.numel() * prepared.element_size(), _stream(stream))
    _check(s, "nsa_compress_prepare")


def nsa_compress_prepared(k, v, prepared, tok_offset, seq_len, cmp_offset, heads: Heads, params: Params, k_cmp, v_cmp,
                          ws, stream=None):
    """nsa_compress with weights from nsa_compress_prepare."""
    B = int(seq_len.numel())
    s = lib().nsa_compress_prepared(_ptr(k, torch.bfloat16), _ptr(v, torch.bfloat16), _ptr(prepared),
                                    _ptr(tok_offset, torch.int64, "cpu"), _ptr(seq_len, torch.int32, "cpu"),
                                    _ptr(cmp_offset, torch.int64, "cpu"), B, ctypes.byref(heads),
                                    ctypes.byref(params), _ptr(k_cmp, torch.bfloat16), _ptr(v_cmp, torch.bfloat16),
                                    _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(s, "nsa_compress_prepared")


def nsa_compress_noalloc(k, v, w_ck, pe_k, w_cv, pe_v, tok_offset, seq_len, cmp_offset, heads: Heads,
                         params: Params, k_cmp, v_cmp, stream=None):
    """nsa_compress without a workspace: scratch is a fixed device array inside
    the library (see include/nsa.h). Calls that overlap on the GPU race."""
    B = int(seq_len.numel())
    s = lib().nsa_compress_noalloc(_ptr(k, torch.bfloat16), _ptr(v, torch.bfloat16), _ptr(w_ck, torch.float32),
                                   _ptr(pe_k, torch.float32), _ptr(w_cv, torch.float32), _ptr(pe_v, torch.float32),
                                   _ptr(tok_offset, torch.int64, "cpu"), _ptr(seq_len, torch.int32, "cpu"),
                                   _ptr(cmp_offset, torch.int64, "cpu"), B, ctypes.byref(heads),
                                   ctypes.byref(params), _ptr(k_cmp, torch.bfloat16), _ptr(v_cmp, torch.bfloat16),
                                   _stream(stream))
    _check(s, "nsa_compress_noalloc")


def nsa_noalloc_check_status(stream=None):
    """Synchronise the stream, read and clear the status word of
    nsa_compress_noalloc's built-in scratch on the current device."""
    _check(lib().nsa_noalloc_check_status(_stream(stream)), "nsa_noalloc_check_status")


def nsa_prefill(q, k, v, k_cmp, v_cmp, gates, cu_seqlens, heads: Heads, params: Params, out, sel_out=None,
                imp_out=None, ws=None, stream=None):
    """cu_seqlens: host int32 [B+1]."""
    B = int(cu_seqlens.numel()) - 1
    s = lib().nsa_prefill(_ptr(q, torch.bfloat16), _ptr(k, torch.bfloat16), _ptr(v, torch.bfloat16),
                          _ptr(k_cmp, torch.bfloat16), _ptr(v_cmp, torch.bfloat16), _ptr(gates, torch.float32),
                          _ptr(cu_seqlens, torch.int32, "cpu"), B, ctypes.byref(heads), ctypes.byref(params),
                          _ptr(out, torch.bfloat16), _ptr(sel_out, torch.int32), _ptr(imp_out, torch.float32),
                          _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(s, "nsa_prefill")


def nsa_decode(q, k_cache, v_cache, k_cmp_cache, v_cmp_cache, cache_lens, max_len: int, gates, heads: Heads,
               params: Params, out, sel_out=None, imp_out=None, ws=None, stream=None):
    """cache_lens: device int32 [B]; caches [B, Lmax, H_kv, d] and [B, Lmax_cmp, H_kv, d]."""
    B, Lmax = int(k_cache.shape[0]), int(k_cache.shape[1])
    Lc = int(k_cmp_cache.shape[1]) if k_cmp_cache is not None else 0
    s = lib().nsa_decode(_ptr(q, torch.bfloat16), _ptr(k_cache, torch.bfloat16), _ptr(v_cache, torch.bfloat16),
                         _ptr(k_cmp_cache, torch.bfloat16), _ptr(v_cmp_cache, torch.bfloat16),
                         _ptr(cache_lens, torch.int32), B, Lmax, Lc, int(max_len), _ptr(gates, torch.float32),
                         ctypes.byref(heads), ctypes.byref(params), _ptr(out, torch.bfloat16),
                         _ptr(sel_out, torch.int32), _ptr(imp_out, torch.float32), _ptr(ws),
                         ws.numel() * ws.element_size(), _stream(stream))
    _check(s, "nsa_decode")


def nsa_compress_paged(k_pool, v_pool, block_table, w_ck, pe_k, w_cv, pe_v, lens_prev, lens, heads: Heads,
                       params: Params, k_cmp_pool, v_cmp_pool, cmp_block_table, ws, stream=None) -> int:
    """Paged caches: pools [n_pages, page_size, H_kv, d] and [n_cmp_pages,
    cmp_page_size, H_kv, d]; block tables device int32 [B, max_pages]; lens_prev
    (None: one token less; zeros: build from scratch) and lens host int32 [B].
    Returns the number of summaries written."""
    n = ctypes.c_int32(0)
    B = int(lens.numel())
    _check(lib().nsa_compress_paged(_ptr(k_pool, torch.bfloat16), _ptr(v_pool, torch.bfloat16), int(k_pool.shape[0]),
                                    int(k_pool.shape[1]), _ptr(block_table, torch.int32), int(block_table.shape[1]),
                                    _ptr(w_ck, torch.float32), _ptr(pe_k, torch.float32), _ptr(w_cv, torch.float32),
                                    _ptr(pe_v, torch.float32), _ptr(lens_prev, torch.int32, "cpu"),
                                    _ptr(lens, torch.int32, "cpu"), B, _ptr(k_cmp_pool, torch.bfloat16),
                                    _ptr(v_cmp_pool, torch.bfloat16), int(k_cmp_pool.shape[0]),
                                    int(k_cmp_pool.shape[1]), _ptr(cmp_block_table, torch.int32),
                                    int(cmp_block_table.shape[1]), ctypes.byref(heads), ctypes.byref(params),
                                    ctypes.byref(n), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "nsa_compress_paged")
    return int(n.value)


def nsa_decode_paged(q, k_pool, v_pool, block_table, k_cmp_pool, v_cmp_pool, cmp_block_table, cache_lens,
                     max_len: int, gates, heads: Heads, params: Params, out, sel_out=None, imp_out=None, ws=None,
                     stream=None):
    """Paged decode (layouts as nsa_compress_paged); cache_lens device int32 [B]."""
    B = int(q.shape[0])
    _check(lib().nsa_decode_paged(_ptr(q, torch.bfloat16), _ptr(k_pool, torch.bfloat16), _ptr(v_pool, torch.bfloat16),
                                  int(k_pool.shape[0]), int(k_pool.shape[1]), _ptr(block_table, torch.int32),
                                  int(block_table.shape[1]), _ptr(k_cmp_pool, torch.bfloat16),
                                  _ptr(v_cmp_pool, torch.bfloat16), int(k_cmp_pool.shape[0]), int(k_cmp_pool.shape[1]),
                                  _ptr(cmp_block_table, torch.int32), int(cmp_block_table.shape[1]),
                                  _ptr(cache_lens, torch.int32), B, int(max_len), _ptr(gates, torch.float32),
                                  ctypes.byref(heads), ctypes.byref(params), _ptr(out, torch.bfloat16),
                                  _ptr(sel_out, torch.int32), _ptr(imp_out, torch.float32), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)), "nsa_decode_paged")


def nsa_prefill_backward(q, k, v, k_cmp, v_cmp, gates, dout, sel, w_ck, pe_k, w_cv, pe_v, cu_seqlens, heads: Heads,
                         params: Params, dq, dk, dv, dgates, dw_ck, dpe_k, dw_cv, dpe_v, ws, stream=None):
    """Gradients of the prefill with the selection held at `sel` (nsa_prefill's
    sel_out). dout bf16 [N, H_q, d_v]; every gradient fp32; cu_seqlens host int32."""
    B = int(cu_seqlens.numel()) - 1
    f32 = torch.float32
    _check(lib().nsa_prefill_backward(_ptr(q, torch.bfloat16), _ptr(k, torch.bfloat16), _ptr(v, torch.bfloat16),
                                      _ptr(k_cmp, torch.bfloat16), _ptr(v_cmp, torch.bfloat16), _ptr(gates, f32),
                                      _ptr(dout, torch.bfloat16), _ptr(sel, torch.int32), _ptr(w_ck, f32),
                                      _ptr(pe_k, f32), _ptr(w_cv, f32), _ptr(pe_v, f32),
                                      _ptr(cu_seqlens, torch.int32, "cpu"), B, ctypes.byref(heads),
                                      ctypes.byref(params), _ptr(dq, f32), _ptr(dk, f32), _ptr(dv, f32),
                                      _ptr(dgates, f32), _ptr(dw_ck, f32), _ptr(dpe_k, f32), _ptr(dw_cv, f32),
                                      _ptr(dpe_v, f32), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "nsa_prefill_backward")


def nsa_dsa_workspace_size(op: int, heads: Heads, dp: DsaParams, batch: int, total_tokens: int, max_len: int) -> int:
    return int(lib().nsa_dsa_workspace_size(op, ctypes.byref(heads), ctypes.byref(dp), batch, total_tokens, max_len))


def nsa_dsa_decode(q, k_cache, v_cache, qi, wi, ki_cache, cache_lens, max_len: int, dp: DsaParams, heads: Heads, out,
                   idx_out=None, score_out=None, ws=None, stream=None):
    """DSA decode: q [B, H_q, d_k]; caches [B, Lmax, H_kv, d]; qi fp8 [B, H_I, d_I];
    wi fp32 [B, H_I]; ki_cache fp8 [B, Lmax, d_I]; cache_lens device int32 [B]."""
    B, Lmax = int(k_cache.shape[0]), int(k_cache.shape[1])
    f8 = torch.float8_e4m3fn
    _check(lib().nsa_dsa_decode(_ptr(q, torch.bfloat16), _ptr(k_cache, torch.bfloat16), _ptr(v_cache, torch.bfloat16),
                                _ptr(qi, f8), _ptr(wi, torch.float32), _ptr(ki_cache, f8),
                                _ptr(cache_lens, torch.int32), B, Lmax, int(max_len), ctypes.byref(dp),
                                ctypes.byref(heads), _ptr(out, torch.bfloat16), _ptr(idx_out, torch.int32),
                                _ptr(score_out, torch.float32), _ptr(ws), ws.numel() * ws.element_size(),
                                _stream(stream)), "nsa_dsa_decode")


def nsa_dsa_prefill(q, k, v, qi, wi, ki, cu_seqlens, dp: DsaParams, heads: Heads, out, idx_out=None, score_out=None,
                    ws=None, stream=None):
    """DSA prefill over packed sequences; cu_seqlens host int32 [B+1]."""
    B = int(cu_seqlens.numel()) - 1
    f8 = torch.float8_e4m3fn
    _check(lib().nsa_dsa_prefill(_ptr(q, torch.bfloat16), _ptr(k, torch.bfloat16), _ptr(v, torch.bfloat16),
                                 _ptr(qi, f8), _ptr(wi, torch.float32), _ptr(ki, f8),
                                 _ptr(cu_seqlens, torch.int32, "cpu"), B, ctypes.byref(dp), ctypes.byref(heads),
                                 _ptr(out, torch.bfloat16), _ptr(idx_out, torch.int32), _ptr(score_out, torch.float32),
                                 _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "nsa_dsa_prefill")


def nsa_profile_enable(enable: bool):
    _check(lib().nsa_profile_enable(1 if enable else 0), "nsa_profile_enable")


def nsa_profile_read() -> dict:
    """{slot name: (total ms, launches)} accumulated since the previous read."""
    n = NSA_PROFILE_SLOTS
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    _check(lib().nsa_profile_read(ms, cnt, n), "nsa_profile_read")
    return {lib().nsa_profile_slot_name(i).decode(): (float(ms[i]), int(cnt[i])) for i in range(n)}


# ---------------------------------------------------------------------------
# convenience helpers (allocation with torch, then the entry points)
# ---------------------------------------------------------------------------

def n_cmp(L: int, l: int = 32, s: int = 16) -> int:
    return (L - l) // s + 1 if L >= l else 0


def n_blk(L: int, l_sel: int = 64) -> int:
    return -(-L // l_sel)


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    nsa_workspace_init(ws)
    return ws


def compress_prepare(w_ck, pe_k, w_cv, pe_v, heads: Heads, params: Params) -> torch.Tensor:
    """The compression weights in prepared form (a device byte tensor)."""
    prepared = torch.empty(nsa_compress_weights_size(heads, params), dtype=torch.uint8, device=w_ck.device)
    nsa_compress_prepare(w_ck, pe_k, w_cv, pe_v, heads, params, prepared)
    return prepared


def compress(k, v, w_ck, pe_k, w_cv, pe_v, seqlens, heads: Heads, params: Params, ws=None, out=None, prepared=None):
    """Packed prefill layout: sequences back to back in k/v. Returns (k_cmp, v_cmp).
    With `prepared` (from compress_prepare) the weight arguments are not read."""
    seqlens = [int(x) for x in seqlens]
    tok = torch.tensor([sum(seqlens[:b]) for b in range(len(seqlens))], dtype=torch.int64)
    ncs = [n_cmp(L, params.l_cmp, params.stride) for L in seqlens]
    cmp_off = torch.tensor([sum(ncs[:b]) for b in range(len(ncs))], dtype=torch.int64)
    total = sum(ncs)
    dev = k.device
    if out is None:
        k_cmp = torch.empty((max(total, 1), heads.H_kv, heads.d_k), dtype=torch.bfloat16, device=dev)
        v_cmp = torch.empty((max(total, 1), heads.H_kv, heads.d_v), dtype=torch.bfloat16, device=dev)
    else:
        k_cmp, v_cmp = out
    if ws is None:
        ws = alloc_workspace(nsa_workspace_size(NSA_OP_COMPRESS, heads, params, len(seqlens), sum(seqlens), 0),
                             dev)
    if prepared is not None:
        nsa_compress_prepared(k, v, prepared, tok, torch.tensor(seqlens, dtype=torch.int32), cmp_off, heads, params,
                              k_cmp, v_cmp, ws)
    else:
        nsa_compress(k, v, w_ck, pe_k, w_cv, pe_v, tok, torch.tensor(seqlens, dtype=torch.int32), cmp_off, heads,
                     params, k_cmp, v_cmp, ws)
    return k_cmp[:total], v_cmp[:total]


def compress_cache(k_cache, v_cache, w_ck, pe_k, w_cv, pe_v, lens, heads: Heads, params: Params, ws=None):
    """Compressed caches [B, Lmax_cmp, H_kv, d] for batched caches [B, Lmax, H_kv, d]."""
    B, Lmax = int(k_cache.shape[0]), int(k_cache.shape[1])
    Lc = max(n_cmp(Lmax, params.l_cmp, params.stride), 1)
    dev = k_cache.device
    kc = torch.zeros((B, Lc, heads.H_kv, heads.d_k), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros((B, Lc, heads.H_kv, heads.d_v), dtype=torch.bfloat16, device=dev)
    lens_l = [int(x) for x in (lens.tolist() if hasattr(lens, "tolist") else lens)]
    if ws is None:
        ws = alloc_workspace(nsa_workspace_size(NSA_OP_COMPRESS, heads, params, B, 0, 0), dev)
    nsa_compress(k_cache, v_cache, w_ck, pe_k, w_cv, pe_v,
                 torch.tensor([b * Lmax for b in range(B)], dtype=torch.int64),
                 torch.tensor(lens_l, dtype=torch.int32),
                 torch.tensor([b * Lc for b in range(B)], dtype=torch.int64), heads, params, kc, vc, ws)
    return kc, vc


def nsa_compress_append_plan(lens_prev, lens, Lmax: int, Lmax_cmp: int, params: Params):
    """Host-only plan of the blocks completed by growth (C ABI of the same name).
    lens_prev/lens: host int32 [B] (lens_prev may be None: one new token).
    Returns (tok_offset int64 [B], seq_len int32 [B], cmp_offset int64 [B], n_blocks)."""
    B = int(lens.numel())
    tok = torch.empty(B, dtype=torch.int64)
    sl = torch.empty(B, dtype=torch.int32)
    co = torch.empty(B, dtype=torch.int64)
    n = ctypes.c_int32(0)
    _check(lib().nsa_compress_append_plan(_ptr(lens_prev, torch.int32, "cpu"), _ptr(lens, torch.int32, "cpu"), B,
                                          int(Lmax), int(Lmax_cmp), ctypes.byref(params), _ptr(tok, None, "cpu"),
                                          _ptr(sl, None, "cpu"), _ptr(co, None, "cpu"), ctypes.byref(n)),
           "nsa_compress_append_plan")
    return tok, sl, co, int(n.value)


def nsa_compress_append(k_cache, v_cache, w_ck, pe_k, w_cv, pe_v, lens_prev, lens, heads: Heads, params: Params,
                        k_cmp_cache, v_cmp_cache, ws, stream=None) -> int:
    """Incremental decode: write the summaries of every block completed while the
    batched caches grew from lens_prev (None: one token less) to lens, in place.
    lens_prev/lens: host int32 [B]. Returns the number of summaries written."""
    B, Lmax = int(k_cache.shape[0]), int(k_cache.shape[1])
    n = ctypes.c_int32(0)
    _check(lib().nsa_compress_append(_ptr(k_cache, torch.bfloat16), _ptr(v_cache, torch.bfloat16),
                                     _ptr(w_ck, torch.float32), _ptr(pe_k, torch.float32), _ptr(w_cv, torch.float32),
                                     _ptr(pe_v, torch.float32), _ptr(lens_prev, torch.int32, "cpu"),
                                     _ptr(lens, torch.int32, "cpu"), B, Lmax, int(k_cmp_cache.shape[1]),
                                     ctypes.byref(heads), ctypes.byref(params), _ptr(k_cmp_cache, torch.bfloat16),
                                     _ptr(v_cmp_cache, torch.bfloat16), ctypes.byref(n), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)), "nsa_compress_append")
    return int(n.value)


def _host_i32(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.to("cpu", torch.int32).contiguous()
    return torch.tensor([int(v) for v in x], dtype=torch.int32)


def append_plan(lens, Lmax: int, Lmax_cmp: int, l: int = 32, s: int = 16, lens_prev=None):
    """Lists (tok_offset, seq_len, cmp_offset) of nsa_compress_append_plan."""
    tok, sl, co, _ = nsa_compress_append_plan(_host_i32(lens_prev), _host_i32(lens), Lmax, Lmax_cmp,
                                              make_params(l_cmp=l, stride=s))
    return tok.tolist(), sl.tolist(), co.tolist()


def compress_append(k_cache, v_cache, w_ck, pe_k, w_cv, pe_v, lens, k_cmp, v_cmp, heads: Heads, params: Params,
                    ws=None, lens_prev=None) -> int:
    """nsa_compress_append with the workspace allocated when not given. Returns
    the number of blocks written (0: nothing to do, no launch)."""
    if ws is None:
        ws = alloc_workspace(nsa_workspace_size(NSA_OP_COMPRESS, heads, params, int(k_cache.shape[0]), 0, 0),
                             k_cache.device)
    return nsa_compress_append(k_cache, v_cache, w_ck, pe_k, w_cv, pe_v, _host_i32(lens_prev), _host_i32(lens),
                               heads, params, k_cmp, v_cmp, ws)


def prefill(q, k, v, k_cmp, v_cmp, gates, cu_seqlens, heads: Heads, params: Params, ws=None, want_sel=False,
            want_imp=False):
    """Returns out (and sel / imp when asked)."""
    cu = cu_seqlens.to("cpu", torch.int32).contiguous()
    B = cu.numel() - 1
    N = int(cu[-1])
    max_len = int((cu[1:] - cu[:-1]).max()) if B > 0 else 0
    dev = q.device
    out = torch.empty((N, heads.H_q, heads.d_v), dtype=torch.bfloat16, device=dev)
    sel = torch.empty((N, heads.H_kv, params.top_n), dtype=torch.int32, device=dev) if want_sel else None
    imp = (torch.zeros((N, heads.H_kv, n_blk(max_len, params.l_sel)), dtype=torch.float32, device=dev)
           if want_imp else None)
    if ws is None:
        ws = alloc_workspace(nsa_workspace_size(NSA_OP_PREFILL, heads, params, B, N, max_len), dev)
    nsa_prefill(q, k, v, k_cmp, v_cmp, gates, cu, heads, params, out, sel, imp, ws)
    res = [out]
    if want_sel:
        res.append(sel)
    if want_imp:
        res.append(imp)
    return res[0] if len(res) == 1 else tuple(res)


def decode(q, k_cache, v_cache, k_cmp_cache, v_cmp_cache, cache_lens_dev, max_len, gates, heads: Heads,
           params: Params, ws=None, want_sel=False, want_imp=False):
    B = int(q.shape[0])
    dev = q.device
    out = torch.empty((B, heads.H_q, heads.d_v), dtype=torch.bfloat16, device=dev)
    sel = torch.empty((B, heads.H_kv, params.top_n), dtype=torch.int32, device=dev) if want_sel else None
    imp = (torch.zeros((B, heads.H_kv, n_blk(max_len, params.l_sel)), dtype=torch.float32, device=dev)
           if want_imp else None)
    if ws is None:
        ws = alloc_workspace(nsa_workspace_size(NSA_OP_DECODE, heads, params, B, 0, max_len), dev)
    nsa_decode(q, k_cache, v_cache, k_cmp_cache, v_cmp_cache, cache_lens_dev, max_len, gates, heads, params, out,
               sel, imp, ws)
    res = [out]
    if want_sel:
        res.append(sel)
    if want_imp:
        res.append(imp)
    return res[0] if len(res) == 1 else tuple(res)


def prefill_backward(q, k, v, k_cmp, v_cmp, gates, dout, sel, w_ck, pe_k, w_cv, pe_v, cu_seqlens, heads: Heads,
                     params: Params, ws=None) -> dict:
    """Allocates the gradients (fp32) and the workspace, calls nsa_prefill_backward."""
    cu = cu_seqlens.to("cpu", torch.int32).contiguous()
    B = cu.numel() - 1
    N = int(cu[-1])
    max_len = int((cu[1:] - cu[:-1]).max()) if B > 0 else 0
    dev = q.device
    g = dict(dq=torch.empty_like(q, dtype=torch.float32), dk=torch.empty_like(k, dtype=torch.float32),
             dv=torch.empty_like(v, dtype=torch.float32), dgates=torch.empty_like(gates),
             dw_ck=torch.empty_like(w_ck), dpe_k=torch.empty_like(pe_k), dw_cv=torch.empty_like(w_cv),
             dpe_v=torch.empty_like(pe_v))
    if ws is None:
        ws = alloc_workspace(nsa_workspace_size(NSA_OP_BACKWARD, heads, params, B, N, max_len), dev)
    nsa_prefill_backward(q, k, v, k_cmp, v_cmp, gates, dout, sel, w_ck, pe_k, w_cv, pe_v, cu, heads, params,
                         g["dq"], g["dk"], g["dv"], g["dgates"], g["dw_ck"], g["dpe_k"], g["dw_cv"], g["dpe_v"], ws)
    return g


def default_scale(d_k: int) -> float:
    return 1.0 / math.sqrt(d_k)
