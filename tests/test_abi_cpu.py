"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, validates arguments on the host and sizes workspaces."""
import ctypes
import os
import re

import pytest

import sparse_attention_long_nsa_b200 as nsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions(name="nsa.h"):
    src = open(os.path.join(ROOT, "include", name)).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nsa_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(nsa.LIB_PATH):
        from sparse_attention_long_nsa_b200 import build
        build.build()
    return nsa.lib()


def test_exports_every_declared_symbol(L):
    declared = _header_functions()
    assert declared, "no functions parsed from include/nsa.h"
    assert set(declared) == set(nsa.EXPORTED)
    for name in declared:
        assert hasattr(L, name), name


def test_checking_build_exports(L):
    """libnsa_check.so exports what nsa.h and nsa_check.h declare; the library
    build does not export the test-only fault setter."""
    if not os.path.exists(nsa.CHECK_LIB_PATH):
        from sparse_attention_long_nsa_b200 import build
        build.build_check()
    C = ctypes.CDLL(nsa.CHECK_LIB_PATH)
    declared = set(_header_functions("nsa.h")) | set(_header_functions("nsa_check.h"))
    assert declared == set(nsa.CHECK_EXPORTED)
    for name in declared:
        assert hasattr(C, name), name
    assert not hasattr(L, "nsa_test_set_fault")
    C.nsa_test_set_fault.restype = ctypes.c_int
    C.nsa_test_set_fault.argtypes = [ctypes.c_int32]
    assert C.nsa_test_set_fault(99) == nsa.NSA_ERR_INVALID_ARG
    assert C.nsa_test_set_fault(0) == nsa.NSA_OK


def test_status_strings(L):
    for s, name in enumerate(["NSA_OK", "NSA_ERR_INVALID_ARG", "NSA_ERR_UNSUPPORTED", "NSA_ERR_WORKSPACE",
                              "NSA_ERR_CUDA", "NSA_ERR_DEVICE_CHECK"]):
        assert nsa.status_name(s) == name


def test_workspace_size_host_only(L):
    h = nsa.Heads(64, 4, 192, 128)
    p = nsa.make_params(top_n=16, window=512)
    ws = nsa.nsa_workspace_size(nsa.NSA_OP_PREFILL, h, p, 1, 8192, 8192)
    # importance [N,Hkv,128] + selection [N,Hkv,16] (the fused kernel keeps its accumulators on chip)
    assert ws >= 8192 * 4 * 128 * 4 + 8192 * 4 * 16 * 4
    assert ws < 8192 * 64 * 128 * 4
    assert nsa.nsa_workspace_size(nsa.NSA_OP_COMPRESS, h, p, 1, 0, 0) > 32 * 192 * 192 * 2
    assert nsa.nsa_workspace_size(nsa.NSA_OP_DECODE, h, p, 32, 0, 65536) > 0
    # invalid / unsupported arguments give 0
    assert nsa.nsa_workspace_size(nsa.NSA_OP_PREFILL, nsa.Heads(64, 5, 192, 128), p, 1, 10, 10) == 0
    assert nsa.nsa_workspace_size(nsa.NSA_OP_PREFILL, nsa.Heads(64, 4, 100, 128), p, 1, 10, 10) == 0
    assert nsa.nsa_workspace_size(nsa.NSA_OP_PREFILL, h, nsa.make_params(top_n=2), 1, 10, 10) == 0
    assert nsa.nsa_workspace_size(7, h, p, 1, 10, 10) == 0


def _call_prefill(L, heads, params, cu, ptr=16, ws_bytes=1 << 30, batch=None):
    cu_arr = (ctypes.c_int32 * len(cu))(*cu)
    P = ctypes.c_void_p(ptr)
    return L.nsa_prefill(P, P, P, P, P, P, cu_arr, len(cu) - 1 if batch is None else batch, ctypes.byref(heads),
                         ctypes.byref(params), P, None, None, P, ws_bytes, None)


def test_prefill_argument_validation_launches_nothing(L):
    h = nsa.Heads(64, 4, 192, 128)
    p = nsa.make_params()
    assert _call_prefill(L, h, p, [0, 100], ptr=0) == nsa.NSA_ERR_INVALID_ARG          # null pointers
    assert _call_prefill(L, h, p, [0, 100], ptr=8) == nsa.NSA_ERR_INVALID_ARG          # misaligned
    assert _call_prefill(L, h, p, [1, 100]) == nsa.NSA_ERR_INVALID_ARG                 # cu_seqlens[0] != 0
    assert _call_prefill(L, h, p, [0, 100, 50]) == nsa.NSA_ERR_INVALID_ARG             # decreasing
    assert _call_prefill(L, h, p, [0, 100], batch=0) == nsa.NSA_ERR_INVALID_ARG
    assert _call_prefill(L, h, p, [0, 100], ws_bytes=16) == nsa.NSA_ERR_WORKSPACE
    assert _call_prefill(L, nsa.Heads(64, 4, 96, 128), p, [0, 100]) == nsa.NSA_ERR_UNSUPPORTED
    assert _call_prefill(L, nsa.Heads(60, 4, 192, 128), p, [0, 100]) == nsa.NSA_ERR_UNSUPPORTED   # G = 15
    assert _call_prefill(L, nsa.Heads(64, 3, 192, 128), p, [0, 100]) == nsa.NSA_ERR_INVALID_ARG
    assert _call_prefill(L, h, nsa.make_params(l_cmp=30), [0, 100]) == nsa.NSA_ERR_INVALID_ARG   # l % s != 0
    assert _call_prefill(L, h, nsa.make_params(l_sel=40), [0, 100]) == nsa.NSA_ERR_INVALID_ARG   # l' % s != 0
    assert _call_prefill(L, h, nsa.make_params(top_n=2), [0, 100]) == nsa.NSA_ERR_INVALID_ARG    # n < forced
    assert _call_prefill(L, h, nsa.make_params(l_cmp=64, stride=32), [0, 100]) == nsa.NSA_ERR_UNSUPPORTED
    assert _call_prefill(L, h, nsa.make_params(top_n=40), [0, 100]) == nsa.NSA_ERR_UNSUPPORTED


def test_decode_and_compress_validation(L):
    h = nsa.Heads(64, 4, 192, 128)
    p = nsa.make_params()
    P = ctypes.c_void_p(16)
    # max_len above Lmax
    assert L.nsa_decode(P, P, P, P, P, P, 2, 100, 5, 200, P, ctypes.byref(h), ctypes.byref(p), P, None, None, P,
                        1 << 30, None) == nsa.NSA_ERR_INVALID_ARG
    # compressed cache too short for max_len
    assert L.nsa_decode(P, P, P, P, P, P, 2, 1000, 5, 1000, P, ctypes.byref(h), ctypes.byref(p), P, None, None, P,
                        1 << 30, None) == nsa.NSA_ERR_INVALID_ARG
    # window too large for the decode union buffer
    assert L.nsa_decode(P, P, P, P, P, P, 2, 1000, 61, 1000, P, ctypes.byref(h),
                        ctypes.byref(nsa.make_params(window=8192)), P, None, None, P, 1 << 30,
                        None) == nsa.NSA_ERR_UNSUPPORTED
    i64 = (ctypes.c_int64 * 1)(0)
    i32 = (ctypes.c_int32 * 1)(-5)
    assert L.nsa_compress(P, P, P, P, P, P, i64, i32, i64, 1, ctypes.byref(h), ctypes.byref(p), P, P, P, 1 << 30,
                          None) == nsa.NSA_ERR_INVALID_ARG
    i32[0] = 100
    assert L.nsa_compress(P, P, P, P, P, P, i64, i32, i64, 1, ctypes.byref(h), ctypes.byref(p), P, P, P, 8,
                          None) == nsa.NSA_ERR_WORKSPACE


def test_prepared_weights_validate_on_host(L):
    """The prepared-weights entry points size their blob and reject bad arguments
    before any launch (fake device pointers are never dereferenced)."""
    h = nsa.Heads(64, 4, 192, 128)
    p = nsa.make_params()
    n = L.nsa_compress_weights_size(ctypes.byref(h), ctypes.byref(p))
    # bf16 W^T of both maps and the fp32 position terms at least
    assert n >= 2 * (32 * 192 * 192 + 32 * 128 * 128) + 4 * (192 + 128)
    assert L.nsa_compress_weights_size(ctypes.byref(nsa.Heads(64, 5, 192, 128)), ctypes.byref(p)) == 0
    fake = ctypes.c_void_p(1 << 20)
    assert L.nsa_compress_prepare(fake, fake, fake, fake, ctypes.byref(h), ctypes.byref(p), None, n,
                                  None) == nsa.NSA_ERR_INVALID_ARG
    assert L.nsa_compress_prepare(fake, fake, fake, fake, ctypes.byref(h), ctypes.byref(p),
                                  ctypes.c_void_p((1 << 20) + 16), n, None) == nsa.NSA_ERR_INVALID_ARG
    assert L.nsa_compress_prepare(fake, fake, fake, fake, ctypes.byref(h), ctypes.byref(p), fake, n - 1,
                                  None) == nsa.NSA_ERR_WORKSPACE
    i64 = (ctypes.c_int64 * 1)(0)
    i32 = (ctypes.c_int32 * 1)(100)
    assert L.nsa_compress_prepared(fake, fake, None, i64, i32, i64, 1, ctypes.byref(h), ctypes.byref(p), fake, fake,
                                   fake, 1 << 30, None) == nsa.NSA_ERR_INVALID_ARG
    assert L.nsa_compress_prepared(fake, fake, fake, i64, i32, i64, 1, ctypes.byref(h), ctypes.byref(p), fake, fake,
                                   fake, 8, None) == nsa.NSA_ERR_WORKSPACE


def test_unsupported_head_sizes_rejected_on_host(L):
    """A value head size of 192 (or any size outside the built ones) is rejected
    before any launch."""
    P = ctypes.c_void_p(16)
    i64 = (ctypes.c_int64 * 1)(0)
    i32 = (ctypes.c_int32 * 1)(100)
    p = nsa.make_params()
    for h in (nsa.Heads(8, 2, 64, 192), nsa.Heads(8, 2, 192, 192), nsa.Heads(8, 2, 96, 64)):
        assert L.nsa_compress(P, P, P, P, P, P, i64, i32, i64, 1, ctypes.byref(h), ctypes.byref(p), P, P, P,
                              1 << 30, None) == nsa.NSA_ERR_UNSUPPORTED


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(nsa, "_lib", None)
    monkeypatch.setattr(nsa, "LIB_PATH", "/nonexistent/libnsa.so")
    with pytest.raises(ImportError):
        nsa.lib()


def test_append_plan_matches_block_counts():
    """Incremental decode: the newest token of a sequence of length L completes a
    compressed block exactly when n_cmp(L) = n_cmp(L - 1) + 1, and that block is
    number n_cmp(L) - 1 with tokens [i*s, i*s + l)."""
    import random
    rng = random.Random(5)
    for l, s in ((32, 16), (32, 32), (64, 16), (16, 8)):
        lens = [rng.randint(1, 3000) for _ in range(64)] + [l - 1, l, l + s - 1, l + s, 1]
        Lmax, Lc = 4096, nsa.n_cmp(4096, l, s)
        tok, sl, co = nsa.append_plan(lens, Lmax, Lc, l, s)
        for b, L in enumerate(lens):
            new_block = nsa.n_cmp(L, l, s) - nsa.n_cmp(L - 1, l, s)
            assert new_block in (0, 1)
            if new_block:
                i = nsa.n_cmp(L, l, s) - 1
                assert (sl[b], tok[b], co[b]) == (l, b * Lmax + i * s, b * Lc + i)
                assert i * s + l == L   # the block ends at the newest token
            else:
                assert sl[b] == 0


def test_append_plan_multi_token_growth():
    """Growth by several tokens: the segment holds exactly the blocks completed
    between the two lengths (the blocks nsa_compress finds in it)."""
    import random
    rng = random.Random(9)
    for l, s in ((32, 16), (32, 32), (64, 16)):
        prev = [rng.randint(0, 5000) for _ in range(64)] + [0, l - 1, l, 100]
        lens = [P + rng.choice([0, 1, 7, 16, 33, 500]) for P in prev]
        Lmax, Lc = 8192, nsa.n_cmp(8192, l, s)
        tok, sl, co = nsa.append_plan(lens, Lmax, Lc, l, s, lens_prev=prev)
        for b, (P, L) in enumerate(zip(prev, lens)):
            new = list(range(nsa.n_cmp(P, l, s), nsa.n_cmp(L, l, s)))
            got = [] if sl[b] == 0 else [(tok[b] - b * Lmax) // s + i for i in range(nsa.n_cmp(sl[b], l, s))]
            assert got == new
            if new:
                assert co[b] == b * Lc + new[0] and (tok[b] - b * Lmax) % s == 0
                assert (tok[b] - b * Lmax) + sl[b] <= L   # the segment ends inside the grown cache


def test_paged_entry_points_validate_on_host(L):
    """Page sizes that would let a selection block (64 tokens) or a tile of 32
    summaries straddle pages, missing tables and inconsistent lengths are
    rejected on the host, before any launch (fake device pointers are never
    dereferenced)."""
    h, p = nsa.Heads(64, 4, 192, 128), nsa.make_params()
    fake = ctypes.c_void_p(1 << 20)
    lens = (ctypes.c_int32 * 2)(100, 200)
    for page, cpage, table in ((48, 32, fake), (64, 16, fake), (64, 32, None), (0, 32, fake)):
        st = L.nsa_decode_paged(fake, fake, fake, 10, page, table, 8, fake, fake, 10, cpage, fake, 8, fake, 2, 200,
                                fake, ctypes.byref(h), ctypes.byref(p), fake, None, None, fake, 1 << 30, None)
        assert st == nsa.NSA_ERR_INVALID_ARG, (page, cpage)
        n = ctypes.c_int32(-1)
        st = L.nsa_compress_paged(fake, fake, 10, page, table, 8, fake, fake, fake, fake, None, lens, 2, fake, fake,
                                  10, cpage, fake, 8, ctypes.byref(h), ctypes.byref(p), ctypes.byref(n), fake,
                                  1 << 30, None)
        assert st == nsa.NSA_ERR_INVALID_ARG, (page, cpage)
    # lengths beyond the tables' capacity (8 pages of 64 tokens)
    big = (ctypes.c_int32 * 2)(100, 600)
    st = L.nsa_compress_paged(fake, fake, 10, 64, fake, 8, fake, fake, fake, fake, None, big, 2, fake, fake, 10, 32,
                              fake, 8, ctypes.byref(h), ctypes.byref(p), None, fake, 1 << 30, None)
    assert st == nsa.NSA_ERR_INVALID_ARG
    # append on a batched cache: lens above Lmax, lens_prev above lens
    st = L.nsa_compress_append(fake, fake, fake, fake, fake, fake, None, big, 2, 512, 31, ctypes.byref(h),
                               ctypes.byref(p), fake, fake, None, fake, 1 << 30, None)
    assert st == nsa.NSA_ERR_INVALID_ARG
    prev = (ctypes.c_int32 * 2)(101, 200)
    st = L.nsa_compress_append(fake, fake, fake, fake, fake, fake, prev, lens, 2, 512, 31, ctypes.byref(h),
                               ctypes.byref(p), fake, fake, None, fake, 1 << 30, None)
    assert st == nsa.NSA_ERR_INVALID_ARG


def _call_backward(L, heads, params, cu, ptr=16, ws_bytes=1 << 62, batch=None):
    cu_arr = (ctypes.c_int32 * len(cu))(*cu)
    P = ctypes.c_void_p(ptr)
    return L.nsa_prefill_backward(*([P] * 12), cu_arr, len(cu) - 1 if batch is None else batch, ctypes.byref(heads),
                                  ctypes.byref(params), *([P] * 8), P, ws_bytes, None)


def test_backward_argument_validation_launches_nothing(L):
    """Every call below is rejected on the host (or has no tokens), so nothing is
    launched and the fake pointers are never dereferenced."""
    h = nsa.Heads(64, 4, 192, 128)
    p = nsa.make_params()
    assert _call_backward(L, h, p, [0, 100], ptr=0) == nsa.NSA_ERR_INVALID_ARG           # null pointers
    assert _call_backward(L, h, p, [0, 100], ptr=8) == nsa.NSA_ERR_INVALID_ARG           # misaligned
    assert _call_backward(L, h, p, [3, 100]) == nsa.NSA_ERR_INVALID_ARG                  # cu_seqlens[0] != 0
    assert _call_backward(L, h, p, [0, 100, 40]) == nsa.NSA_ERR_INVALID_ARG              # negative length
    assert _call_backward(L, h, p, [0, 100], batch=0) == nsa.NSA_ERR_INVALID_ARG
    assert _call_backward(L, h, p, [0, 100], batch=nsa.NSA_MAX_BATCH + 1) == nsa.NSA_ERR_UNSUPPORTED
    assert _call_backward(L, h, p, [0, 100], ws_bytes=256) == nsa.NSA_ERR_WORKSPACE
    assert _call_backward(L, nsa.Heads(64, 4, 96, 128), p, [0, 100]) == nsa.NSA_ERR_UNSUPPORTED
    assert _call_backward(L, h, nsa.make_params(top_n=2), [0, 100]) == nsa.NSA_ERR_INVALID_ARG
    # a sequence whose block list does not fit the query kernel's shared memory
    assert _call_backward(L, h, p, [0, 1 << 26]) == nsa.NSA_ERR_UNSUPPORTED
    assert b"too long" in L.nsa_last_error_detail()
    # no tokens: valid, nothing to do
    assert _call_backward(L, h, p, [0, 0, 0]) == nsa.NSA_OK
    # the size query grows with the tokens and rejects what the entry point rejects
    small = nsa.nsa_workspace_size(nsa.NSA_OP_BACKWARD, h, p, 2, 300, 200)
    assert 0 < small < nsa.nsa_workspace_size(nsa.NSA_OP_BACKWARD, h, p, 2, 3000, 2000)
    assert nsa.nsa_workspace_size(nsa.NSA_OP_BACKWARD, nsa.Heads(64, 4, 96, 128), p, 2, 300, 200) == 0


def _dsa(H_I=8, d_I=128, top_k=2048, scale=0.0):
    return nsa.DsaParams(H_I, d_I, top_k, scale)


def test_dsa_workspace_size_host_only(L):
    h = nsa.Heads(64, 4, 192, 128)
    dp = _dsa()
    # decode: header + scores [batch, max_len] + kept tokens [batch, top_k], each 256-byte aligned
    def a256(x):
        return (x + 255) // 256 * 256
    assert nsa.nsa_dsa_workspace_size(nsa.NSA_OP_DSA_DECODE, h, dp, 32, 0, 65536) == \
        256 + a256(32 * 65536 * 4) + a256(32 * 2048 * 4)
    # prefill: the score rows of one chunk of queries fill at most 2^26 floats
    ws = nsa.nsa_dsa_workspace_size(nsa.NSA_OP_DSA_PREFILL, h, dp, 1, 8192, 8192)
    assert ws == 256 + a256(8192 * 8192 * 4) + a256(8192 * 2048 * 4)
    ws_long = nsa.nsa_dsa_workspace_size(nsa.NSA_OP_DSA_PREFILL, h, dp, 1, 65536, 65536)
    chunk = (1 << 26) // 65536
    assert ws_long == 256 + a256(chunk * 65536 * 4) + a256(chunk * 2048 * 4)
    for bad in (_dsa(H_I=0), _dsa(d_I=48), _dsa(H_I=17), _dsa(top_k=0), _dsa(top_k=65537), _dsa(scale=-1.0),
                _dsa(scale=float("nan"))):
        assert nsa.nsa_dsa_workspace_size(nsa.NSA_OP_DSA_DECODE, h, bad, 1, 0, 100) == 0
    assert nsa.nsa_dsa_workspace_size(nsa.NSA_OP_DSA_DECODE, h, dp, 0, 0, 100) == 0
    assert nsa.nsa_dsa_workspace_size(nsa.NSA_OP_DSA_DECODE, h, dp, 1, 0, 0) == 0
    assert nsa.nsa_dsa_workspace_size(nsa.NSA_OP_DSA_PREFILL, h, dp, 1, -1, 100) == 0
    assert nsa.nsa_dsa_workspace_size(nsa.NSA_OP_DECODE, h, dp, 1, 0, 100) == 0


def test_dsa_argument_validation_launches_nothing(L):
    """As for the backward: every call is rejected before a launch."""
    h = nsa.Heads(64, 4, 192, 128)
    dp = _dsa()

    def dec(ptr=16, batch=2, Lmax=1000, max_len=1000, dp=dp, heads=h, ws_bytes=1 << 40):
        P = ctypes.c_void_p(ptr)
        return L.nsa_dsa_decode(P, P, P, P, P, P, P, batch, Lmax, max_len, ctypes.byref(dp), ctypes.byref(heads), P,
                                None, None, P, ws_bytes, None)

    assert dec(ptr=0) == nsa.NSA_ERR_INVALID_ARG
    assert dec(ptr=8) == nsa.NSA_ERR_INVALID_ARG
    assert dec(batch=0) == nsa.NSA_ERR_INVALID_ARG
    assert dec(batch=nsa.NSA_MAX_BATCH + 1) == nsa.NSA_ERR_UNSUPPORTED
    assert dec(max_len=0) == nsa.NSA_ERR_INVALID_ARG
    assert dec(Lmax=500) == nsa.NSA_ERR_INVALID_ARG                     # max_len above Lmax
    assert dec(ws_bytes=1024) == nsa.NSA_ERR_WORKSPACE
    assert dec(dp=_dsa(d_I=96)) == nsa.NSA_ERR_UNSUPPORTED
    assert dec(dp=_dsa(top_k=-1)) == nsa.NSA_ERR_INVALID_ARG
    assert dec(heads=nsa.Heads(64, 4, 192, 96)) == nsa.NSA_ERR_UNSUPPORTED

    def pre(cu, ptr=16, ws_bytes=1 << 40, dp=dp, batch=None):
        cu_arr = (ctypes.c_int32 * len(cu))(*cu)
        P = ctypes.c_void_p(ptr)
        return L.nsa_dsa_prefill(P, P, P, P, P, P, cu_arr, len(cu) - 1 if batch is None else batch,
                                 ctypes.byref(dp), ctypes.byref(h), P, None, None, P, ws_bytes, None)

    assert pre([0, 100], ptr=0) == nsa.NSA_ERR_INVALID_ARG
    assert pre([0, 100], ptr=8) == nsa.NSA_ERR_INVALID_ARG
    assert pre([5, 100]) == nsa.NSA_ERR_INVALID_ARG
    assert pre([0, 100, 99]) == nsa.NSA_ERR_INVALID_ARG
    assert pre([0, 100], batch=0) == nsa.NSA_ERR_INVALID_ARG
    assert pre([0, 100], ws_bytes=4096) == nsa.NSA_ERR_WORKSPACE
    assert pre([0, 100], dp=_dsa(H_I=32)) == nsa.NSA_ERR_UNSUPPORTED
    assert pre([0, 0, 0]) == nsa.NSA_OK                                  # no tokens: nothing to do
