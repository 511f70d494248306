"""The checking build on the GPU, and output buffers surrounded by canaries.

* libnsa_check.so (index checks that record a bounds error in the status word,
  test fault injection, 20 ms wait limit; include/nsa_check.h) runs prefill and
  decode parity cases: no index check fires and the results match the oracle.
* Output buffers with canary rows before and after them: no kernel writes
  outside the rows it was given (both builds).
* The failure path of the bounded waits: a producer withholds one tile, the
  kernel's waits on it run out, the kernel records a timeout and returns;
  nsa_check_device_status reports NSA_ERR_DEVICE_CHECK, clears the word, and the
  next call on the same context computes the right result. No fault, trap or
  endless wait is involved: every wait is bounded in time.
"""
import time

import numpy as np
import pytest
import torch

import nsa_workloads as W
import sparse_attention_long_nsa_b200 as nsa
from tests import nsa_parity as NP

pytestmark = pytest.mark.gpu

CFG = W.CONFIGS
PAD = 7   # canary rows on each side


def test_checking_build_parity_no_bounds_errors():
    with nsa.checking_library():
        NP.run_prefill_case(CFG["prefill_tiny_1k"], [1024, 300, 31], n_random_rows=256)
        NP.run_prefill_case(CFG["prefill_8k"], [1500, 700], n_random_rows=64, seed=11)
        NP.run_decode_case(CFG["decode_64k"], [20000, 3000, 33, 1], seed=3, cmp_rows=[1])


def _canary(shape, dtype):
    """A buffer with PAD extra rows on each side, every byte set to a pattern;
    returns (whole buffer, the interior view handed to the library)."""
    full = torch.empty((shape[0] + 2 * PAD,) + tuple(shape[1:]), dtype=dtype, device="cuda")
    full.view(torch.uint8).fill_(0xA7)
    return full, full[PAD:PAD + shape[0]]


def _pads_intact(full):
    b = full.view(torch.uint8)
    rows = b.reshape(full.shape[0], -1)
    return bool((rows[:PAD] == 0xA7).all()) and bool((rows[-PAD:] == 0xA7).all())


@pytest.mark.parametrize("checking", [False, True])
def test_outputs_leave_canary_rows_untouched(checking):
    cfg = CFG["prefill_8k"]
    seqlens = [700, 64, 1300]
    heads, par = NP.heads_of(cfg), NP.params_of(cfg)
    ctx = nsa.checking_library() if checking else _null()
    with ctx:
        inp = W.make_prefill_inputs(cfg, device="cuda", seqlens=seqlens, seed=17)
        kc, vc = nsa.compress(inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], seqlens,
                              heads, par)
        N, mx = sum(seqlens), max(seqlens)
        ref_out, ref_sel = nsa.prefill(inp["q"], inp["k"], inp["v"], kc, vc, inp["gates"], inp["cu_seqlens"], heads,
                                       par, want_sel=True)
        fo, o = _canary((N, cfg.H_q, cfg.d_v), torch.bfloat16)
        fs, s_ = _canary((N, cfg.H_kv, cfg.top_n), torch.int32)
        fi, i_ = _canary((N, cfg.H_kv, nsa.n_blk(mx)), torch.float32)
        ws = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_PREFILL, heads, par, len(seqlens), N, mx), "cuda")
        nsa.nsa_prefill(inp["q"], inp["k"], inp["v"], kc, vc, inp["gates"], inp["cu_seqlens"], heads, par, o, s_, i_,
                        ws)
        torch.cuda.synchronize()
        nsa.nsa_check_device_status(ws)
        assert _pads_intact(fo) and _pads_intact(fs) and _pads_intact(fi)
        assert torch.equal(s_, ref_sel)
        assert torch.equal(o, ref_out)

        dcfg = CFG["decode_64k"]
        dinp = W.make_decode_inputs(dcfg, device="cuda", lens=[9000, 33, 4100], seed=19)
        kcc, vcc = nsa.compress_cache(dinp["k_cache"], dinp["v_cache"], dinp["w_ck"], dinp["pe_k"], dinp["w_cv"],
                                      dinp["pe_v"], dinp["cache_lens"], heads, par)
        B, Lmax = 3, int(dinp["k_cache"].shape[1])
        lens = dinp["cache_lens"].to("cuda")
        ref_d, ref_ds = nsa.decode(dinp["q"], dinp["k_cache"], dinp["v_cache"], kcc, vcc, lens, Lmax, dinp["gates"],
                                   heads, par, want_sel=True)
        fo, o = _canary((B, dcfg.H_q, dcfg.d_v), torch.bfloat16)
        fs, s_ = _canary((B, dcfg.H_kv, dcfg.top_n), torch.int32)
        fi, i_ = _canary((B, dcfg.H_kv, nsa.n_blk(Lmax)), torch.float32)
        ws = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_DECODE, heads, par, B, 0, Lmax), "cuda")
        nsa.nsa_decode(dinp["q"], dinp["k_cache"], dinp["v_cache"], kcc, vcc, lens, Lmax, dinp["gates"], heads, par,
                       o, s_, i_, ws)
        torch.cuda.synchronize()
        nsa.nsa_check_device_status(ws)
        assert _pads_intact(fo) and _pads_intact(fs) and _pads_intact(fi)
        assert torch.equal(s_, ref_ds)
        assert torch.equal(o, ref_d)


class _null:
    def __enter__(self):
        return None

    def __exit__(self, *a):
        return False


def _expect_timeout(ws):
    with pytest.raises(nsa.NSAError) as ei:
        nsa.nsa_check_device_status(ws)
    assert ei.value.status == nsa.NSA_ERR_DEVICE_CHECK
    assert "status 0x1" in str(ei.value), str(ei.value)
    nsa.nsa_check_device_status(ws)   # the word was cleared


def test_bounded_wait_failure_path_decode():
    cfg = CFG["decode_64k"]
    heads, par = NP.heads_of(cfg), NP.params_of(cfg)
    inp = W.make_decode_inputs(cfg, device="cuda", lens=[5000, 70000], seed=5)
    lens = inp["cache_lens"].to("cuda")
    Lmax = int(inp["k_cache"].shape[1])
    kc, vc = nsa.compress_cache(inp["k_cache"], inp["v_cache"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"],
                                inp["cache_lens"], heads, par)
    ref, ref_sel = nsa.decode(inp["q"], inp["k_cache"], inp["v_cache"], kc, vc, lens, Lmax, inp["gates"], heads, par,
                              want_sel=True)
    with nsa.checking_library():
        ws = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_DECODE, heads, par, 2, 0, Lmax), "cuda")
        nsa.nsa_test_set_fault(nsa.FAULT_DECODE_FINE_TILE)
        t0 = time.time()
        try:
            nsa.decode(inp["q"], inp["k_cache"], inp["v_cache"], kc, vc, lens, Lmax, inp["gates"], heads, par, ws=ws)
            torch.cuda.synchronize()
        finally:
            nsa.nsa_test_set_fault(nsa.FAULT_NONE)
        assert time.time() - t0 < 10.0
        _expect_timeout(ws)
        out, sel = nsa.decode(inp["q"], inp["k_cache"], inp["v_cache"], kc, vc, lens, Lmax, inp["gates"], heads,
                              par, ws=ws, want_sel=True)
        torch.cuda.synchronize()
        nsa.nsa_check_device_status(ws)
    assert torch.equal(sel, ref_sel)
    NP.assert_close(NP.f64(out), NP.f64(ref), "decode after a recorded timeout")


def test_bounded_wait_failure_path_prefill():
    cfg = CFG["prefill_8k"]
    seqlens = [900, 2000]
    heads, par = NP.heads_of(cfg), NP.params_of(cfg)
    inp = W.make_prefill_inputs(cfg, device="cuda", seqlens=seqlens, seed=6)
    kc, vc = nsa.compress(inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], seqlens, heads,
                          par)
    ref, ref_sel = nsa.prefill(inp["q"], inp["k"], inp["v"], kc, vc, inp["gates"], inp["cu_seqlens"], heads, par,
                               want_sel=True)
    N, mx = sum(seqlens), max(seqlens)
    with nsa.checking_library():
        ws = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_PREFILL, heads, par, 2, N, mx), "cuda")
        nsa.nsa_test_set_fault(nsa.FAULT_PREFILL_K_TILE)
        t0 = time.time()
        try:
            nsa.prefill(inp["q"], inp["k"], inp["v"], kc, vc, inp["gates"], inp["cu_seqlens"], heads, par, ws=ws)
            torch.cuda.synchronize()
        finally:
            nsa.nsa_test_set_fault(nsa.FAULT_NONE)
        assert time.time() - t0 < 10.0
        _expect_timeout(ws)
        out, sel = nsa.prefill(inp["q"], inp["k"], inp["v"], kc, vc, inp["gates"], inp["cu_seqlens"], heads, par,
                               ws=ws, want_sel=True)
        torch.cuda.synchronize()
        nsa.nsa_check_device_status(ws)
    assert torch.equal(sel, ref_sel)
    NP.assert_close(NP.f64(out), NP.f64(ref), "prefill after a recorded timeout")
