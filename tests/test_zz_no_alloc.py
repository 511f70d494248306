"""nsa_compress_noalloc: the compression entry point for callers that cannot
allocate device memory where they compress (graph capture in progress, a fixed
memory plan, a host framework that owns every allocation). Its scratch is a
fixed device array inside libnsa.so instead of a caller workspace.

Called through the C ABI twice in a row (the array keeps the previous call's
contents, so the second call checks that nothing stale leaks through) and
compared with nsa_compress, which takes an explicit workspace, and with the
fp64 oracle's compression, within the tolerance the parity tests use for
compressed K/V. Kept in a file of its own
that is collected last."""
import pytest
import torch

import nsa_workloads as W
import sparse_attention_long_nsa_b200 as nsa
from oracle import nsa_oracle as O
from tests import nsa_parity as NP

pytestmark = pytest.mark.gpu


def _offsets(seqlens, params):
    tok, cmp_, t, c = [], [], 0, 0
    for L in seqlens:
        tok.append(t)
        cmp_.append(c)
        t += L
        c += nsa.n_cmp(L, params.l_cmp, params.stride)
    return (torch.tensor(tok, dtype=torch.int64), torch.tensor(seqlens, dtype=torch.int32),
            torch.tensor(cmp_, dtype=torch.int64), c)


@pytest.mark.parametrize("cfg_name,seqlens", [("prefill_8k", [1500, 64, 700]), ("prefill_tiny_1k", [1024, 31, 333])])
def test_noalloc_matches_workspace_entry_point(cfg_name, seqlens):
    cfg = W.CONFIGS[cfg_name]
    heads, par = NP.heads_of(cfg), NP.params_of(cfg)
    tok, lens, cmp_off, total = _offsets(seqlens, par)
    ref_k = ref_v = None
    # reference: the workspace entry point
    inp = W.make_prefill_inputs(cfg, device="cuda", seqlens=seqlens, seed=123)
    ws = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_COMPRESS, heads, par, len(seqlens), 0, 0), "cuda")
    ref_k = torch.empty((total, cfg.H_kv, cfg.d_k), dtype=torch.bfloat16, device="cuda")
    ref_v = torch.empty((total, cfg.H_kv, cfg.d_v), dtype=torch.bfloat16, device="cuda")
    nsa.nsa_compress(inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], tok, lens, cmp_off,
                     heads, par, ref_k, ref_v, ws)
    torch.cuda.synchronize()
    for call in range(2):
        # different inputs for the first call, so a stale scratch would show
        if call == 0:
            other = W.make_prefill_inputs(cfg, device="cuda", seqlens=seqlens, seed=999)
            k_tmp = torch.empty_like(ref_k)
            v_tmp = torch.empty_like(ref_v)
            nsa.nsa_compress_noalloc(other["k"], other["v"], other["w_ck"], other["pe_k"], other["w_cv"],
                                     other["pe_v"], tok, lens, cmp_off, heads, par, k_tmp, v_tmp)
        k_out = torch.full_like(ref_k, float("nan"))
        v_out = torch.full_like(ref_v, float("nan"))
        nsa.nsa_compress_noalloc(inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], tok, lens,
                                 cmp_off, heads, par, k_out, v_out)
        torch.cuda.synchronize()
        NP.assert_close(NP.f64(k_out), NP.f64(ref_k), f"k_cmp (no-alloc call {call})", relative_to_rms=True)
        NP.assert_close(NP.f64(v_out), NP.f64(ref_v), f"v_cmp (no-alloc call {call})", relative_to_rms=True)
    # and against the fp64 oracle's own compression of every sequence
    op = NP.oracle_params(cfg)
    w_ck, pe_k, w_cv, pe_v = (NP.f64(inp[x]) for x in ("w_ck", "pe_k", "w_cv", "pe_v"))
    for b, L in enumerate(seqlens):
        t0, c0, nc = int(tok[b]), int(cmp_off[b]), nsa.n_cmp(L, par.l_cmp, par.stride)
        if nc == 0:
            continue
        kb, vb = NP.f64(inp["k"][t0:t0 + L]), NP.f64(inp["v"][t0:t0 + L])
        NP.assert_close(NP.f64(k_out[c0:c0 + nc]), O.compress(kb, w_ck, pe_k, op["l_cmp"], op["stride"]),
                        "k_cmp (no-alloc) vs oracle", relative_to_rms=True)
        NP.assert_close(NP.f64(v_out[c0:c0 + nc]), O.compress(vb, w_cv, pe_v, op["l_cmp"], op["stride"]),
                        "v_cmp (no-alloc) vs oracle", relative_to_rms=True)


def test_noalloc_under_graph_capture():
    """After one eager call (which resolves the scratch address), the call is
    captured into a CUDA graph and replayed on new inputs copied into the captured
    tensors. Neither an eager call nor a replay allocates (torch's allocator and
    the device's free memory are unchanged across them); the replay matches
    nsa_compress on the new inputs, and the status word reads clean."""
    cfg = W.CONFIGS["prefill_tiny_1k"]
    seqlens = [1024, 31, 333]
    heads, par = NP.heads_of(cfg), NP.params_of(cfg)
    tok, lens, cmp_off, total = _offsets(seqlens, par)
    inp = W.make_prefill_inputs(cfg, device="cuda", seqlens=seqlens, seed=7)
    k_out = torch.empty((total, cfg.H_kv, cfg.d_k), dtype=torch.bfloat16, device="cuda")
    v_out = torch.empty((total, cfg.H_kv, cfg.d_v), dtype=torch.bfloat16, device="cuda")
    args = (inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], tok, lens, cmp_off, heads, par,
            k_out, v_out)
    nsa.nsa_compress_noalloc(*args)
    torch.cuda.synchronize()
    nsa.nsa_noalloc_check_status()
    alloc0, free0 = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
    nsa.nsa_compress_noalloc(*args)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc0 and torch.cuda.mem_get_info()[0] == free0
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=side):
        nsa.nsa_compress_noalloc(*args, stream=side)
    torch.cuda.synchronize()
    new = W.make_prefill_inputs(cfg, device="cuda", seqlens=seqlens, seed=8)
    for name in ("k", "v", "w_ck", "pe_k", "w_cv", "pe_v"):
        inp[name].copy_(new[name])
    k_out.fill_(float("nan"))
    v_out.fill_(float("nan"))
    torch.cuda.synchronize()
    alloc1, free1 = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
    graph.replay()
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc1 and torch.cuda.mem_get_info()[0] == free1
    nsa.nsa_noalloc_check_status()
    ws = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_COMPRESS, heads, par, len(seqlens), 0, 0), "cuda")
    ref_k, ref_v = torch.empty_like(k_out), torch.empty_like(v_out)
    nsa.nsa_compress(new["k"], new["v"], new["w_ck"], new["pe_k"], new["w_cv"], new["pe_v"], tok, lens, cmp_off,
                     heads, par, ref_k, ref_v, ws)
    torch.cuda.synchronize()
    NP.assert_close(NP.f64(k_out), NP.f64(ref_k), "k_cmp (graph replay)", relative_to_rms=True)
    NP.assert_close(NP.f64(v_out), NP.f64(ref_v), "v_cmp (graph replay)", relative_to_rms=True)
    del graph


def test_noalloc_rejects_invalid_arguments():
    cfg = W.CONFIGS["prefill_8k"]
    par = NP.params_of(cfg)
    tok, lens, cmp_off, total = _offsets([100], par)
    x = torch.zeros((100, 4, 192), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((32 * 192, 192), dtype=torch.float32, device="cuda")
    pe = torch.zeros((32, 192), dtype=torch.float32, device="cuda")
    out = torch.zeros((max(total, 1), 4, 192), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nsa.NSAError) as ei:
        nsa.nsa_compress_noalloc(x, x, w, pe, w, pe, tok, lens, cmp_off, nsa.Heads(64, 4, 96, 96), par, out, out)
    assert ei.value.status == nsa.NSA_ERR_UNSUPPORTED
