"""Paged KV caches on the GPU (nsa_decode_paged, nsa_compress_paged).

The raw and compressed caches are scattered over pools of pages in a random
order (unused pages hold NaN), and the same decode / compression through the
page tables must give bit-identical results to the contiguous layout. The
contiguous path is compared with the fp64 oracle by the parity tests; one
paged case is also compared with the oracle directly here.
"""
import numpy as np
import pytest
import torch

import nsa_workloads as W
import sparse_attention_long_nsa_b200 as nsa
from oracle import nsa_oracle as O
from tests import nsa_parity as NP

pytestmark = pytest.mark.gpu

CFG = W.CONFIGS


def to_pages(x, page, spare, gen):
    """x [B, L, H, d] (L a multiple of page) -> (pool [n_pages, page, H, d], table
    int32 [B, L / page]); the pages are placed in a random order among `spare`
    extra NaN pages."""
    B, L = int(x.shape[0]), int(x.shape[1])
    per = L // page
    n = B * per + spare
    perm = torch.randperm(n, generator=gen)
    pool = torch.full((n, page) + tuple(x.shape[2:]), float("nan"), dtype=x.dtype, device=x.device)
    table = perm[:B * per].reshape(B, per).to(torch.int32)
    pool[table.reshape(-1).long().to(x.device)] = x.reshape(B * per, page, *x.shape[2:])
    return pool, table.to(x.device)


def from_pages(pool, table):
    B, per = table.shape
    return pool[table.reshape(-1).long()].reshape(B, per * pool.shape[1], *pool.shape[2:])


@pytest.mark.parametrize("page,cpage", [(64, 32), (256, 128), (1024, 64)])
def test_paged_decode_identical_to_contiguous(page, cpage):
    cfg = CFG["decode_64k"]
    lens = [20000, 3001, 65536, 33, 1]
    inp = W.make_decode_inputs(cfg, device="cuda", lens=lens, seed=51)
    heads, par = NP.heads_of(cfg), NP.params_of(cfg)
    kc, vc = nsa.compress_cache(inp["k_cache"], inp["v_cache"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"],
                                inp["cache_lens"], heads, par)
    B, Lmax = len(lens), int(inp["k_cache"].shape[1])
    lens_d = inp["cache_lens"].to("cuda")
    ref_out, ref_sel, ref_imp = nsa.decode(inp["q"], inp["k_cache"], inp["v_cache"], kc, vc, lens_d, Lmax,
                                           inp["gates"], heads, par, want_sel=True, want_imp=True)
    g = torch.Generator().manual_seed(page)
    kp, bt = to_pages(inp["k_cache"], page, 5, g)
    vp, bt2 = to_pages(inp["v_cache"], page, 5, torch.Generator().manual_seed(page))
    assert torch.equal(bt, bt2)
    Lc = int(kc.shape[1])
    pad = -Lc % cpage
    kcp, cbt = to_pages(torch.nn.functional.pad(kc, (0, 0, 0, 0, 0, pad)), cpage, 3, torch.Generator().manual_seed(7))
    vcp, _ = to_pages(torch.nn.functional.pad(vc, (0, 0, 0, 0, 0, pad)), cpage, 3, torch.Generator().manual_seed(7))
    out = torch.empty_like(ref_out)
    sel = torch.empty_like(ref_sel)
    imp = torch.zeros_like(ref_imp)
    ws = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_DECODE, heads, par, B, 0, Lmax), "cuda")
    nsa.nsa_decode_paged(inp["q"], kp, vp, bt, kcp, vcp, cbt, lens_d, Lmax, inp["gates"], heads, par, out, sel, imp,
                         ws)
    torch.cuda.synchronize()
    nsa.nsa_check_device_status(ws)
    assert torch.equal(sel, ref_sel)
    assert torch.equal(out, ref_out)
    for b, L in enumerate(lens):   # importance rows of blocks 0 .. j_t
        assert torch.equal(imp[b, :, :(L - 1) // 64 + 1], ref_imp[b, :, :(L - 1) // 64 + 1])
    if page == 256:
        # one paged case against the oracle directly (selection and output)
        op = NP.oracle_params(cfg)
        kcc, vcc = from_pages(kcp, cbt), from_pages(vcp, cbt)
        orc = O.decode(inp["q"], inp["k_cache"], inp["v_cache"], kcc, vcc, lens, inp["gates"], op)
        gs = sel.cpu().numpy()
        for b in range(B):
            for gg in range(cfg.H_kv):
                assert [int(x) for x in gs[b, gg] if x >= 0] == orc["sel"][(b, gg)]
        NP.assert_close(NP.f64(out), orc["out"], "paged decode vs oracle")


def test_paged_decode_invalid_page_is_reported():
    """A page id outside the pool is recorded as a bounds error in the status word
    (and read as page 0): the call returns, the context stays usable."""
    cfg = CFG["decode_64k"]
    lens = [4000, 700]
    inp = W.make_decode_inputs(cfg, device="cuda", lens=lens, seed=52)
    heads, par = NP.heads_of(cfg), NP.params_of(cfg)
    kc, vc = nsa.compress_cache(inp["k_cache"], inp["v_cache"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"],
                                inp["cache_lens"], heads, par)
    Lmax = int(inp["k_cache"].shape[1])
    kp, bt = to_pages(torch.nn.functional.pad(inp["k_cache"], (0, 0, 0, 0, 0, 96)), 64, 0,
                      torch.Generator().manual_seed(1))
    vp, _ = to_pages(torch.nn.functional.pad(inp["v_cache"], (0, 0, 0, 0, 0, 96)), 64, 0,
                     torch.Generator().manual_seed(1))
    Lc = int(kc.shape[1])
    kcp, cbt = to_pages(torch.nn.functional.pad(kc, (0, 0, 0, 0, 0, -Lc % 32)), 32, 0, torch.Generator().manual_seed(2))
    vcp, _ = to_pages(torch.nn.functional.pad(vc, (0, 0, 0, 0, 0, -Lc % 32)), 32, 0, torch.Generator().manual_seed(2))
    bad = bt.clone()
    bad[0, (lens[0] - 1) // 64] = kp.shape[0] + 5   # the page holding sequence 0's newest token
    lens_d = inp["cache_lens"].to("cuda")
    out = torch.empty((2, cfg.H_q, cfg.d_v), dtype=torch.bfloat16, device="cuda")
    ws = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_DECODE, heads, par, 2, 0, Lmax + 96), "cuda")
    nsa.nsa_decode_paged(inp["q"], kp, vp, bad, kcp, vcp, cbt, lens_d, Lmax, inp["gates"], heads, par, out, None,
                         None, ws)
    with pytest.raises(nsa.NSAError) as ei:
        nsa.nsa_check_device_status(ws)
    assert ei.value.status == nsa.NSA_ERR_DEVICE_CHECK and "status 0x2" in str(ei.value)
    nsa.nsa_decode_paged(inp["q"], kp, vp, bt, kcp, vcp, cbt, lens_d, Lmax, inp["gates"], heads, par, out, None,
                         None, ws)
    torch.cuda.synchronize()
    nsa.nsa_check_device_status(ws)
    ref = nsa.decode(inp["q"], inp["k_cache"], inp["v_cache"], kc, vc, lens_d, Lmax, inp["gates"], heads, par)
    assert torch.equal(out, ref)


@pytest.mark.parametrize("page,cpage", [(64, 32), (512, 256)])
def test_paged_compress_identical_to_contiguous(page, cpage):
    """Whole compressed caches built from a paged raw cache, then the same caches
    grown by uneven chunks: every summary equals the contiguous compression's."""
    cfg = CFG["decode_64k"]
    lens = [9000, 100, 4097, 31]
    inp = W.make_decode_inputs(cfg, device="cuda", lens=lens, seed=53, Lmax=16384)
    heads, par = NP.heads_of(cfg), NP.params_of(cfg)
    B, Lmax = len(lens), 16384
    kc, vc = nsa.compress_cache(inp["k_cache"], inp["v_cache"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"],
                                inp["cache_lens"], heads, par)
    kp, bt = to_pages(inp["k_cache"], page, 4, torch.Generator().manual_seed(3))
    vp, _ = to_pages(inp["v_cache"], page, 4, torch.Generator().manual_seed(3))
    Lc = nsa.n_cmp(Lmax)
    ncp = -(-Lc // cpage)
    cperm = torch.randperm(B * ncp + 2, generator=torch.Generator().manual_seed(4))
    cbt = cperm[:B * ncp].reshape(B, ncp).to(torch.int32).cuda()
    kcp = torch.full((B * ncp + 2, cpage, cfg.H_kv, cfg.d_k), float("nan"), dtype=torch.bfloat16, device="cuda")
    vcp = torch.full((B * ncp + 2, cpage, cfg.H_kv, cfg.d_v), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_COMPRESS, heads, par, B, 0, 0), "cuda")
    # grow from empty in uneven steps: first to half of each length, then the rest
    half = torch.tensor([L // 2 for L in lens], dtype=torch.int32)
    full = torch.tensor(lens, dtype=torch.int32)
    n1 = nsa.nsa_compress_paged(kp, vp, bt, inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"],
                                torch.zeros(B, dtype=torch.int32), half, heads, par, kcp, vcp, cbt, ws)
    n2 = nsa.nsa_compress_paged(kp, vp, bt, inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], half, full, heads,
                                par, kcp, vcp, cbt, ws)
    torch.cuda.synchronize()
    nsa.nsa_check_device_status(ws)
    assert n1 + n2 == sum(nsa.n_cmp(L) for L in lens)
    kcc, vcc = from_pages(kcp, cbt), from_pages(vcp, cbt)
    for b, L in enumerate(lens):
        nc = nsa.n_cmp(L)
        assert torch.equal(kcc[b, :nc], kc[b, :nc]), b
        assert torch.equal(vcc[b, :nc], vc[b, :nc]), b
