"""GPU backward (nsa_prefill_backward) against the fp64 backward oracle.

Stage-wise, as for the forward: the oracle's attention steps take the GPU's
bf16 compressed keys/values and the GPU forward's selection (the selection is
held fixed in the backward); the compression's backward follows its fp64
definition from the raw tokens, W and pe. Every gradient is compared element
by element over the whole sequence (the key gradients depend on every query, so
no row sampling).

Tolerance (derivation): the GPU forms the probabilities P and the softmax
gradients dz in fp32 and rounds them to bf16 (unit roundoff u = 2^-8) as MMA
operands, with fp32 accumulation; each gradient element is a sum of many such
products, so its relative error has an RMS of about u/sqrt(3) ~ 2.3e-3 per
rounded operand, a few of which chain (P -> O -> <dout, O> -> dz -> dq). The
bound is relative RMS <= 1e-2 per gradient tensor and, element-wise, |err| <=
5e-2 * max|want| (the largest elements are sums of the same products).
dL/dpe_k is zero in exact arithmetic (pe_k shifts all compressed logits of a row
equally): the GPU value must be below 1e-3 of the dW_ck scale.
"""
import numpy as np
import pytest
import torch

import nsa_workloads as W
import sparse_attention_long_nsa_b200 as nsa
from oracle import nsa_backward as B
from tests import nsa_parity as NP

pytestmark = pytest.mark.gpu

CFG = W.CONFIGS
TOL_RRMS = 1e-2
TOL_MAX_REL = 5e-2


def _cmp(got, want, what, stats):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = np.abs(got - want)
    scale = float(np.abs(want).max()) if want.size else 0.0
    rms = float(np.sqrt(np.mean(want ** 2))) if want.size else 0.0
    rrms = float(np.sqrt(np.mean(err ** 2))) / rms if rms > 0 else 0.0
    mrel = float(err.max()) / scale if scale > 0 else float(err.max() if err.size else 0.0)
    stats[what] = (rrms, mrel)
    assert rrms <= TOL_RRMS, f"{what}: relative RMS {rrms:.3e} > {TOL_RRMS}"
    assert mrel <= TOL_MAX_REL, f"{what}: max error {mrel:.3e} of max|want| > {TOL_MAX_REL}"


def run_backward_case(cfg, seqlens, seed=0):
    heads, par, op = NP.heads_of(cfg), NP.params_of(cfg), NP.oracle_params(cfg)
    inp = W.make_prefill_inputs(cfg, device="cuda", seqlens=seqlens, seed=seed)
    kc, vc = nsa.compress(inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], seqlens, heads,
                          par)
    cu = inp["cu_seqlens"]
    out, sel = nsa.prefill(inp["q"], inp["k"], inp["v"], kc, vc, inp["gates"], cu, heads, par, want_sel=True)
    gen = torch.Generator(device="cuda").manual_seed(seed + 17)
    dout = torch.randn(out.shape, generator=gen, device="cuda").to(torch.bfloat16)
    N, mx = int(cu[-1]), max(seqlens)
    ws = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_BACKWARD, heads, par, len(seqlens), N, mx), "cuda")
    g = nsa.prefill_backward(inp["q"], inp["k"], inp["v"], kc, vc, inp["gates"], dout, sel, inp["w_ck"],
                             inp["pe_k"], inp["w_cv"], inp["pe_v"], cu, heads, par, ws=ws)
    torch.cuda.synchronize()
    nsa.nsa_check_device_status(ws)
    f = NP.f64
    selh = sel.cpu().numpy()
    stats = {}
    dw = {n: 0.0 for n in ("dw_ck", "dpe_k", "dw_cv", "dpe_v")}
    # the oracle's gradients of the packed batch (a one-token sequence has exactly
    # zero dq and dk, so tensors are compared over the whole batch, where such
    # rows are bounded by the batch's scale)
    want = {n: np.zeros(tuple(g[n].shape)) for n in ("dq", "dk", "dv", "dgates")}
    coff = 0
    for b, T in enumerate(seqlens):
        s0 = int(cu[b])
        nc = nsa.n_cmp(T, op["l_cmp"], op["stride"])
        if T == 0:
            continue
        sl = {(t, gg): [int(x) for x in selh[s0 + t, gg] if x >= 0] for t in range(T) for gg in range(cfg.H_kv)}
        r = B.backward(f(inp["q"][s0:s0 + T]), f(inp["k"][s0:s0 + T]), f(inp["v"][s0:s0 + T]), f(inp["w_ck"]),
                       f(inp["pe_k"]), f(inp["w_cv"]), f(inp["pe_v"]), f(inp["gates"][s0:s0 + T]),
                       f(dout[s0:s0 + T]), op, sel=sl, kc=f(kc[coff:coff + nc]), vc=f(vc[coff:coff + nc]))
        coff += nc
        NP.assert_close(f(out[s0:s0 + T]), r["out"], "forward output (same selection)")
        for name in want:
            want[name][s0:s0 + T] = r[name]
        for name in dw:
            dw[name] = dw[name] + r[name]
    for name in want:
        _cmp(f(g[name]), want[name], name, stats)
    for name in ("dw_ck", "dw_cv", "dpe_v"):
        _cmp(f(g[name]), dw[name], name, stats)
    assert float(np.abs(f(g["dpe_k"])).max()) <= 1e-3 * max(float(np.abs(dw["dw_ck"]).max()), 1e-30)
    return stats


def test_backward_tiny_gqa4():
    st = run_backward_case(CFG["prefill_tiny_1k"], [1024], seed=1)
    print({k: f"{v[0]:.2e}/{v[1]:.2e}" for k, v in st.items()})


def test_backward_gqa16_ragged():
    """The benched heads (64 query heads in 4 groups, d_k=192, d_v=128) on a ragged
    batch spanning several selection blocks past top-n, with a one-token sequence."""
    st = run_backward_case(CFG["prefill_8k"], [1500, 1, 700], seed=2)
    print({k: f"{v[0]:.2e}/{v[1]:.2e}" for k, v in st.items()})


@pytest.mark.parametrize("H_q,H_kv,d_k,d_v", [(8, 1, 128, 64), (4, 2, 64, 128), (4, 4, 192, 64)])
def test_backward_group_sizes(H_q, H_kv, d_k, d_v):
    cfg = W.small_config(T=1100, H_q=H_q, H_kv=H_kv, d_k=d_k, d_v=d_v, top_n=16, window=256, seed=21)
    run_backward_case(cfg, [1100, 257], seed=3)
