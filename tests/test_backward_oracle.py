"""Pins of the fp64 backward oracle (oracle/nsa_backward.py), no GPU.

* Directional finite differences: for a random direction u of every input
  (q, k, v, W_ck, pe_k, W_cv, pe_v, gates), (L(x + eps u) - L(x - eps u)) / 2 eps
  of L = <dout, out> from the FORWARD oracle (selection held fixed) equals
  <grad, u> from the backward oracle.
* Dense reductions: with top-n covering every block and gates (0, 1, 0), or a
  window >= T and gates (0, 0, 1), NSA is dense causal attention, so dq, dk, dv
  equal torch's fp64 autograd of scaled_dot_product_attention (a library
  routine), and the compression weights get no gradient.
* Planted mistakes (no softmax-backward correction, a dropped scale, W not
  transposed in the compression backward, a missing position-embedding term)
  each fail a pin.
"""
import numpy as np
import pytest
import torch

import nsa_workloads as W
from oracle import nsa_backward as B
from oracle import nsa_oracle as O


def _case(T=300, H_q=4, H_kv=2, d=16, top_n=4, window=100, seed=3):
    cfg = W.small_config(T=T, H_q=H_q, H_kv=H_kv, d_k=d, d_v=d, top_n=top_n, window=window, seed=seed)
    inp = W.make_prefill_inputs(cfg)
    f = lambda x: x.double().numpy()  # noqa: E731
    x = {n: f(inp[n]) for n in ("q", "k", "v", "w_ck", "pe_k", "w_cv", "pe_v", "gates")}
    rng = np.random.default_rng(seed)
    dout = rng.standard_normal((T, H_q, d))
    return cfg, x, dout


NAMES = ("q", "k", "v", "w_ck", "pe_k", "w_cv", "pe_v", "gates")
GRAD = dict(q="dq", k="dk", v="dv", w_ck="dw_ck", pe_k="dpe_k", w_cv="dw_cv", pe_v="dpe_v", gates="dgates")


def _fd_check(cfg, x, dout, backward=B.backward, eps=1e-6, n_dir=2, tol=1e-6):
    p = cfg.params()
    g = backward(*(x[n] for n in NAMES), dout, p)
    sel = g["sel"]
    rng = np.random.default_rng(11)
    worst = 0.0
    for name in NAMES:
        for _ in range(n_dir):
            u = rng.standard_normal(x[name].shape)
            xp = dict(x)
            xm = dict(x)
            xp[name] = x[name] + eps * u
            xm[name] = x[name] - eps * u
            lp = B.loss_forward(*(xp[n] for n in NAMES), dout, p, sel)
            lm = B.loss_forward(*(xm[n] for n in NAMES), dout, p, sel)
            fd = (lp - lm) / (2 * eps)
            an = float(np.sum(g[GRAD[name]] * u))
            # rounding noise of the two fp64 losses, divided by 2 eps
            noise = 1e-14 * max(1.0, abs(lp), abs(lm)) / eps
            rel = abs(fd - an) / max(abs(fd), abs(an), noise / tol)
            worst = max(worst, rel)
            assert rel <= tol, f"d/d{name}: finite difference {fd:.10e} vs backward {an:.10e} (rel {rel:.2e})"
    return worst


def test_backward_matches_finite_differences():
    cfg, x, dout = _case()
    _fd_check(cfg, x, dout)


def test_key_position_embedding_gets_no_gradient():
    """pe_k adds the same vector vec(pe_k).W_ck to every compressed key, which
    shifts every compressed logit of a row by the same amount; softmax ignores
    such a shift, so dL/dpe_k = 0 exactly (the value embedding pe_v does not
    cancel)."""
    cfg, x, dout = _case()
    g = B.backward(*(x[n] for n in NAMES), dout, cfg.params())
    scale_k = float(np.abs(g["dw_ck"]).max())
    assert float(np.abs(g["dpe_k"]).max()) <= 1e-12 * max(scale_k, 1.0)
    assert float(np.abs(g["dpe_v"]).max()) > 1e-3


def test_backward_finite_differences_gqa1_short():
    # a sequence shorter than the first compressed block for some rows, G = 1
    cfg, x, dout = _case(T=90, H_q=2, H_kv=2, d=8, top_n=3, window=40, seed=5)
    _fd_check(cfg, x, dout)


def _dense_grads(x, dout, G, scale):
    q = torch.tensor(x["q"], requires_grad=True)
    k = torch.tensor(x["k"], requires_grad=True)
    v = torch.tensor(x["v"], requires_grad=True)
    qq = q.permute(1, 0, 2)[None]
    kk = k.repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    vv = v.repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, is_causal=True, scale=scale)[0].permute(1, 0, 2)
    (o * torch.tensor(dout)).sum().backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("branch", ["slc", "win"])
def test_backward_dense_reduction(branch):
    T = 200
    cfg, x, dout = _case(T=T, H_q=4, H_kv=1, d=16, top_n=4, window=50, seed=7)
    e = np.zeros_like(x["gates"])
    e[..., 1 if branch == "slc" else 2] = 1.0
    x = dict(x, gates=e)
    p = dict(cfg.params(), **(dict(top_n=O.n_blk(T, 64)) if branch == "slc" else dict(window=T + 5)))
    g = B.backward(*(x[n] for n in NAMES), dout, p)
    dq, dk, dv = _dense_grads(x, dout, cfg.G, p["scale"])
    for name, want in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert np.allclose(g[name], want, rtol=1e-10, atol=1e-10), name
    for name in ("dw_ck", "dpe_k", "dw_cv", "dpe_v"):
        assert np.all(g[name] == 0.0), name


_ATTEND_BW = B.attend_backward
_COMPRESS_BW = B.compress_backward


def _mut_no_correction(qh, K, V, o, p, dO, scale):
    dq, dK, dV = _ATTEND_BW(qh, K, V, o, p, dO, scale)
    if K.shape[0] == 0:
        return dq, dK, dV
    dz = p * (dO @ np.asarray(V).T)          # mistake: no "- <dO, o>"
    return scale * (dz @ K), scale * (dz.T @ qh), dV


def _mut_no_scale(qh, K, V, o, p, dO, scale):
    dq, dK, dV = _ATTEND_BW(qh, K, V, o, p, dO, scale)
    return dq, dK / scale, dV                # mistake: scale dropped from dK


def _mut_dw_without_pe(x, Wm, pe, dc, l, s):
    dx, dW, dpe = _COMPRESS_BW(x, Wm, pe, dc, l, s)
    _, dW0, _ = _COMPRESS_BW(x, Wm, np.zeros_like(pe), dc, l, s)
    return dx, dW0, dpe                      # mistake: the block without pe in dW


def _mut_no_pe(x, Wm, pe, dc, l, s):
    dx, dW, dpe = _COMPRESS_BW(x, Wm, pe, dc, l, s)
    return dx, dW, np.zeros_like(dpe)        # mistake: pe treated as a constant


@pytest.mark.parametrize("target,mutant", [("attend_backward", _mut_no_correction),
                                           ("attend_backward", _mut_no_scale),
                                           ("compress_backward", _mut_dw_without_pe),
                                           ("compress_backward", _mut_no_pe)])
def test_backward_pins_catch_planted_mistakes(monkeypatch, target, mutant):
    cfg, x, dout = _case(T=160, H_q=4, H_kv=2, d=8, top_n=3, window=40, seed=9)
    monkeypatch.setattr(B, target, mutant)
    with pytest.raises(AssertionError):
        _fd_check(cfg, x, dout, n_dir=1)
