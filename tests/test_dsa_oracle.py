"""Pins of the DSA oracle (oracle/dsa_oracle.py), no GPU.

* The page's count: 2048 kept tokens of a 131,072-token context, about 1.6 %.
* top_k >= t + 1 keeps every token, so DSA is dense causal attention: equal to
  torch's fp64 scaled_dot_product_attention (a library routine).
* An independent dense formulation (oracle/brute.py: score matrix by einsum,
  rank by lexicographic sort, keep mask, masked softmax) agrees on tiny inputs.
* Selection against exhaustive enumeration with integer (tied) scores: the kept
  set is the unique one whose every kept score beats every dropped one, ties to
  the lower index.
* ReLU: indexer heads with negative dot products contribute nothing; negative
  weights lower the score.
* Planted mistakes (no ReLU, weights ignored, ties to the higher index) each fail
  a pin.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

import nsa_workloads as W
from oracle import brute
from oracle import dsa_oracle as D

GOLD = os.path.join(os.path.dirname(__file__), "golden", "dsa_keys_fraction.json")


def _inp(T=96, H_q=4, H_kv=2, d=16, H_I=3, d_I=8, seed=4):
    cfg = W.DSAConfig("t", "prefill", 1, T, H_q, H_kv, d, d, H_I=H_I, d_I=d_I, top_k=20, seed=seed)
    x = W.make_dsa_prefill_inputs(cfg)
    return cfg, {n: x[n].double().numpy() for n in ("q", "k", "v", "qi", "wi", "ki")}


def test_page_key_fraction():
    g = json.load(open(GOLD))
    T, k = g["context"], g["top_k"]
    rng = np.random.default_rng(0)
    scores = rng.standard_normal(T)
    sel = D.select_tokens(scores, T - 1, k)
    assert len(sel) == g["kept"]
    assert round(100.0 * len(sel) / T, 1) == g["percent_rounded"]


def test_dense_when_top_k_covers_the_prefix():
    cfg, x = _inp(T=80)
    out = D.prefill(x["q"], x["k"], x["v"], x["qi"], x["wi"], x["ki"], 80, cfg.scale)["out"]
    q = torch.tensor(x["q"]).permute(1, 0, 2)[None]
    k = torch.tensor(x["k"]).repeat_interleave(cfg.G, 1).permute(1, 0, 2)[None]
    v = torch.tensor(x["v"]).repeat_interleave(cfg.G, 1).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=cfg.scale)[0]
    assert np.allclose(out, ref.permute(1, 0, 2).numpy(), atol=1e-12, rtol=1e-12)


@pytest.mark.parametrize("top_k", [1, 7, 20, 50])
def test_structured_matches_dense_formulation(top_k):
    cfg, x = _inp(T=96)
    r = D.prefill(x["q"], x["k"], x["v"], x["qi"], x["wi"], x["ki"], top_k, cfg.scale)
    out_b, keep = brute.dsa_brute(x["q"], x["k"], x["v"], x["qi"], x["wi"], x["ki"], top_k, cfg.scale)
    for t in range(96):
        assert r["sel"][t] == sorted(np.nonzero(keep[t])[0].tolist()), t
    assert np.allclose(r["out"], out_b, atol=1e-12, rtol=1e-12)


def test_selection_exhaustive_with_ties():
    rng = np.random.default_rng(3)
    for _ in range(300):
        n, k = int(rng.integers(2, 9)), int(rng.integers(1, 6))
        scores = rng.integers(0, 3, size=n).astype(float)   # many exact ties
        t = n - 1
        want = None
        if t + 1 <= k:
            want = list(range(n))
        else:
            for c in itertools.combinations(range(n), k):
                cs = set(c)
                if all(scores[a] > scores[b] or (scores[a] == scores[b] and a < b)
                       for a in cs for b in range(n) if b not in cs):
                    assert want is None   # unique
                    want = list(c)
        assert D.select_tokens(scores, t, k) == want


def test_relu_and_weight_signs():
    qi = np.array([[1.0, 0.0], [0.0, 1.0]])
    ki = np.array([[2.0, -3.0], [-1.0, -1.0], [0.5, 4.0]])
    w = np.array([1.0, 1.0])
    assert np.allclose(D.index_scores(qi, w, ki), [2.0, 0.0, 4.5])       # negative dots clipped
    assert np.allclose(D.index_scores(qi, np.array([1.0, -2.0]), ki), [2.0, 0.0, 0.5 - 8.0])


def _mut_no_relu(qi_t, wi_t, ki):
    return (np.asarray(ki, float) @ np.asarray(qi_t, float).T) @ np.asarray(wi_t, float)


def _mut_no_weights(qi_t, wi_t, ki):
    return np.maximum(np.asarray(ki, float) @ np.asarray(qi_t, float).T, 0.0).sum(axis=1)


def _mut_ties_high(scores, t, top_k):
    if t + 1 <= top_k:
        return list(range(t + 1))
    order = sorted(range(t + 1), key=lambda s: (-float(scores[s]), -s))
    return sorted(order[:top_k])


@pytest.mark.parametrize("target,mutant", [("index_scores", _mut_no_relu), ("index_scores", _mut_no_weights),
                                           ("select_tokens", _mut_ties_high)])
def test_pins_catch_planted_mistakes(monkeypatch, target, mutant):
    monkeypatch.setattr(D, target, mutant)
    with pytest.raises(AssertionError):
        if target == "select_tokens":
            test_selection_exhaustive_with_ties()
        else:
            test_structured_matches_dense_formulation(20)
            test_relu_and_weight_signs()
