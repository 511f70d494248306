"""Pins for the CPU oracle: every check compares it with something other than
itself (values the pages print, closed forms, library routines, brute force on
tiny inputs, invariants). CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import brute
from oracle import nsa_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _params(l=32, s=16, ls=64, n=4, w=128, ff=1, fl=2, d_k=64):
    return dict(l_cmp=l, stride=s, l_sel=ls, top_n=n, window=w, force_first=ff,
                force_local=fl, scale=1.0 / math.sqrt(d_k))


def _rand(T, H_q, H_kv, d_k, d_v, seed, n_c=None, l=32, s=16):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(T, H_q, d_k))
    k = rng.normal(size=(T, H_kv, d_k))
    v = rng.normal(size=(T, H_kv, d_v))
    nc = O.n_cmp(T, l, s) if n_c is None else n_c
    kc = rng.normal(size=(nc, H_kv, d_k))
    vc = rng.normal(size=(nc, H_kv, d_v))
    gates = 1.0 / (1.0 + np.exp(-rng.normal(size=(T, H_q, 3))))
    return q, k, v, kc, vc, gates


# --------------------------------------------------------------------------
# P7: the page's printed window mask (T=4, w=2)
# --------------------------------------------------------------------------

def test_window_mask_matches_page_example():
    g = _gold("window_mask_T4_w2.json")
    T, w = g["T"], g["w"]
    want = np.array(g["mask"], dtype=bool)
    got = np.zeros((T, T), dtype=bool)
    for t in range(T):
        got[t, O.window_keys(t, w)] = True
    assert (got == want).all()
    assert (brute.window_mask(T, w) == want).all()


# --------------------------------------------------------------------------
# P8: the FlexAttention demo's printed pair fraction (window 256 + 4 sink tokens)
# --------------------------------------------------------------------------

def test_window_plus_sink_pair_fraction_matches_page():
    g = _gold("flex_window_sink.json")
    T, w, sink = g["T"], g["window"], g["sink"]
    kept = 0
    for t in range(T):
        keys = set(O.window_keys(t, w).tolist()) | set(range(min(sink, t + 1)))
        kept += len(keys)
    causal = T * (T + 1) // 2
    assert round(kept / causal, 3) == g["pair_fraction_3dp"]


# --------------------------------------------------------------------------
# P2: closed-form key counts and the pages' key-count tables
# --------------------------------------------------------------------------

def _count(t, l, s, ls, n, w, sel=None):
    nvis = O.cmp_visible(t, l, s)
    jt = t // ls
    if sel is None:
        # any admissible selection: forced {0, jt-1, jt} plus the lowest free
        sel = O.select(np.zeros(jt + 1), t, ls, n, 1, 2)
    return nvis, len(O.selected_keys(sel, t, ls)), len(O.window_keys(t, w))


def test_counts_closed_form_grid():
    l, s, ls, n, w = 32, 16, 64, 16, 512
    for t in list(range(0, 300)) + [1023, 1024, 4095, 8191, 65535]:
        nvis, nsel, nwin = _count(t, l, s, ls, n, w)
        assert nvis == (0 if t < l - 1 else (t - l + 1) // s + 1)
        jt = t // ls
        want_sel = t + 1 if jt + 1 <= n else (n - 1) * ls + (t % ls) + 1
        assert nsel == want_sel
        assert nwin == min(w, t + 1)


def test_key_count_table_of_page():
    g = _gold("keys_per_query.json")
    for row in g["table"]:
        T = row["context"]
        nvis, nsel, nwin = _count(T - 1, 32, 16, 64, 16, 512)
        total = nvis + nsel + nwin
        # The page rounds the compressed count to T/16; the exact count at the
        # last position is one lower (the block ending at T is not yet whole).
        assert abs(total - row["nsa_approx"]) <= 1
        assert round(row["full"] / total, 1) == row["ratio"]


def test_compute_budget_of_lesson():
    g = _gold("keys_per_query.json")
    for row in g["budget"]:
        N, l, k, b, w = row["N"], row["l"], row["k"], row["b"], row["w"]
        nvis, nsel, nwin = _count(N - 1, l, l, b, k, w)
        assert (nvis, nsel, nwin) == (row["cmp"], row["sel"], row["win"])
        assert nvis + nsel + nwin == row["total"]
        if "ratio_int" in row:
            assert int(row["full"] / row["total"]) == row["ratio_int"]
    sm = g["small"]
    nvis, nsel, nwin = _count(sm["N"] - 1, sm["l"], sm["l"], sm["l"], sm["k"], sm["w"])
    assert (nvis, nsel, nwin) == (sm["cmp"], sm["sel"], sm["win"])
    assert math.floor(10 * sm["N"] / (nvis + nsel + nwin)) / 10 == sm["ratio_1dp_floor"]


# --------------------------------------------------------------------------
# P5: mean-pool special case of the compressor; brute-force compression
# --------------------------------------------------------------------------

def test_compress_mean_pool_special_case():
    rng = np.random.default_rng(3)
    T, H, d, l = 200, 2, 8, 16
    x = rng.normal(size=(T, H, d))
    W = np.concatenate([np.eye(d)] * l, axis=0) / l
    got = O.compress(x, W, np.zeros((l, d)), l, l)
    nfull = T // l
    want = x[:nfull * l].reshape(nfull, l, H, d).mean(axis=1)
    assert got.shape == want.shape
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-13)


@pytest.mark.parametrize("l,s", [(32, 16), (8, 4), (8, 8), (12, 4)])
def test_compress_vs_explicit_sum(l, s):
    rng = np.random.default_rng(l * 100 + s)
    T, H, d, do = 70, 2, 6, 5
    x = rng.normal(size=(T, H, d))
    W = rng.normal(size=(l * d, do))
    pe = rng.normal(size=(l, d))
    np.testing.assert_allclose(O.compress(x, W, pe, l, s), brute.compress_brute(x, W, pe, l, s),
                               rtol=1e-12, atol=1e-12)


def test_compress_position_embedding_is_a_bias():
    rng = np.random.default_rng(5)
    T, H, d, l, s = 64, 1, 4, 8, 4
    x = rng.normal(size=(T, H, d))
    W = rng.normal(size=(l * d, 3))
    pe = rng.normal(size=(l, d))
    a = O.compress(x, W, pe, l, s)
    b = O.compress(x, W, np.zeros_like(pe), l, s) + (pe.reshape(-1) @ W)[None, None, :]
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# omega: scalar definition vs grid, and the l=32/s=16/l'=64 weight pattern
# --------------------------------------------------------------------------

def test_omega_pattern_for_default_blocks():
    # compressed token 4j-1 straddles blocks j-1 and j (16 tokens each); 4j..4j+2
    # lie inside block j (32 tokens); 4j+3 straddles j and j+1
    for j in range(1, 6):
        assert O.omega(4 * j - 1, j, 32, 16, 64) == 1.0
        assert O.omega(4 * j - 1, j - 1, 32, 16, 64) == 1.0
        for i in (4 * j, 4 * j + 1, 4 * j + 2):
            assert O.omega(i, j, 32, 16, 64) == 2.0
        assert O.omega(4 * j + 3, j, 32, 16, 64) == 1.0
        assert O.omega(4 * j + 3, j + 1, 32, 16, 64) == 1.0
        assert O.omega(4 * j + 4, j - 1, 32, 16, 64) == 0.0
    M = O.omega_matrix(40, 12, 32, 16, 64)
    for i in range(40):
        for j in range(12):
            assert M[i, j] == O.omega(i, j, 32, 16, 64)


# --------------------------------------------------------------------------
# selection vs exhaustive enumeration (ties included)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(6))
def test_select_vs_enumeration(seed):
    rng = np.random.default_rng(seed)
    for _ in range(60):
        ls = 8
        t = int(rng.integers(0, 80))
        jt = t // ls
        n = int(rng.integers(3, 7))
        # integer scores produce many exact ties
        imp = rng.integers(0, 4, size=jt + 1).astype(float)
        a = O.select(imp, t, ls, n, 1, 2)
        b = brute.select_brute(imp, t, ls, n, 1, 2)
        assert a == b
        assert len(a) == min(n, jt + 1)
        assert a == sorted(a)
        if jt + 1 > n:
            assert {0, jt - 1, jt} <= set(a)


def test_select_ties_go_to_lower_index():
    imp = np.ones(10)
    assert O.select(imp, 9 * 64, 64, 5, 1, 2) == [0, 1, 2, 8, 9]


# --------------------------------------------------------------------------
# P1: structured oracle vs mask-based brute force on tiny inputs
# --------------------------------------------------------------------------

GRID = [
    # l, s, ls, n, w, G, H_kv, T
    (32, 16, 64, 4, 128, 4, 1, 512),
    (8, 4, 16, 4, 20, 2, 2, 100),
    (8, 8, 8, 3, 5, 1, 2, 61),
    (16, 8, 32, 5, 40, 4, 1, 200),
    (4, 2, 8, 3, 7, 2, 1, 50),
    (8, 4, 16, 16, 500, 2, 1, 90),   # n covers all blocks and w >= T
]


@pytest.mark.parametrize("l,s,ls,n,w,G,H_kv,T", GRID)
def test_structured_vs_brute(l, s, ls, n, w, G, H_kv, T):
    d_k, d_v = 8, 6
    p = _params(l, s, ls, n, w, 1, 2, d_k)
    q, k, v, kc, vc, gates = _rand(T, G * H_kv, H_kv, d_k, d_v, seed=T + n, l=l, s=s)
    r = O.prefill(q, k, v, kc, vc, gates, p)
    out_b, sel_b, imp_b = brute.nsa_prefill_brute(q, k, v, kc, vc, gates, p)
    np.testing.assert_allclose(r["out"], out_b, rtol=1e-12, atol=1e-12)
    for key in sel_b:
        assert r["sel"][key] == sel_b[key]
        np.testing.assert_allclose(r["imp"][key], imp_b[key], rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# P3: importance mass invariant, forced blocks, nonnegativity
# --------------------------------------------------------------------------

def test_importance_mass_invariant():
    l, s, ls = 32, 16, 64
    G, H_kv, T = 4, 2, 400
    p = _params(l, s, ls, 4, 128, 1, 2, 16)
    q, k, v, kc, vc, gates = _rand(T, G * H_kv, H_kv, 16, 8, seed=11)
    r = O.prefill(q, k, v, kc, vc, gates, p, rows=range(0, T, 7))
    for (t, g), imp in r["imp"].items():
        assert (imp >= 0).all()
        want = G * l / s if t >= l - 1 else 0.0
        assert abs(imp.sum() - want) < 1e-10
        jt = t // ls
        if jt + 1 > 4:
            assert {0, jt - 1, jt} <= set(r["sel"][(t, g)])


# --------------------------------------------------------------------------
# P4: dense reductions against the library's scaled_dot_product_attention
# --------------------------------------------------------------------------

def _sdpa_causal(q, k, v, G):
    # q [T, H_q, d], k/v [T, H_kv, *] -> [T, H_q, dv] in float64
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(np.repeat(k, G, axis=1)).permute(1, 0, 2)[None]
    vt = torch.from_numpy(np.repeat(v, G, axis=1)).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    return o[0].permute(1, 0, 2).numpy()


@pytest.mark.parametrize("branch", ["slc", "win"])
def test_dense_reduction(branch):
    T, G, H_kv, d_k, d_v = 300, 4, 2, 16, 12
    q, k, v, kc, vc, gates = _rand(T, G * H_kv, H_kv, d_k, d_v, seed=21)
    if branch == "slc":
        p = _params(32, 16, 64, 64, 16, 1, 2, d_k)      # n >= n_blk
        gates = np.zeros_like(gates)
        gates[..., 1] = 1.0
    else:
        p = _params(32, 16, 64, 4, T + 5, 1, 2, d_k)    # w >= T
        gates = np.zeros_like(gates)
        gates[..., 2] = 1.0
    r = O.prefill(q, k, v, kc, vc, gates, p)
    np.testing.assert_allclose(r["out"], _sdpa_causal(q, k, v, G), rtol=1e-10, atol=1e-12)


# --------------------------------------------------------------------------
# P6: the output is linear in the gates
# --------------------------------------------------------------------------

def test_gate_linearity():
    T, G, H_kv = 150, 2, 2
    p = _params(16, 8, 32, 3, 20, 1, 2, 8)
    q, k, v, kc, vc, gates = _rand(T, G * H_kv, H_kv, 8, 8, seed=31, l=16, s=8)
    rows = [0, 14, 15, 16, 63, 64, 100, 149]
    full = O.prefill(q, k, v, kc, vc, gates, p, rows=rows)["out"]
    acc = np.zeros_like(full)
    for b in range(3):
        e = np.zeros_like(gates)
        e[..., b] = 1.0
        ob = O.prefill(q, k, v, kc, vc, e, p, rows=rows)["out"]
        acc += gates[rows][:, :, b:b + 1] * ob
    np.testing.assert_allclose(full, acc, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# decode = last row of prefill on the same sequence (cache holds the new token)
# --------------------------------------------------------------------------

def test_decode_matches_prefill_last_row():
    rng = np.random.default_rng(41)
    H_q, H_kv, d_k, d_v = 4, 2, 8, 8
    l, s = 16, 8
    lens = [70, 33, 15, 128]
    Lmax = max(lens)
    p = _params(l, s, 32, 3, 24, 1, 2, d_k)
    w_ck = rng.normal(size=(l * d_k, d_k)) / 10
    w_cv = rng.normal(size=(l * d_v, d_v)) / 10
    pe_k, pe_v = rng.normal(size=(l, d_k)), rng.normal(size=(l, d_v))
    B = len(lens)
    q = rng.normal(size=(B, H_q, d_k))
    kcache = rng.normal(size=(B, Lmax, H_kv, d_k))
    vcache = rng.normal(size=(B, Lmax, H_kv, d_v))
    gates = rng.uniform(size=(B, H_q, 3))
    ncm = O.n_cmp(Lmax, l, s)
    kcc = np.zeros((B, ncm, H_kv, d_k))
    vcc = np.zeros((B, ncm, H_kv, d_v))
    for b, L in enumerate(lens):
        n = O.n_cmp(L, l, s)
        kcc[b, :n] = O.compress(kcache[b, :L], w_ck, pe_k, l, s)
        vcc[b, :n] = O.compress(vcache[b, :L], w_cv, pe_v, l, s)
    dec = O.decode(q, kcache, vcache, kcc, vcc, lens, gates, p)
    for b, L in enumerate(lens):
        qq = np.zeros((L, H_q, d_k))
        qq[L - 1] = q[b]
        gg = np.zeros((L, H_q, 3))
        gg[L - 1] = gates[b]
        r = O.prefill_full(qq, kcache[b, :L], vcache[b, :L], w_ck, pe_k, w_cv, pe_v, gg, p,
                           rows=[L - 1])
        np.testing.assert_allclose(dec["out"][b], r["out"][0], rtol=1e-12, atol=1e-13)
        for g in range(H_kv):
            assert dec["sel"][(b, g)] == r["sel"][(L - 1, g)]


# --------------------------------------------------------------------------
# P8: the needle-in-a-haystack demo's printed table, recomputed through the
# oracle's own attention, mean-pool compression, importance and selection
# --------------------------------------------------------------------------

def test_needle_demo_reproduces_printed_table():
    g = _gold("needle_demo.json")
    rng = np.random.default_rng(0)
    T, d = 8192, 64
    q = rng.normal(size=d)
    K = rng.normal(size=(T, d))
    V = rng.normal(size=(T, d))
    needle = np.arange(3000, 3016)
    K[needle] = 8 * np.sqrt(d) * q / (q @ q) + 0.1 * rng.normal(size=(16, d))
    V[needle] = 3.0
    scale = 1.0 / np.sqrt(d)

    def run(idx):
        o, pw = O.attend(q[None], K[idx], V[idx], scale)
        return o[0], pw[0][np.isin(idx, needle)].sum()

    full, w_full = run(np.arange(T))
    assert round(w_full, 2) == g["needle_weight_full"]

    def cos(o):
        return float(o @ full / np.linalg.norm(o) / np.linalg.norm(full))

    rows = {r["method"]: r for r in g["rows"]}
    win = O.window_keys(T - 1, 512)
    r = rows["window 512"]
    assert len(win) == r["keys"] and round(100 * len(win) / T, 1) == r["frac_pct"]
    assert round(cos(run(win)[0]), 3) == r["cos"]

    rnd = np.sort(rng.choice(T, 256, replace=False))
    r = rows["random 256 keys"]
    assert round(abs(cos(run(rnd)[0])), 3) == abs(r["cos"])

    # mean-pooled blocks of 64 (compress with an averaging map, stride = block)
    B = 64
    Wmean = np.concatenate([np.eye(d)] * B, axis=0) / B
    blocks = O.compress(K[:, None, :], Wmean, np.zeros((B, d)), B, B)[:, 0]
    # ranking blocks by softmax weight = ranking by score; with l = s = l' the
    # overlap weight is 1 on the block itself
    _, pc = O.attend(q[None], blocks, blocks, 1.0)
    imp = O.importance(pc, T - 1, B, B, B)
    sel = O.select(imp, T - 1, B, 16, 0, 0)
    idx = np.union1d(O.selected_keys(sel, T - 1, B), win)
    r = rows["top-16 blocks + window"]
    assert len(idx) == r["keys"] and round(100 * len(idx) / T, 1) == r["frac_pct"]
    assert round(cos(run(idx)[0]), 3) == r["cos"]
