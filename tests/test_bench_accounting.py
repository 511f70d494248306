"""The work bench.py divides by: per-branch (query, key) pair counts of a prefill
and unique K/V bytes of a decode step, checked against the oracle's own key sets
built row by row (no GPU)."""
import numpy as np
import pytest
import torch

import bench
import nsa_workloads as W
from oracle import nsa_oracle as O


@pytest.mark.parametrize("T,kw", [
    (1, {}), (31, {}), (32, {}), (100, {}), (1500, {}),
    (700, dict(top_n=4, window=128)), (900, dict(l_sel=32, top_n=8, window=64)),
])
def test_prefill_pairs_match_oracle_key_sets(T, kw):
    cfg = W.small_config(T=T, **kw)
    p = cfg.params()
    rng = np.random.default_rng(T)
    pc = ps = pw = 0
    for t in range(T):
        pc += O.cmp_visible(t, p["l_cmp"], p["stride"])
        imp = rng.random(t // p["l_sel"] + 1)   # the count does not depend on which blocks win
        sel = O.select(imp, t, p["l_sel"], p["top_n"], p["force_first"], p["force_local"])
        ps += len(O.selected_keys(sel, t, p["l_sel"]))
        pw += len(O.window_keys(t, p["window"]))
    assert bench.prefill_pairs(T, cfg) == (pc, ps, pw)


def test_prefill_work_totals():
    """FLOPs: 2 (d_k + d_v) per pair and query head, plus the compression GEMM."""
    cfg = W.CONFIGS["prefill_8k"]
    pc, ps, pw = bench.prefill_pairs(cfg.T, cfg)
    assert (pc, ps, pw) == (2085391, 7639040, 4063488)
    w = bench.prefill_work(cfg)
    assert w["prefill_attn"] == (pc + ps + pw) * 2 * (cfg.d_k + cfg.d_v) * cfg.H_q
    nc = O.n_cmp(cfg.T, cfg.l_cmp, cfg.stride)
    assert w["compress_gemm"] == 2 * cfg.l_cmp * (cfg.d_k ** 2 + cfg.d_v ** 2) * nc * cfg.H_kv
    assert w["dense_causal"] == cfg.T * (cfg.T + 1) // 2 * 2 * (cfg.d_k + cfg.d_v) * cfg.H_q


def test_decode_bytes_count_unique_keys():
    cfg = W.small_config(T=5000, H_q=8, H_kv=2, d_k=64, d_v=128)
    p = cfg.params()
    lens = [5000, 1, 700, 64]
    rng = np.random.default_rng(3)
    sel = np.full((len(lens), cfg.H_kv, p["top_n"]), -1, dtype=np.int32)
    want_fine = 0
    for b, L in enumerate(lens):
        t = L - 1
        for g in range(cfg.H_kv):
            s = O.select(rng.random(t // p["l_sel"] + 1), t, p["l_sel"], p["top_n"], p["force_first"],
                         p["force_local"])
            sel[b, g, :len(s)] = s
            keys = set(O.selected_keys(s, t, p["l_sel"]).tolist()) | set(O.window_keys(t, p["window"]).tolist())
            want_fine += len(keys) * (cfg.d_k + cfg.d_v) * 2
    want_cmp = sum(O.n_cmp(L, p["l_cmp"], p["stride"]) for L in lens) * cfg.H_kv * (cfg.d_k + cfg.d_v) * 2
    assert bench.decode_bytes(cfg, lens, torch.from_numpy(sel)) == (want_cmp, want_fine)
