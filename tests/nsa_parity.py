"""Shared parity machinery: run the CUDA path through the C ABI, run the CPU
oracle on the same seeded inputs, compare element by element.

Acceptance (NSA forward, fp64 oracle vs bf16/fp32 GPU path):
  outputs        max-abs <= 2e-2 and relative RMS <= 5e-3
  compressed K/V each element within u*|x| + 1.5e-2*RMS (u = 2^-8, bf16) and
                 relative RMS <= 5e-3 (vs the oracle's own fp64 compression from
                 the fp32 weights; see assert_close)
  importance     |gpu - oracle| <= 1e-4 * (largest oracle block score of the row)
  selection      identical index sets; a difference is accepted only at a near
                 tie (relative gap <= 1e-5 in the oracle's scores) and only if
                 the oracle, fed the GPU's scores, picks the GPU's set; the
                 output rows are then compared against the oracle rerun with it.
Stage-wise: the oracle's steps 2-7 consume the GPU's bf16 compressed K/V, so a
selection is never flipped by the compression rounding alone.
End to end (e2e_rows): the oracle also runs on its own fp64 compression of the
fp32 weights. The GPU rounds the compressed keys to bf16 (relative 2^-9), which
moves a logit by about 2^-9 and a block score by about 1e-3 relative, so there
a selection may differ only where the oracle's own scores of the swapped blocks
are within E2E_TIE (1e-2) of each other, the GPU's set must follow from its own
scores, and the output rows are compared with the oracle rerun on that set.
The outputs then also carry the compressed branch's inherited error: the bf16
compressed keys and values differ from the fp64 ones by a relative RMS of about
0.8u*sqrt(2) = 4.4e-3 (u = 2^-8: bf16 block tokens and weights in the l*d-term
sums, and the rounding of the summaries), so the end-to-end bound is max-abs
2e-2 and relative RMS E2E_RRMS = 1e-2 (the stage-wise 5e-3 plus that term).
"""
from __future__ import annotations

import numpy as np
import torch

import nsa_workloads as W
import sparse_attention_long_nsa_b200 as nsa
from oracle import nsa_oracle as O

TOL_MAX = 2e-2
TOL_RRMS = 5e-3
TOL_IMP = 1e-4
NEAR_TIE = 1e-5
E2E_TIE = 1e-2
E2E_RRMS = 1e-2


def heads_of(cfg):
    return nsa.Heads(cfg.H_q, cfg.H_kv, cfg.d_k, cfg.d_v)


def params_of(cfg, **over):
    p = dict(l_cmp=cfg.l_cmp, stride=cfg.stride, l_sel=cfg.l_sel, top_n=cfg.top_n, window=cfg.window,
             force_first=cfg.force_first, force_local=cfg.force_local)
    p.update(over)
    return nsa.make_params(**p)


def oracle_params(cfg, **over):
    p = cfg.params()
    p.update(over)
    return p


def f64(t):
    return t.detach().to("cpu").double().numpy()


BF16_U = 2.0 ** -8      # unit roundoff of bf16 (8 significant bits)
TOL_CMP_ABS = 1.5e-2    # compressed K/V: multiple of RMS covering the input roundings


def assert_close(got, want, what, tol_max=TOL_MAX, tol_rrms=TOL_RRMS, relative_to_rms=False):
    """Outputs: max-abs <= tol_max, relative RMS <= tol_rrms.

    relative_to_rms (compressed K/V, values of order 1 with tails to ~5 RMS):
    each element within BF16_U*|want| (the final bf16 rounding) plus
    TOL_CMP_ABS*RMS. The second term covers the rounding of the block tokens
    and of W to bf16: per product a relative error of variance 2u^2/3, i.e. an
    error of standard deviation ~0.8u*RMS on the sum, times a 5-6 sigma tail over
    millions of elements."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = np.abs(got - want)
    rms = float(np.sqrt(np.mean(want ** 2))) if want.size else 0.0
    max_err = float(err.max()) if err.size else 0.0
    rrms = float(np.sqrt(np.mean(err ** 2))) / rms if rms > 0 else float(np.sqrt(np.mean(err ** 2)))
    if relative_to_rms:
        excess = err - (BF16_U * np.abs(want) + TOL_CMP_ABS * rms)
        worst = float(excess.max()) if excess.size else -1.0
        assert worst <= 0, f"{what}: element error above u|x| + {TOL_CMP_ABS}*RMS by {worst:.3e} (max-abs {max_err:.3e})"
    else:
        assert max_err <= tol_max, f"{what}: max-abs {max_err:.3e} > {tol_max:.3e}"
    assert rrms <= tol_rrms, f"{what}: relative RMS {rrms:.3e} > {tol_rrms:.3e}"
    return max_err, rrms


def sample_rows(T, n_random, rng):
    edges = [0, 1, 15, 30, 31, 32, 47, 63, 64, 65, 127, 128, 511, 512, 513, 1023, 1024, T - 2, T - 1]
    rows = {r for r in edges if 0 <= r < T}
    if n_random >= T:
        rows |= set(range(T))
    else:
        rows |= set(rng.choice(T, size=n_random, replace=False).tolist())
    return sorted(rows)


def check_selection_and_outputs(keyed_rows, gpu_sel, gpu_imp, gpu_out, orc, rerun, op, H_kv, stats):
    """keyed_rows: list of (oracle row key, query position t). gpu_sel [rows, H_kv, n],
    gpu_imp [rows, H_kv, nb], gpu_out [rows, H_q, dv] (numpy); orc = oracle result
    over the same rows; rerun(override) -> oracle output rows with the override."""
    override = {}
    for ri, (key, t) in enumerate(keyed_rows):
        jt = t // op["l_sel"]
        for g in range(H_kv):
            gs = [int(x) for x in gpu_sel[ri, g] if x >= 0]
            osel = orc["sel"][(key, g)]
            oimp = orc["imp"][(key, g)]
            gimp = gpu_imp[ri, g, :jt + 1] if gpu_imp is not None else None
            if gimp is not None and len(oimp):
                scale = max(float(np.max(oimp)), 1e-30)
                d = float(np.max(np.abs(gimp - oimp)))
                assert d <= TOL_IMP * scale + 1e-7, f"importance t={t} g={g}: {d:.3e} (scale {scale:.3e})"
            assert len(gs) == min(op["top_n"], jt + 1), (t, g, gs)
            if gs != osel:
                assert gimp is not None, (t, g, gs, osel)
                assert O.near_tie(oimp, osel, t, op["l_sel"], op["force_first"], op["force_local"], NEAR_TIE), \
                    f"selection differs without a near tie at t={t} g={g}: gpu {gs} oracle {osel}"
                resel = O.select(gimp.astype(np.float64), t, op["l_sel"], op["top_n"], op["force_first"],
                                 op["force_local"])
                assert resel == gs, f"GPU selection not reproducible from its scores at t={t} g={g}"
                override[(key, g)] = gs
                stats["near_ties"] = stats.get("near_ties", 0) + 1
    want = orc["out"] if not override else rerun(override)
    return assert_close(gpu_out, want, "output")


def check_end_to_end(keyed_rows, gpu_sel, gpu_imp, gpu_out, orc, rerun, op, H_kv, stats):
    """GPU rows against the oracle run on its own fp64 compression (see header)."""
    override = {}
    for ri, (key, t) in enumerate(keyed_rows):
        jt = t // op["l_sel"]
        for g in range(H_kv):
            gs = [int(x) for x in gpu_sel[ri, g] if x >= 0]
            osel = orc["sel"][(key, g)]
            if gs == osel:
                continue
            oimp = orc["imp"][(key, g)]
            gimp = gpu_imp[ri, g, :jt + 1]
            lost, extra = set(osel) - set(gs), set(gs) - set(osel)
            a = min(float(oimp[j]) for j in lost)
            b = max(float(oimp[j]) for j in extra)
            assert a - b <= E2E_TIE * max(abs(a), abs(b), 1e-30), \
                f"end to end: selection differs beyond the compression rounding at t={t} g={g}: gpu {gs} oracle {osel}"
            resel = O.select(gimp.astype(np.float64), t, op["l_sel"], op["top_n"], op["force_first"],
                             op["force_local"])
            assert resel == gs, f"GPU selection not reproducible from its scores at t={t} g={g}"
            override[(key, g)] = gs
            stats["e2e_swaps"] = stats.get("e2e_swaps", 0) + 1
    want = orc["out"] if not override else rerun(override)
    return assert_close(gpu_out, want, "output (end to end)", tol_rrms=E2E_RRMS)


def run_prefill_case(cfg, seqlens, n_random_rows=64, seed=None, param_over=None, gates=None, rng_seed=0,
                     e2e_rows=0, k_cmp_fn=None):
    """Full GPU prefill (compress + prefill) on packed sequences; oracle on
    sampled rows of every sequence. Returns stats."""
    param_over = param_over or {}
    inp = W.make_prefill_inputs(cfg, device="cuda", seqlens=seqlens, seed=seed)
    if gates is not None:
        inp["gates"] = gates(inp["gates"])
    heads = heads_of(cfg)
    par = params_of(cfg, **param_over)
    op = oracle_params(cfg, **param_over)
    k_cmp, v_cmp = nsa.compress(inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], seqlens,
                                heads, par)
    stage_only = k_cmp_fn is not None
    if stage_only:   # the case replaces the compressed keys (constructed inputs)
        k_cmp = k_cmp_fn(k_cmp)
    cu = inp["cu_seqlens"]
    ws = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_PREFILL, heads, par, len(seqlens),
                                                    int(cu[-1]), max(seqlens)), "cuda")
    out, sel, imp = nsa.prefill(inp["q"], inp["k"], inp["v"], k_cmp, v_cmp, inp["gates"], cu, heads, par, ws=ws,
                                want_sel=True, want_imp=True)
    torch.cuda.synchronize()
    nsa.nsa_check_device_status(ws)
    rng = np.random.default_rng(rng_seed)
    stats = {}
    w_ck, pe_k, w_cv, pe_v = (f64(inp[x]) for x in ("w_ck", "pe_k", "w_cv", "pe_v"))
    coff = 0
    for b, T in enumerate(seqlens):
        s0 = int(cu[b])
        nc = nsa.n_cmp(T, op["l_cmp"], op["stride"])
        kb = f64(inp["k"][s0:s0 + T])
        vb = f64(inp["v"][s0:s0 + T])
        kcg = f64(k_cmp[coff:coff + nc])
        vcg = f64(v_cmp[coff:coff + nc])
        coff += nc
        kco = vco = None
        if nc and not stage_only:
            kco = O.compress(kb, w_ck, pe_k, op["l_cmp"], op["stride"])
            vco = O.compress(vb, w_cv, pe_v, op["l_cmp"], op["stride"])
            assert_close(kcg, kco, "k_cmp", relative_to_rms=True)
            assert_close(vcg, vco, "v_cmp", relative_to_rms=True)
        if T == 0:
            continue
        rows = sample_rows(T, n_random_rows, rng)
        qb, gb = inp["q"][s0:s0 + T], inp["gates"][s0:s0 + T]   # rows converted on demand
        orc = O.prefill(qb, kb, vb, kcg, vcg, gb, op, rows=rows)
        idx = torch.tensor([s0 + r for r in rows], dtype=torch.long, device="cuda")
        gsel = sel.index_select(0, idx).cpu().numpy()
        gimp = imp.index_select(0, idx).cpu().numpy().astype(np.float64)
        gout = f64(out.index_select(0, idx))

        def rerun(override, qb=qb, kb=kb, vb=vb, kcg=kcg, vcg=vcg, gb=gb, rows=rows):
            return O.prefill(qb, kb, vb, kcg, vcg, gb, op, rows=rows, sel_override=override)["out"]
        m, r = check_selection_and_outputs([(t, t) for t in rows], gsel, gimp, gout, orc, rerun, op, cfg.H_kv,
                                           stats)
        stats.setdefault("max_abs", []).append(m)
        stats.setdefault("rrms", []).append(r)
        stats.setdefault("gpu", []).append(dict(rows=rows, sel=gsel, imp=gimp))
        if e2e_rows and nc and not stage_only:
            pick = sorted(rng.choice(len(rows), size=min(e2e_rows, len(rows)), replace=False).tolist())
            erows = [rows[i] for i in pick]
            orc_e = O.prefill(qb, kb, vb, kco, vco, gb, op, rows=erows)

            def rerun_e(override, qb=qb, kb=kb, vb=vb, kco=kco, vco=vco, gb=gb, erows=erows):
                return O.prefill(qb, kb, vb, kco, vco, gb, op, rows=erows, sel_override=override)["out"]
            m, r = check_end_to_end([(t, t) for t in erows], gsel[pick], gimp[pick], gout[pick], orc_e, rerun_e, op,
                                    cfg.H_kv, stats)
            stats.setdefault("e2e_max_abs", []).append(m)
            stats.setdefault("e2e_rrms", []).append(r)
    return stats


def run_decode_case(cfg, lens=None, batch_rows=None, seed=None, Lmax=None, param_over=None, cmp_rows=None,
                    kc_fn=None):
    """lens=None draws the configuration's own lengths; batch_rows may be a
    function of the drawn lengths. cmp_rows (default: every checked sequence)
    limits the sequences whose compressed caches are recomputed by the oracle
    (a function of the lengths, like batch_rows); kc_fn replaces the compressed
    key cache (constructed inputs)."""
    param_over = param_over or {}
    inp = W.make_decode_inputs(cfg, device="cuda", lens=lens, seed=seed, Lmax=Lmax)
    heads = heads_of(cfg)
    par = params_of(cfg, **param_over)
    op = oracle_params(cfg, **param_over)
    lens_t = inp["cache_lens"]
    kc, vc = nsa.compress_cache(inp["k_cache"], inp["v_cache"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"],
                                lens_t, heads, par)
    if kc_fn is not None:
        kc = kc_fn(kc)
        cmp_rows = []
    max_len = int(inp["k_cache"].shape[1])
    ws = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_DECODE, heads, par, len(lens_t), 0, max_len), "cuda")
    out, sel, imp = nsa.decode(inp["q"], inp["k_cache"], inp["v_cache"], kc, vc, lens_t.to("cuda"), max_len,
                               inp["gates"], heads, par, ws=ws, want_sel=True, want_imp=True)
    torch.cuda.synchronize()
    nsa.nsa_check_device_status(ws)
    B = len(lens_t)
    if callable(batch_rows):
        batch_rows = batch_rows([int(x) for x in lens_t])
    batch_rows = list(range(B)) if batch_rows is None else batch_rows
    if callable(cmp_rows):
        cmp_rows = cmp_rows([int(x) for x in lens_t])
    cmp_rows = set(batch_rows if cmp_rows is None else cmp_rows)
    w_ck, pe_k, w_cv, pe_v = (f64(inp[x]) for x in ("w_ck", "pe_k", "w_cv", "pe_v"))
    gsel_all = sel.cpu().numpy()
    gimp_all = imp.cpu().numpy().astype(np.float64)
    stats = {"gpu": dict(lens=[int(x) for x in lens_t], sel=gsel_all, imp=gimp_all)}
    gout_all = f64(out)
    for b in batch_rows:
        L = int(lens_t[b])
        nc = nsa.n_cmp(L, op["l_cmp"], op["stride"])
        t = L - 1
        if nc and b in cmp_rows:
            kb = f64(inp["k_cache"][b, :L])
            vb = f64(inp["v_cache"][b, :L])
            kco = O.compress(kb, w_ck, pe_k, op["l_cmp"], op["stride"])
            vco = O.compress(vb, w_cv, pe_v, op["l_cmp"], op["stride"])
            assert_close(f64(kc[b, :nc]), kco, "k_cmp cache", relative_to_rms=True)
            assert_close(f64(vc[b, :nc]), vco, "v_cmp cache", relative_to_rms=True)
            # end to end: the oracle on its own fp64 compressed caches
            one = dict(q=inp["q"][b:b + 1], k=inp["k_cache"][b:b + 1], v=inp["v_cache"][b:b + 1],
                       g=inp["gates"][b:b + 1])
            orc_e = O.decode(one["q"], one["k"], one["v"], kco[None], vco[None], [L], one["g"], op)

            def rerun_e(override, one=one, kco=kco, vco=vco, L=L, b=b):
                ov = {(0, g): v for (bb, g), v in override.items()}
                return O.decode(one["q"], one["k"], one["v"], kco[None], vco[None], [L], one["g"], op,
                                sel_override=ov)["out"]
            m, r = check_end_to_end([(0, t)], gsel_all[b:b + 1], gimp_all[b:b + 1], gout_all[b:b + 1], orc_e,
                                    rerun_e, op, cfg.H_kv, stats)
            stats.setdefault("e2e_max_abs", []).append(m)
        orc = O.decode(inp["q"], inp["k_cache"], inp["v_cache"], kc, vc, lens_t, inp["gates"], op, batch_rows=[b])

        def rerun(override, b=b):
            return O.decode(inp["q"], inp["k_cache"], inp["v_cache"], kc, vc, lens_t, inp["gates"], op,
                            batch_rows=[b], sel_override=override)["out"]
        m, r = check_selection_and_outputs([(b, t)], gsel_all[b:b + 1], gimp_all[b:b + 1], gout_all[b:b + 1], orc,
                                           rerun, op, cfg.H_kv, stats)
        stats.setdefault("max_abs", []).append(m)
        stats.setdefault("rrms", []).append(r)
    return stats

