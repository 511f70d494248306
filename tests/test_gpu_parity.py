"""GPU parity: the CUDA path (called through the C ABI) against the CPU oracle
on the same seeded inputs. See tests/nsa_parity.py for the acceptance rules."""
import numpy as np
import pytest
import torch

import nsa_workloads as W
import sparse_attention_long_nsa_b200 as nsa
from oracle import nsa_oracle as O
from tests import nsa_parity as NP

pytestmark = pytest.mark.gpu

CFG = W.CONFIGS


def test_prefill_tiny_full():
    """1024-token GQA-4 prefill, every row compared."""
    st = NP.run_prefill_case(CFG["prefill_tiny_1k"], [1024], n_random_rows=1024)
    assert max(st["max_abs"]) <= NP.TOL_MAX


@pytest.mark.parametrize("seqlens", [[100, 1000, 37], [31, 32, 33, 64, 65], [1], [700]])
def test_prefill_tiny_varlen(seqlens):
    NP.run_prefill_case(CFG["prefill_tiny_1k"], seqlens, n_random_rows=400, seed=7)


@pytest.mark.parametrize("seqlens", [[1500], [700, 64, 1300]])
def test_prefill_gqa16_ragged(seqlens):
    """H_q=64, H_kv=4, d_k=192, d_v=128 at lengths spanning several tiles and a ragged tail."""
    NP.run_prefill_case(CFG["prefill_8k"], seqlens, n_random_rows=128, seed=11)


def test_prefill_8k_sampled():
    """The benched 8K prefill, in the same launch configuration, on sampled rows;
    64 of them also end to end against the oracle's own fp64 compression."""
    st = NP.run_prefill_case(CFG["prefill_8k"], [8192], n_random_rows=1024, e2e_rows=64)
    assert st["e2e_max_abs"]


def test_prefill_64k_sampled():
    """The 64K prefill in the benched launch configuration: 1024 random rows plus
    the edges, 64 of them also end to end."""
    st = NP.run_prefill_case(CFG["prefill_64k"], [65536], n_random_rows=1024, e2e_rows=64)
    assert st["e2e_max_abs"]


def _ties_checked(stats, op, H_kv):
    """Every checked row whose free candidates hold exact ties at the selection
    boundary picks the lowest indices among them (the GPU's set must equal the
    oracle's selection rule applied to the GPU's own scores, compared exactly).
    Returns how many (row, group) pairs had such a tie."""
    n_tied = 0
    for rec in stats["gpu"] if isinstance(stats["gpu"], list) else [stats["gpu"]]:
        rows = rec["rows"] if "rows" in rec else [L - 1 for L in rec["lens"]]
        for ri, t in enumerate(rows):
            jt = t // op["l_sel"]
            if jt + 1 <= op["top_n"]:
                continue
            for g in range(H_kv):
                imp = rec["imp"][ri, g, :jt + 1].astype(np.float64)
                gs = [int(x) for x in rec["sel"][ri, g] if x >= 0]
                want = O.select(imp, t, op["l_sel"], op["top_n"], op["force_first"], op["force_local"])
                assert gs == want, f"t={t} g={g}: gpu {gs}, lowest-index rule on the gpu's scores {want}"
                forced = O.forced_blocks(t, op["l_sel"], op["force_first"], op["force_local"])
                free = sorted((float(imp[j]) for j in range(jt + 1) if j not in forced), reverse=True)
                need = op["top_n"] - len(forced)
                if need < len(free) and free[need - 1] == free[need]:
                    n_tied += 1
    return n_tied


def _zero_keys(kc):
    return torch.zeros_like(kc)


def test_prefill_beyond_64k_radix_topn_and_ties():
    """66,000 tokens: 1032 candidate blocks, beyond the register top-n (the radix
    select path); 256 random rows plus the edges. Then the same sequence with all
    compressed keys zero: every compressed probability of a row is equal, so the
    interior blocks tie exactly and the lowest indices must win."""
    cfg = W.small_config(name="prefill_66k", T=66000, H_q=64, H_kv=4, d_k=192, d_v=128, seed=1005)
    NP.run_prefill_case(cfg, [66000], n_random_rows=256)
    st = NP.run_prefill_case(cfg, [66000], n_random_rows=64, k_cmp_fn=_zero_keys)
    assert _ties_checked(st, cfg.params(), cfg.H_kv) > 0


def test_prefill_importance_through_workspace():
    """80,000 tokens (1250 candidate blocks): the tile's importance rows no longer
    fit in shared memory next to two V stages, so they go through the fp32
    workspace; 128 random rows plus the edges."""
    cfg = W.small_config(name="prefill_80k", T=80000, H_q=16, H_kv=1, d_k=192, d_v=128, seed=1006)
    NP.run_prefill_case(cfg, [80000], n_random_rows=128)


def test_compress_prepared_weights_match():
    """nsa_compress_prepared with weights from nsa_compress_prepare writes the same
    bits as nsa_compress (the same conversion, once instead of per call), over
    several sequences, for two head shapes."""
    for cfg_name, seqlens in (("prefill_8k", [1500, 64, 700, 31]), ("prefill_tiny_1k", [1024, 333])):
        cfg = CFG[cfg_name]
        heads, par = NP.heads_of(cfg), NP.params_of(cfg)
        inp = W.make_prefill_inputs(cfg, device="cuda", seqlens=seqlens, seed=31)
        args = (inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], seqlens, heads, par)
        kc, vc = nsa.compress(*args)
        prepared = nsa.compress_prepare(inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], heads, par)
        for _ in range(2):   # the blob is read, not consumed
            kp, vp = nsa.compress(*args, prepared=prepared)
            torch.cuda.synchronize()
            assert torch.equal(kp.view(torch.int16), kc.view(torch.int16))
            assert torch.equal(vp.view(torch.int16), vc.view(torch.int16))


def test_prefill_exact_ties_register_topn():
    """All compressed keys zero (exact ties between interior blocks) on the
    register top-n path of the prefill (GQA 16 and GQA 4)."""
    for cfg, T in ((CFG["prefill_8k"], 4000), (CFG["prefill_tiny_1k"], 1024)):
        st = NP.run_prefill_case(cfg, [T], n_random_rows=256, k_cmp_fn=_zero_keys)
        assert _ties_checked(st, cfg.params(), cfg.H_kv) > 0


def test_prefill_exact_ties_register_radix_topn():
    """All compressed keys zero at 40,000 tokens (625 candidate blocks, the
    register radix top-n): interior blocks tie exactly and the lowest indices
    must win."""
    cfg = W.small_config(name="prefill_40k", T=40000, H_q=64, H_kv=4, d_k=192, d_v=128, seed=1007)
    st = NP.run_prefill_case(cfg, [40000], n_random_rows=64, k_cmp_fn=_zero_keys)
    assert _ties_checked(st, cfg.params(), cfg.H_kv) > 0


def _dense_ref(inp, G, scale):
    q = inp["q"].double().permute(1, 0, 2)[None]
    k = inp["k"].double().repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    v = inp["v"].double().repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)[0].permute(1, 0, 2)


@pytest.mark.parametrize("branch", ["slc", "win"])
def test_prefill_dense_reduction(branch):
    """top-n covering every block (gates 0,1,0) or a window >= T (gates 0,0,1)
    reduces NSA to dense causal attention."""
    cfg = W.small_config(T=1000, H_q=16, H_kv=1, d_k=128, d_v=128, top_n=16, window=64, seed=5)
    T = cfg.T
    inp = W.make_prefill_inputs(cfg, device="cuda")
    e = torch.zeros_like(inp["gates"])
    e[..., 1 if branch == "slc" else 2] = 1.0
    over = dict(top_n=16) if branch == "slc" else dict(window=T + 3)
    heads = NP.heads_of(cfg)
    par = NP.params_of(cfg, **over)
    kc, vc = nsa.compress(inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], [T], heads, par)
    out = nsa.prefill(inp["q"], inp["k"], inp["v"], kc, vc, e, inp["cu_seqlens"], heads, par)
    torch.cuda.synchronize()
    ref = _dense_ref(inp, cfg.G, 1.0 / np.sqrt(cfg.d_k)).cpu().numpy()
    NP.assert_close(NP.f64(out), ref, f"dense reduction ({branch})")


def test_prefill_gate_linearity():
    cfg = CFG["prefill_tiny_1k"]
    inp = W.make_prefill_inputs(cfg, device="cuda", seqlens=[777])
    heads, par = NP.heads_of(cfg), NP.params_of(cfg)
    kc, vc = nsa.compress(inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], [777], heads, par)
    full = nsa.prefill(inp["q"], inp["k"], inp["v"], kc, vc, inp["gates"], inp["cu_seqlens"], heads, par).double()
    acc = torch.zeros_like(full)
    for b in range(3):
        e = torch.zeros_like(inp["gates"])
        e[..., b] = 1.0
        ob = nsa.prefill(inp["q"], inp["k"], inp["v"], kc, vc, e, inp["cu_seqlens"], heads, par).double()
        acc += inp["gates"][..., b:b + 1].double() * ob
    NP.assert_close(full.cpu().numpy(), acc.cpu().numpy(), "gate linearity")


def test_prefill_deterministic():
    cfg = CFG["prefill_tiny_1k"]
    inp = W.make_prefill_inputs(cfg, device="cuda")
    heads, par = NP.heads_of(cfg), NP.params_of(cfg)
    kc, vc = nsa.compress(inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], [1024], heads, par)
    a = nsa.prefill(inp["q"], inp["k"], inp["v"], kc, vc, inp["gates"], inp["cu_seqlens"], heads, par,
                    want_sel=True)
    b = nsa.prefill(inp["q"], inp["k"], inp["v"], kc, vc, inp["gates"], inp["cu_seqlens"], heads, par,
                    want_sel=True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("d_k,d_v", [(dk, dv) for dk in (64, 128, 192) for dv in (64, 128)])
def test_compress_every_head_size_pair(d_k, d_v):
    """Keys and values of every supported (d_k, d_v) pair share one GEMM launch
    (one instantiation per pair; d_v = 192 is rejected on the host, checked in
    the CPU tests): both maps against the fp64 oracle over two
    sequences, one of them with a ragged tail; the K reduction is split (few row
    tiles)."""
    seqlens = [600, 77]
    cfg = W.small_config(T=sum(seqlens), H_q=8, H_kv=2, d_k=d_k, d_v=d_v, seed=41)
    heads, par = NP.heads_of(cfg), NP.params_of(cfg)
    inp = W.make_prefill_inputs(cfg, device="cuda", seqlens=seqlens, seed=41)
    kc, vc = nsa.compress(inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], seqlens, heads,
                          par)
    torch.cuda.synchronize()
    op = NP.oracle_params(cfg)
    w_ck, pe_k, w_cv, pe_v = (NP.f64(inp[x]) for x in ("w_ck", "pe_k", "w_cv", "pe_v"))
    t0 = c0 = 0
    for L in seqlens:
        nc = nsa.n_cmp(L, par.l_cmp, par.stride)
        kb, vb = NP.f64(inp["k"][t0:t0 + L]), NP.f64(inp["v"][t0:t0 + L])
        NP.assert_close(NP.f64(kc[c0:c0 + nc]), O.compress(kb, w_ck, pe_k, op["l_cmp"], op["stride"]),
                        f"k_cmp d_k={d_k}", relative_to_rms=True)
        NP.assert_close(NP.f64(vc[c0:c0 + nc]), O.compress(vb, w_cv, pe_v, op["l_cmp"], op["stride"]),
                        f"v_cmp d_v={d_v}", relative_to_rms=True)
        t0 += L
        c0 += nc


def test_compress_mean_pool_on_gpu():
    """Averaging weights, no position embedding, stride = block: the compressed
    keys are the block means (up to bf16 rounding of the weights 1/32)."""
    cfg = CFG["prefill_tiny_1k"]
    inp = W.make_prefill_inputs(cfg, device="cuda", seqlens=[640])
    d = cfg.d_k
    Wm = torch.cat([torch.eye(d)] * 32, 0).cuda() / 32
    pe = torch.zeros(32, d, device="cuda")
    heads = NP.heads_of(cfg)
    kc, _ = nsa.compress(inp["k"], inp["v"], Wm, pe, Wm, pe, [640], heads, NP.params_of(cfg))
    # stride 16 rows; blocks starting at multiples of 32 are rows 0, 2, 4, ...
    means = inp["k"].double().reshape(20, 32, 1, d).mean(1)
    NP.assert_close(NP.f64(kc[0::2]), means.cpu().numpy(), "mean-pool compression", relative_to_rms=True)


@pytest.mark.parametrize("lens", [[8192, 3000, 33, 1], [31, 32, 64, 65, 127, 128, 129, 1000]])
def test_decode_small(lens):
    cfg = CFG["decode_64k"]
    NP.run_decode_case(cfg, lens, seed=3)


def test_decode_matches_prefill_last_row():
    """The decode kernels and the prefill kernels agree on the last position."""
    cfg = CFG["prefill_8k"]
    T = 3000
    inp = W.make_prefill_inputs(cfg, device="cuda", seqlens=[T])
    heads, par = NP.heads_of(cfg), NP.params_of(cfg)
    kc, vc = nsa.compress(inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], [T], heads, par)
    out_p, sel_p = nsa.prefill(inp["q"], inp["k"], inp["v"], kc, vc, inp["gates"], inp["cu_seqlens"], heads, par,
                               want_sel=True)
    lens = torch.tensor([T], dtype=torch.int32, device="cuda")
    out_d, sel_d = nsa.decode(inp["q"][T - 1:T].contiguous(), inp["k"][None], inp["v"][None], kc[None], vc[None],
                              lens, T, inp["gates"][T - 1:T].contiguous(), heads, par, want_sel=True)
    torch.cuda.synchronize()
    assert torch.equal(sel_p[T - 1], sel_d[0])
    NP.assert_close(NP.f64(out_d[0]), NP.f64(out_p[T - 1]), "decode vs prefill")


def test_decode_64k_all_sequences():
    """The benched 64K decode batch: every one of the 32 sequences (selection and
    output); the compressed caches of four of them recomputed by the oracle, and
    those four also end to end."""
    cfg = CFG["decode_64k"]
    NP.run_decode_case(cfg, [cfg.T] * cfg.B, cmp_rows=[0, 7, 13, 31])


def test_decode_varlen_all_sequences():
    """The varlen decode batch (64 cache lengths drawn in [8192, 131072]): every
    sequence; the shortest, median and longest compressed caches recomputed by
    the oracle (and checked end to end)."""
    cfg = CFG["decode_varlen"]

    def pick(lens):
        order = np.argsort(lens)
        return [int(order[0]), int(order[len(lens) // 2]), int(order[-1])]
    NP.run_decode_case(cfg, None, cmp_rows=pick)


def test_decode_longest_caches_fallback_topn_and_ties():
    """The longest supported cache (262,144 tokens: 4096 candidate blocks, beyond
    the CTA-wide top-n, so the warp radix select runs) next to a 170,001-token and
    a short cache; then the same caches with zero compressed keys (exact ties)."""
    cfg = CFG["decode_64k"]
    lens = [262144, 170001, 5000]
    NP.run_decode_case(cfg, lens, seed=41, cmp_rows=[2])
    st = NP.run_decode_case(cfg, lens, seed=41, kc_fn=_zero_keys)
    assert _ties_checked(st, cfg.params(), cfg.H_kv) > 0


def test_decode_exact_ties_cta_topn():
    """Zero compressed keys on the CTA-wide top-n path (up to 2560 candidates)."""
    cfg = CFG["decode_64k"]
    st = NP.run_decode_case(cfg, [20000, 65536, 3001, 160000], seed=43, kc_fn=_zero_keys)
    assert _ties_checked(st, cfg.params(), cfg.H_kv) > 0


def test_decode_work_counter_returns_to_zero():
    """The compressed decode pass takes its (sequence, KV head, chunk) items from
    a counter in the workspace header. After every call the counter words are 0
    again, so calls that reuse one workspace (with fewer items than SMs, and with
    more) give the same bytes as a call on a fresh workspace."""
    cfg = CFG["decode_64k"]
    heads, par = NP.heads_of(cfg), NP.params_of(cfg)
    for lens in ([1, 700, 20000], [65536] * 8 + [3001, 160000]):
        inp = W.make_decode_inputs(cfg, device="cuda", lens=lens, seed=47)
        lens_t = inp["cache_lens"].to("cuda")
        kc, vc = nsa.compress_cache(inp["k_cache"], inp["v_cache"], inp["w_ck"], inp["pe_k"], inp["w_cv"],
                                    inp["pe_v"], inp["cache_lens"], heads, par)
        max_len = int(inp["k_cache"].shape[1])
        nbytes = nsa.nsa_workspace_size(nsa.NSA_OP_DECODE, heads, par, len(lens), 0, max_len)
        outs = []
        for ws in [nsa.alloc_workspace(nbytes, "cuda")] * 3 + [nsa.alloc_workspace(nbytes, "cuda")]:
            out, sel = nsa.decode(inp["q"], inp["k_cache"], inp["v_cache"], kc, vc, lens_t, max_len, inp["gates"],
                                  heads, par, ws=ws, want_sel=True)
            torch.cuda.synchronize()
            nsa.nsa_check_device_status(ws)
            hdr = ws[:16].cpu().numpy().view(np.uint32)
            assert hdr[2] == 0 and hdr[3] == 0, hdr
            outs.append((out.clone(), sel.clone()))
        for out, sel in outs[1:]:
            assert torch.equal(out, outs[0][0]) and torch.equal(sel, outs[0][1])


def test_decode_incremental_compressed_cache():
    """A decode loop that appends one token per sequence and step and compresses each
    newly completed block (compress_append) builds the same compressed caches as the
    fp64 oracle compressing the grown sequences, and as one call over the whole cache."""
    cfg = CFG["decode_64k"]
    lens0, steps = [20, 100, 1001, 4090], 48
    lens_end = [L + steps for L in lens0]
    inp = W.make_decode_inputs(cfg, device="cuda", lens=lens_end, seed=31)
    heads, par, op = NP.heads_of(cfg), NP.params_of(cfg), NP.oracle_params(cfg)
    kc, vc = nsa.compress_cache(inp["k_cache"], inp["v_cache"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"],
                                lens0, heads, par)
    ws = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_COMPRESS, heads, par, len(lens0), 0, 0), "cuda")
    written = 0
    for step in range(1, steps + 1):
        written += nsa.compress_append(inp["k_cache"], inp["v_cache"], inp["w_ck"], inp["pe_k"], inp["w_cv"],
                                       inp["pe_v"], [L + step for L in lens0], kc, vc, heads, par, ws=ws)
    torch.cuda.synchronize()
    nsa.nsa_check_device_status(ws)
    assert written == sum(nsa.n_cmp(L + steps) - nsa.n_cmp(L) for L in lens0)
    kc1, vc1 = nsa.compress_cache(inp["k_cache"], inp["v_cache"], inp["w_ck"], inp["pe_k"], inp["w_cv"],
                                  inp["pe_v"], lens_end, heads, par)
    w_ck, pe_k, w_cv, pe_v = (NP.f64(inp[x]) for x in ("w_ck", "pe_k", "w_cv", "pe_v"))
    for b, L in enumerate(lens_end):
        nc = nsa.n_cmp(L)
        if nc == 0:
            continue
        kb, vb = NP.f64(inp["k_cache"][b, :L]), NP.f64(inp["v_cache"][b, :L])
        NP.assert_close(NP.f64(kc[b, :nc]), O.compress(kb, w_ck, pe_k, op["l_cmp"], op["stride"]), "appended k_cmp",
                        relative_to_rms=True)
        NP.assert_close(NP.f64(vc[b, :nc]), O.compress(vb, w_cv, pe_v, op["l_cmp"], op["stride"]), "appended v_cmp",
                        relative_to_rms=True)
        # same kernel arithmetic per block: at most a bf16 rounding step apart from one call
        d = (kc[b, :nc].float() - kc1[b, :nc].float()).abs()
        assert float(d.max()) <= 2.0 ** -7 * float(kc1[b, :nc].float().abs().max())


def test_decode_incremental_growth_by_chunks():
    """Sequences that grow by several tokens at a time (7, 16, 33 and 500 per round,
    one size per sequence) through nsa_compress_append with the previous lengths:
    each call writes one segment of many blocks per sequence into the compressed
    caches in place; the grown caches match the fp64 oracle and one call over the
    whole cache."""
    cfg = CFG["decode_64k"]
    lens0, grow, rounds = [20, 100, 1001, 4090], [7, 16, 33, 500], 5
    lens_end = [L + g * rounds for L, g in zip(lens0, grow)]
    inp = W.make_decode_inputs(cfg, device="cuda", lens=lens_end, seed=37)
    heads, par, op = NP.heads_of(cfg), NP.params_of(cfg), NP.oracle_params(cfg)
    kc, vc = nsa.compress_cache(inp["k_cache"], inp["v_cache"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"],
                                lens0, heads, par)
    ws = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_COMPRESS, heads, par, len(lens0), 0, 0), "cuda")
    written = 0
    for r in range(1, rounds + 1):
        prev = [L + g * (r - 1) for L, g in zip(lens0, grow)]
        cur = [L + g * r for L, g in zip(lens0, grow)]
        written += nsa.compress_append(inp["k_cache"], inp["v_cache"], inp["w_ck"], inp["pe_k"], inp["w_cv"],
                                       inp["pe_v"], cur, kc, vc, heads, par, ws=ws, lens_prev=prev)
    torch.cuda.synchronize()
    nsa.nsa_check_device_status(ws)
    assert written == sum(nsa.n_cmp(b) - nsa.n_cmp(a) for a, b in zip(lens0, lens_end))
    kc1, vc1 = nsa.compress_cache(inp["k_cache"], inp["v_cache"], inp["w_ck"], inp["pe_k"], inp["w_cv"],
                                  inp["pe_v"], lens_end, heads, par)
    w_ck, pe_k, w_cv, pe_v = (NP.f64(inp[x]) for x in ("w_ck", "pe_k", "w_cv", "pe_v"))
    for b, L in enumerate(lens_end):
        nc = nsa.n_cmp(L)
        kb, vb = NP.f64(inp["k_cache"][b, :L]), NP.f64(inp["v_cache"][b, :L])
        NP.assert_close(NP.f64(kc[b, :nc]), O.compress(kb, w_ck, pe_k, op["l_cmp"], op["stride"]), "grown k_cmp",
                        relative_to_rms=True)
        NP.assert_close(NP.f64(vc[b, :nc]), O.compress(vb, w_cv, pe_v, op["l_cmp"], op["stride"]), "grown v_cmp",
                        relative_to_rms=True)
        d = (kc[b, :nc].float() - kc1[b, :nc].float()).abs()
        assert float(d.max()) <= 2.0 ** -7 * float(kc1[b, :nc].float().abs().max())


# GQA groups of 8, 2 and 1 heads take the other compile-time head reductions of the
# importance; with them the remaining supported (d_k, d_v) pairs
GROUP_SHAPES = [(8, 1, 128, 64), (4, 2, 64, 128), (4, 4, 192, 64)]


@pytest.mark.parametrize("H_q,H_kv,d_k,d_v", GROUP_SHAPES)
def test_prefill_group_sizes(H_q, H_kv, d_k, d_v):
    """Ragged batch with an empty sequence and a one-token sequence."""
    cfg = W.small_config(T=1100, H_q=H_q, H_kv=H_kv, d_k=d_k, d_v=d_v, top_n=16, window=256, seed=21)
    NP.run_prefill_case(cfg, [0, 1100, 1, 257], n_random_rows=96, seed=21)


@pytest.mark.parametrize("H_q,H_kv,d_k,d_v", GROUP_SHAPES)
def test_decode_group_sizes(H_q, H_kv, d_k, d_v):
    cfg = W.small_config(T=3000, H_q=H_q, H_kv=H_kv, d_k=d_k, d_v=d_v, top_n=16, window=256, seed=22)
    NP.run_decode_case(cfg, lens=[3000, 1, 31, 32, 700], seed=22)
