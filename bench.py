"""Benchmark of the NSA forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl nsa|reference]

One step = the whole hot path on one batch of synthetic input: block
compression of K and V, compressed attention + block importance, top-n
selection, selected-block attention, sliding-window attention + gated combine
(the 8K prefill: B=1, T=8192, H_q=64, H_kv=4, d_k=192, d_v=128, l=32, stride 16,
l'=64, top-n 16, w=512). The decode path (B=32 sequences, 64K cache each) is
timed the same way and reported in the "decode" object of the same line.

N > 1 (torchrun, one process per GPU): every rank runs its own replica of the
workload (the path needs no exchange between GPUs: independent sequences);
timings are the max over ranks, value = all ranks' tokens / that time.

--impl reference times the CPU oracle (numpy fp64) on the host cores on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import nsa_workloads as W  # noqa: E402

METRIC = "NSA prefill tokens/s & % bf16 TC peak; 64k decode tokens/s & HBM GB/s"
PREFILL = W.CONFIGS["prefill_8k"]
DECODE = W.CONFIGS["decode_64k"]
L2_FLUSH_BYTES = 256 << 20


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant
# kernels from one ncu capture each, valid only for the kernel source it was taken
# on (the bench reports null once that file changes). The decode capture ran 8
# sequences; its traffic is scaled to the bench's 32 (the stream is per sequence).
NCU_TRAFFIC = {
    "prefill_attn": dict(bytes=232.535808e6 + 102.639360e6, src="prefill.cu",
                         sha1="fe74b5e0732b48a3b4ff97b468fa0b9e4100689f"),
    "dec_cmp": dict(bytes=(84.101376e6 + 2.978816e6) * 32 / 8, src="decode.cu",
                    sha1="dbff8042aebed087fa021e617ebdf2f0475b1f68"),
}


def ncu_traffic(kernel):
    """Measured bytes per launch for `kernel`, or None when unknown or stale."""
    import hashlib
    e = NCU_TRAFFIC.get(kernel)
    if e is None:
        return None
    path = os.path.join(ROOT, "sparse_attention_long_nsa_b200", "csrc", e["src"])
    try:
        with open(path, "rb") as f:
            if hashlib.sha1(f.read()).hexdigest() != e["sha1"]:
                return None
    except OSError:
        return None
    return e["bytes"]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), tc=float(d["bf16_tflops"]), tc_sus=float(d["bf16_tflops_sustained"]),
                    src="measured")
    return dict(hbm=6650.0, tc=1590.0, tc_sus=1400.0, src="fallback")


# ---------------------------------------------------------------------------
# algorithmic work (useful FLOPs / bytes), from the closed-form key counts
# ---------------------------------------------------------------------------

def prefill_pairs(T, cfg):
    """(query, key) pairs per query head for each branch over positions 0..T-1."""
    t = np.arange(T, dtype=np.int64)
    l, s, ls, n, w = cfg.l_cmp, cfg.stride, cfg.l_sel, cfg.top_n, cfg.window
    cmp = np.where(t >= l - 1, (t - l + 1) // s + 1, 0)
    jt = t // ls
    sel = np.where(jt + 1 <= n, t + 1, (n - 1) * ls + (t % ls) + 1)
    win = np.minimum(w, t + 1)
    return int(cmp.sum()), int(sel.sum()), int(win.sum())


def prefill_work(cfg):
    T = cfg.T
    pc, ps, pw = prefill_pairs(T, cfg)
    per_pair = 2 * (cfg.d_k + cfg.d_v) * cfg.H_q
    nc = (T - cfg.l_cmp) // cfg.stride + 1
    comp = 2 * cfg.l_cmp * (cfg.d_k ** 2 + cfg.d_v ** 2) * nc * cfg.H_kv
    return dict(prefill_attn=(pc + ps + pw) * per_pair, compress_gemm=comp,
                total=(pc + ps + pw) * per_pair + comp,
                dense_causal=T * (T + 1) // 2 * per_pair)


def decode_bytes(cfg, lens, sel):
    """Unique K/V bytes the decode must read: every compressed key, and the raw
    keys of the selected blocks united with the window (per KV head)."""
    row = (cfg.d_k + cfg.d_v) * 2
    cmp_b = 0
    fine_b = 0
    sel = sel.cpu().numpy()
    for b, L in enumerate(lens):
        nc = (L - cfg.l_cmp) // cfg.stride + 1 if L >= cfg.l_cmp else 0
        t = L - 1
        for g in range(cfg.H_kv):
            keys = set(range(max(0, t - cfg.window + 1), t + 1))
            for j in sel[b, g]:
                if j >= 0:
                    keys.update(range(j * cfg.l_sel, min((j + 1) * cfg.l_sel, t + 1)))
            fine_b += len(keys) * row
            cmp_b += nc * row
    return cmp_b, fine_b


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for nm, v in zip(names, f[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; no data-path collective)
# ---------------------------------------------------------------------------

def dist_setup(n_gpus):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        rank = int(os.environ["RANK"])
        if backend == "nccl":
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", rank)))
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return rank, ws
    return 0, 1


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------

def timed_steps(step, steps, warmup, flush, ws):
    """Device time of `steps` calls of step(), L2 flushed before each one
    (outside the events). Returns (mean ms per step, max over ranks)."""
    for _ in range(warmup):
        flush()
        step()
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        flush()
        a.record(st)
        step()
        b.record(st)
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in evs) / steps
    return max_over_ranks(ms, ws)


def run_nsa(args, rank, ws):
    import sparse_attention_long_nsa_b200 as nsa
    dev = torch.device("cuda", torch.cuda.current_device())
    pk = peaks()
    cfg = PREFILL
    heads = nsa.Heads(cfg.H_q, cfg.H_kv, cfg.d_k, cfg.d_v)
    par = nsa.make_params(cfg.l_cmp, cfg.stride, cfg.l_sel, cfg.top_n, cfg.window, cfg.force_first,
                          cfg.force_local)
    T = cfg.T
    inp = W.make_prefill_inputs(cfg, device=dev, seed=cfg.seed + 97 * rank)
    cu = inp["cu_seqlens"]
    nc = nsa.n_cmp(T)
    k_cmp = torch.empty((nc, cfg.H_kv, cfg.d_k), dtype=torch.bfloat16, device=dev)
    v_cmp = torch.empty((nc, cfg.H_kv, cfg.d_v), dtype=torch.bfloat16, device=dev)
    out = torch.empty((T, cfg.H_q, cfg.d_v), dtype=torch.bfloat16, device=dev)
    ws_c = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_COMPRESS, heads, par, 1, T, T), dev)
    ws_p = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_PREFILL, heads, par, 1, T, T), dev)
    tok = torch.zeros(1, dtype=torch.int64)
    seq = torch.tensor([T], dtype=torch.int32)
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def flush():
        # evict L2 by writing a buffer twice its size, then read it back so that L2
        # holds clean lines: otherwise the write-back of ~126 MB of dirty lines
        # competes with the first microseconds of the timed kernels
        flush_buf.fill_(1)
        flush_buf.view(torch.int32).max()

    def step():
        nsa.nsa_compress(inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], tok, seq, tok,
                         heads, par, k_cmp, v_cmp, ws_c)
        nsa.nsa_prefill(inp["q"], inp["k"], inp["v"], k_cmp, v_cmp, inp["gates"], cu, heads, par, out, None, None,
                        ws_p)

    # ---- device-timed prefill (the step alone), then a second timed region with
    # the library's per-kernel event profiler on: its events sit between the
    # kernels and add gaps, so the step time is taken without them
    step()
    torch.cuda.synchronize()
    nsa.nsa_check_device_status(ws_p)
    with ClockSampler(torch.cuda.current_device()) as clk:
        ms = timed_steps(step, args.steps, args.warmup, flush, ws)
    nsa.nsa_profile_read()
    nsa.nsa_profile_enable(True)
    psteps = min(args.steps, 50)
    timed_steps(step, psteps, args.warmup, flush, ws)
    prof = nsa.nsa_profile_read()
    nsa.nsa_profile_enable(False)
    nsa.nsa_check_device_status(ws_p)
    # the profile covers warm-up + timed steps of the profiled region
    n_calls = psteps + args.warmup
    launches = sum(c for _, c in prof.values())
    work = prefill_work(cfg)
    kern = {k: v for k, v in prof.items() if v[1] > 0}
    dominant = max(kern, key=lambda k: kern[k][0])
    dom_ms = kern[dominant][0] / kern[dominant][1]
    dom_flops = work.get(dominant, 0)
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12 if dom_flops else None
    tokens = T * ws
    value = tokens / (ms * 1e-3)

    # ---- end to end through the C ABI with host buffers
    host = {k: inp[k].to("cpu").pin_memory() for k in ("q", "k", "v", "gates", "w_ck", "pe_k", "w_cv", "pe_v")}
    dev_bufs = {k: torch.empty_like(inp[k]) for k in host}
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host.numel() * out_host.element_size()

    def e2e_step():
        for k_, t_ in host.items():
            dev_bufs[k_].copy_(t_, non_blocking=True)
        nsa.nsa_compress(dev_bufs["k"], dev_bufs["v"], dev_bufs["w_ck"], dev_bufs["pe_k"], dev_bufs["w_cv"],
                         dev_bufs["pe_v"], tok, seq, tok, heads, par, k_cmp, v_cmp, ws_c)
        nsa.nsa_prefill(dev_bufs["q"], dev_bufs["k"], dev_bufs["v"], k_cmp, v_cmp, dev_bufs["gates"], cu, heads,
                        par, out, None, None, ws_p)
        out_host.copy_(out, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 30))
    ms_e2e = timed_steps(e2e_step, e2e_steps, args.warmup, flush, ws)
    torch.cuda.synchronize()

    # ---- decode (64K cache, B=32): caches built once, then timed
    dcfg = DECODE
    dinp = W.make_decode_inputs(dcfg, device=dev, seed=dcfg.seed + 97 * rank)
    dheads = nsa.Heads(dcfg.H_q, dcfg.H_kv, dcfg.d_k, dcfg.d_v)
    dpar = nsa.make_params(dcfg.l_cmp, dcfg.stride, dcfg.l_sel, dcfg.top_n, dcfg.window, dcfg.force_first,
                           dcfg.force_local)
    lens = dinp["cache_lens"]
    kc, vc = nsa.compress_cache(dinp["k_cache"], dinp["v_cache"], dinp["w_ck"], dinp["pe_k"], dinp["w_cv"],
                                dinp["pe_v"], lens, dheads, dpar)
    lens_d = lens.to(dev)
    Lmax = int(dinp["k_cache"].shape[1])
    ws_d = nsa.alloc_workspace(nsa.nsa_workspace_size(nsa.NSA_OP_DECODE, dheads, dpar, dcfg.B, 0, Lmax), dev)
    dout = torch.empty((dcfg.B, dcfg.H_q, dcfg.d_v), dtype=torch.bfloat16, device=dev)
    dsel = torch.empty((dcfg.B, dcfg.H_kv, dcfg.top_n), dtype=torch.int32, device=dev)

    def dstep():
        nsa.nsa_decode(dinp["q"], dinp["k_cache"], dinp["v_cache"], kc, vc, lens_d, Lmax, dinp["gates"], dheads,
                       dpar, dout, dsel, None, ws_d)

    dstep()
    torch.cuda.synchronize()
    nsa.nsa_check_device_status(ws_d)
    dsteps = max(args.steps, 20)
    dms = timed_steps(dstep, dsteps, args.warmup, flush, ws)
    nsa.nsa_check_device_status(ws_d)
    nsa.nsa_profile_read()
    nsa.nsa_profile_enable(True)
    dpsteps = min(dsteps, 50)
    timed_steps(dstep, dpsteps, args.warmup, flush, ws)
    dprof = nsa.nsa_profile_read()
    nsa.nsa_profile_enable(False)
    cmp_b, fine_b = decode_bytes(dcfg, [int(x) for x in lens], dsel)
    dbytes = cmp_b + fine_b
    dgbs = dbytes / (dms * 1e-3) / 1e9
    dk = {k: v for k, v in dprof.items() if v[1] > 0}
    d_dom = max(dk, key=lambda k: dk[k][0])
    d_dom_ms = dk[d_dom][0] / dk[d_dom][1]
    d_dom_bytes = cmp_b if d_dom == "dec_cmp" else (fine_b if d_dom == "dec_fine" else None)

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = oracle_prefill_rate(inp, cfg, budget_s=args.cpu_seconds)

    if rank != 0:
        return None
    res = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) q/k/v, N(0,1/(l*d)) compression weights, sigmoid(N(0,1)) gates)",
        "config": {
            "workload": "prefill_8k: B=1 T=8192 causal, H_q=64 H_kv=4, d_k=192 d_v=128, l=32 stride=16 "
                        "l'=64 top-n=16 (1 initial + 2 local forced) w=512; step = nsa_compress + nsa_prefill",
            "global_batch": ws, "seq_len": T, "parallelism": f"replicas x{ws}",
            "l2": "flushed before every timed step (256 MB write, then a read of it, outside the events)",
            "useful_flop_per_step": work["total"], "dense_causal_flop_per_step": work["dense_causal"],
        },
        "tflops_useful": work["total"] / (ms * 1e-3) / 1e12 * ws,
        "tc_frac_useful": work["total"] / (ms * 1e-3) / 1e12 / pk["tc"],
        "roofline": {
            "kernel": dominant, "bound": "tensor",
            "achieved": achieved, "peak": pk["tc"], "unit": "TFLOP/s",
            "frac": (achieved / pk["tc"]) if achieved else None,
            "peak_source": f"{pk['src']} bf16 dense (burst)",
            "traffic": ncu_traffic(dominant),
            "ms_per_launch": dom_ms,
            "algorithmic_flop_per_launch": dom_flops,
        },
        "kernels_ms_per_step": {k: v[0] / n_calls for k, v in kern.items()},
        "gpu_launches": int(round(launches / n_calls)) * args.steps,
        "e2e": {"value": tokens / (ms_e2e * 1e-3), "unit": "tokens/s", "ms_per_step": ms_e2e,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clk.summary(),
        "decode": {
            "workload": "decode_64k: B=32 x 1 query, cache 65536 each, H_q=64 H_kv=4, d_k=192 d_v=128",
            "tokens_per_s": dcfg.B * ws / (dms * 1e-3), "ms_per_step": dms,
            "bytes_per_step": dbytes, "bytes_compressed": cmp_b, "bytes_fine": fine_b,
            "hbm_gbs": dgbs, "hbm_frac": dgbs / pk["hbm"], "hbm_peak_gbs": pk["hbm"],
            "kernels_ms_per_step": {k: v[0] / (dpsteps + args.warmup) for k, v in dk.items()},
            "roofline": {"kernel": d_dom, "bound": "hbm",
                         "achieved": (d_dom_bytes / (d_dom_ms * 1e-3) / 1e9) if d_dom_bytes else None,
                         "peak": pk["hbm"], "unit": "GB/s",
                         "frac": (d_dom_bytes / (d_dom_ms * 1e-3) / 1e9 / pk["hbm"]) if d_dom_bytes else None,
                         "traffic": ncu_traffic(d_dom)},
        },
        "cpu_baseline": cpu,
    }
    return res


# ---------------------------------------------------------------------------
# the oracle, timed on the host (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------

def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_prefill_rate(inp, cfg, budget_s=15.0, max_rows=None):
    """Oracle tokens/s on the 8K prefill: the full compression of K and V, plus
    evenly spaced query rows until the time budget is spent; the rate is T over
    (compression time + T x mean time per row)."""
    from oracle import nsa_oracle as O
    p = cfg.params()
    T = cfg.T
    k = inp["k"].double().cpu().numpy()
    v = inp["v"].double().cpu().numpy()
    t0 = time.perf_counter()
    kc = O.compress(k, inp["w_ck"].double().cpu().numpy(), inp["pe_k"].double().cpu().numpy(), p["l_cmp"],
                    p["stride"])
    vc = O.compress(v, inp["w_cv"].double().cpu().numpy(), inp["pe_v"].double().cpu().numpy(), p["l_cmp"],
                    p["stride"])
    t_cmp = time.perf_counter() - t0
    q = inp["q"]
    g = inp["gates"]
    order = np.random.default_rng(0).permutation(T)
    done = 0
    t1 = time.perf_counter()
    while done < T and (time.perf_counter() - t1) < budget_s and (max_rows is None or done < max_rows):
        batch = order[done:done + 16]
        O.prefill(q, k, v, kc, vc, g, p, rows=batch.tolist())
        done += len(batch)
    t_rows = time.perf_counter() - t1
    est = t_cmp + T * t_rows / max(done, 1)
    return {"value": T / est, "unit": "tokens/s", "cores": _threads(), "kind": "oracle",
            "sample": f"full K/V compression ({t_cmp:.1f} s) + {done} of {T} query rows drawn uniformly "
                      f"({t_rows:.1f} s); rate = T / (compression + T x mean row time)",
            "host_cpus": os.cpu_count()}


def run_reference(args, rank, ws):
    if rank != 0:
        return None
    cfg = PREFILL
    inp = W.make_prefill_inputs(cfg, device="cpu")
    vals = []
    budget = max(2.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup + args.steps):
        r = oracle_prefill_rate(inp, cfg, budget_s=budget, max_rows=64)
        if i >= args.warmup:
            vals.append(r)
    value = float(np.mean([r["value"] for r in vals]))
    ms = cfg.T / value * 1e3
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "prefill_8k (as the nsa arm), CPU oracle on a bounded sample per step",
                   "global_batch": 1, "seq_len": cfg.T, "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": vals[-1]["cores"], "kind": "oracle",
                         "sample": vals[-1]["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_case(case):
    """Two untimed invocations of one workload, for kernel profilers (no JSON line):
    prefill = compression + prefill of the 8K workload; decode = 8 sequences of the
    64K decode workload."""
    import sparse_attention_long_nsa_b200 as nsa
    dev = torch.device("cuda", 0)
    if case == "prefill":
        cfg = PREFILL
        inp = W.make_prefill_inputs(cfg, device=dev)
        heads = nsa.Heads(cfg.H_q, cfg.H_kv, cfg.d_k, cfg.d_v)
        par = nsa.make_params(cfg.l_cmp, cfg.stride, cfg.l_sel, cfg.top_n, cfg.window, cfg.force_first,
                              cfg.force_local)
        for _ in range(2):
            kc, vc = nsa.compress(inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], [cfg.T],
                                  heads, par)
            nsa.prefill(inp["q"], inp["k"], inp["v"], kc, vc, inp["gates"], inp["cu_seqlens"], heads, par)
    else:
        cfg = DECODE
        inp = W.make_decode_inputs(cfg, device=dev, lens=[cfg.T] * 8)
        heads = nsa.Heads(cfg.H_q, cfg.H_kv, cfg.d_k, cfg.d_v)
        par = nsa.make_params(cfg.l_cmp, cfg.stride, cfg.l_sel, cfg.top_n, cfg.window, cfg.force_first,
                              cfg.force_local)
        kc, vc = nsa.compress_cache(inp["k_cache"], inp["v_cache"], inp["w_ck"], inp["pe_k"], inp["w_cv"],
                                    inp["pe_v"], inp["cache_lens"], heads, par)
        lens = inp["cache_lens"].to(dev)
        for _ in range(2):
            nsa.decode(inp["q"], inp["k_cache"], inp["v_cache"], kc, vc, lens, cfg.T, inp["gates"], heads, par)
    torch.cuda.synchronize()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["nsa", "reference"], default="nsa")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", choices=["prefill", "decode"], default=None,
                    help="run two untimed invocations of one workload for a profiler, print nothing")
    args = ap.parse_args()
    if args.case:
        run_case(args.case)
        return
    if args.warmup < 3:
        args.warmup = 3
    rank, ws = dist_setup(args.gpus)
    try:
        res = run_reference(args, rank, ws) if args.impl == "reference" else run_nsa(args, rank, ws)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
