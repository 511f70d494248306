"""In-kernel timelines of the prefill and decode kernels.

    python -m sparse_attention_long_nsa_b200.trace prefill      # 8K prefill
    python -m sparse_attention_long_nsa_b200.trace prefill64k   # 64K prefill, one KV group
    python -m sparse_attention_long_nsa_b200.trace decode    # 64K decode, B=32

Builds a copy of libnsa.so with the compile-time trace points on
(-DNSA_PREFILL_TRACE -DNSA_DECODE_TRACE) into _build/trace/, runs the workload a
few times and prints a summary of the last launch:

* prefill: for four CTAs (KV head 0, the last query tile of each quarter), the clock64
  at the end of each phase (C1, C2, top-n, W, S) and, per 64-key tile, when its S
  was ready for the softmax, when the softmax finished it, and when the S and P.V
  products were issued; then the mean tile period and softmax latency of the
  selected-block phase.
* decode: per fine-pass CTA (KV head 0, sequences 0..7) the clock64 at the end of
  each prologue step, and the global-timer spans of every CTA of both kernels.

The trace points cost a few percent of the kernels' time; the library build is
not affected.
"""
from __future__ import annotations

import ctypes
import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from . import build as _b

OUT = os.path.join(_b.ROOT, "_build", "trace")


def build_trace_lib() -> str:
    os.makedirs(OUT, exist_ok=True)
    lib = os.path.join(OUT, "libnsa.so")
    srcs = glob.glob(os.path.join(_b.CSRC, "*")) + [os.path.join(_b.ROOT, "include", "nsa.h")]
    if os.path.exists(lib) and os.path.getmtime(lib) > max(os.path.getmtime(x) for x in srcs):
        return lib
    flags = [*_b.ARCH, *_b.FLAGS, "-DNSA_PREFILL_TRACE", "-DNSA_DECODE_TRACE"]

    def comp(src):
        o = os.path.join(OUT, os.path.basename(src) + ".o")
        r = subprocess.run([_b.NVCC, *flags, "-c", src, "-o", o], capture_output=True, text=True)
        if r.returncode:
            raise RuntimeError(r.stderr)
        return o

    with ThreadPoolExecutor(8) as ex:
        objs = list(ex.map(comp, sorted(glob.glob(os.path.join(_b.CSRC, "*.cu")))))
    subprocess.run([_b.NVCC, *_b.ARCH, "-shared", "-o", lib, *objs, "-lcudart"], check=True)
    return lib


def _prefill(nsa, L, long=False):
    import dataclasses
    import torch
    import nsa_workloads as W
    cfg = W.CONFIGS["prefill_8k"]
    if long:
        cfg = dataclasses.replace(W.CONFIGS["prefill_64k"], H_q=16, H_kv=1)
    inp = W.make_prefill_inputs(cfg, device="cuda")
    heads = nsa.Heads(cfg.H_q, cfg.H_kv, cfg.d_k, cfg.d_v)
    par = nsa.make_params(cfg.l_cmp, cfg.stride, cfg.l_sel, cfg.top_n, cfg.window, cfg.force_first,
                          cfg.force_local)
    kc, vc = nsa.compress(inp["k"], inp["v"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"], [cfg.T], heads,
                          par)
    for _ in range(4):
        nsa.prefill(inp["q"], inp["k"], inp["v"], kc, vc, inp["gates"], inp["cu_seqlens"], heads, par)
    torch.cuda.synchronize()
    tiles = np.zeros((4, 12, 320, 4), np.uint64)
    ph = np.zeros((4, 12, 8), np.uint64)
    assert L.nsa_prefill_trace_read(tiles.ctypes.data_as(ctypes.c_void_p), ph.ctypes.data_as(ctypes.c_void_p)) == 0
    tiles, ph = tiles.astype(np.int64), ph.astype(np.int64)
    for c in range(4):
        t0 = ph[c, 0, 0]
        if t0 == 0:
            continue
        P = [int(ph[c, 0, k] - t0) for k in range(1, 6)]
        nt = cfg.T * cfg.H_q // cfg.H_kv // 128
        print(f"query tile {(c + 1) * (nt // 4) - 1}: phase ends (cycles) C1 {P[0]}  C2 {P[1]}  top-n {P[2]}  "
              f"W {P[3]}  S {P[4]}")
        rows = []
        for j in range(320):
            sr = [tiles[c, w, j, 0] for w in range(8) if tiles[c, w, j, 0]]
            dn = [tiles[c, w, j, 3] for w in range(8) if tiles[c, w, j, 3]]
            if not sr:
                break
            rows.append((j, min(sr) - t0, max(dn) - t0 if dn else -1, tiles[c, 9, j, 0] - t0 if tiles[c, 9, j, 0] else -1,
                         tiles[c, 10, j, 2] - t0 if tiles[c, 10, j, 2] else -1))
        for name, lo, hi in (("C1", 0, P[0]), ("C2", P[0], P[1]), ("W", P[2], P[3])):
            ph_t = [r for r in rows if lo <= r[1] < hi]
            if len(ph_t) > 2:
                print(f"  {name}: {len(ph_t)} tiles, period "
                      f"{(ph_t[-1][1] - ph_t[0][1]) / (len(ph_t) - 1):.0f} cycles/tile")
        s_tiles = [r for r in rows if r[1] >= P[3]]
        if len(s_tiles) > 2:
            per = (s_tiles[-1][1] - s_tiles[0][1]) / (len(s_tiles) - 1)
            lat = np.mean([r[2] - r[1] for r in s_tiles if r[2] > 0])
            print(f"  selected phase: {len(s_tiles)} tiles, period {per:.0f} cycles/tile, softmax latency "
                  f"{lat:.0f} cycles (S ready -> last warp done)")
        print("  tile: S ready | softmax done | S issued | P.V issued   (cycles from CTA start)")
        for r in rows[:: max(1, len(rows) // 12)]:
            print("  %4d: %7d | %7d | %7d | %7d" % r)


def _decode(nsa, L):
    import torch
    import nsa_workloads as W
    cfg = W.CONFIGS["decode_64k"]
    inp = W.make_decode_inputs(cfg, device="cuda")
    heads = nsa.Heads(cfg.H_q, cfg.H_kv, cfg.d_k, cfg.d_v)
    par = nsa.make_params(cfg.l_cmp, cfg.stride, cfg.l_sel, cfg.top_n, cfg.window, cfg.force_first,
                          cfg.force_local)
    kc, vc = nsa.compress_cache(inp["k_cache"], inp["v_cache"], inp["w_ck"], inp["pe_k"], inp["w_cv"], inp["pe_v"],
                                inp["cache_lens"], heads, par)
    lens = inp["cache_lens"].to("cuda")
    for _ in range(4):
        nsa.decode(inp["q"], inp["k_cache"], inp["v_cache"], kc, vc, lens, cfg.T, inp["gates"], heads, par)
    torch.cuda.synchronize()
    d = np.zeros((8, 16), np.uint64)
    assert L.nsa_decode_trace_read(d.ctypes.data_as(ctypes.c_void_p)) == 0
    names = ["partials copied", "chunks merged", "g_cmp*o_cmp", "importance", "top-n", "union", "stream",
             "combined"]
    print("fine pass, cycles from CTA start (KV head 0):")
    print("  seq  " + "  ".join(f"{n:>15s}" for n in names))
    for b, r in enumerate(d.astype(np.int64)):
        print(f"  {b:3d}  " + "  ".join(f"{int(x - r[0]):15d}" for x in r[1:9]))
    cs = np.zeros((256, 3), np.uint64)
    fs = np.zeros((512, 3), np.uint64)
    assert L.nsa_decode_cspan_read(cs.ctypes.data_as(ctypes.c_void_p)) == 0
    assert L.nsa_decode_fspan_read(fs.ctypes.data_as(ctypes.c_void_p)) == 0
    cs, fs = cs.astype(np.int64)[:148], fs.astype(np.int64)[:cfg.B * cfg.H_kv]
    t0 = cs[:, 0].min()
    print("compressed pass CTAs (us): start %.1f..%.1f, end %.1f..%.1f" % (
        (cs[:, 0].min() - t0) / 1e3, (cs[:, 0].max() - t0) / 1e3, (cs[:, 1].min() - t0) / 1e3,
        (cs[:, 1].max() - t0) / 1e3))
    print("fine pass CTAs (us):       start %.1f..%.1f, end %.1f..%.1f" % (
        (fs[:, 0].min() - t0) / 1e3, (fs[:, 0].max() - t0) / 1e3, (fs[:, 1].min() - t0) / 1e3,
        (fs[:, 1].max() - t0) / 1e3))


def main():
    what = sys.argv[1] if len(sys.argv) > 1 else "prefill"
    root = _b.ROOT
    if root not in sys.path:
        sys.path.insert(0, root)
    import sparse_attention_long_nsa_b200 as nsa
    nsa.LIB_PATH = build_trace_lib()
    L = nsa.lib()
    L.nsa_prefill_trace_read.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    L.nsa_decode_trace_read.argtypes = [ctypes.c_void_p]
    L.nsa_decode_cspan_read.argtypes = [ctypes.c_void_p]
    L.nsa_decode_fspan_read.argtypes = [ctypes.c_void_p]
    if what == "decode":
        _decode(nsa, L)
    else:
        _prefill(nsa, L, long=what == "prefill64k")


if __name__ == "__main__":
    main()
