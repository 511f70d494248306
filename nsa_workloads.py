"""Seeded synthetic workloads for NSA (Native Sparse Attention) forward.

This module only draws random inputs and names the workload shapes. It holds none
of the method's arithmetic, so both the CUDA path (through the tests and the bench)
and the CPU oracle can be fed from it without sharing any computation.

Shapes and distributions follow the workloads the NSA pages describe: compression
block l=32 with stride 16, selection block l'=64, top-n blocks, sliding window w,
GQA-grouped heads ("Разреженное внимание — NSA и DSA", ai.flicky.cc, section
"NSA: три ветви"), and the small 1024-token case of the "Native Sparse Attention"
lesson (aiengineeringfromscratch.com, step 6, key-count printout).

Draw order (fixed so that any consumer reproduces the same tensors):
  prefill: q, k, v ~ N(0,1) (fp32 drawn, rounded to bf16); W_ck ~ N(0, 1/(l*d_k))
           (variance; std = 1/sqrt(l*d_k)); pe_k ~ N(0, 0.02) (std 0.02); then W_cv,
           pe_v the same way with d_v; gates = sigmoid(N(0,1)) of shape [T, H_q, 3].
  decode:  cache lengths first (varlen only: uniform integers in [lo, hi]); then q,
           the K cache, the V cache, W_ck, pe_k, W_cv, pe_v, gates, as above.
  DSA:     (decode: cache lengths first, as above) q, k, v as above, then the
           indexer's queries q_I [*, H_I, d_I] and keys k_I [*, d_I] ~ N(0,1)
           rounded to FP8 E4M3, and its weights w_I [*, H_I] ~ N(0,1) fp32
           ("Разреженное внимание — NSA и DSA", section "DSA: молниеносный
           индексатор": a few small heads, FP8, weights that depend on the query).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class NSAConfig:
    name: str
    kind: str                 # "prefill" or "decode"
    B: int
    T: int                    # prefill length, or the decode cache length (max for varlen)
    H_q: int
    H_kv: int
    d_k: int
    d_v: int
    l_cmp: int = 32
    stride: int = 16
    l_sel: int = 64
    top_n: int = 16
    window: int = 512
    force_first: int = 1
    force_local: int = 2
    len_lo: Optional[int] = None   # varlen decode: lengths ~ U[len_lo, len_hi]
    len_hi: Optional[int] = None
    seed: int = 1000

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv

    def params(self) -> dict:
        return dict(l_cmp=self.l_cmp, stride=self.stride, l_sel=self.l_sel,
                    top_n=self.top_n, window=self.window,
                    force_first=self.force_first, force_local=self.force_local,
                    scale=1.0 / math.sqrt(self.d_k))


CONFIGS = {
    # 1024-token GQA-4 prefill, d=64, n=4, w=128
    "prefill_tiny_1k": NSAConfig("prefill_tiny_1k", "prefill", 1, 1024, 4, 1, 64, 64,
                                 top_n=4, window=128, seed=1000),
    # 8K prefill, 64 query heads in 4 GQA groups of 16, d_k=192, d_v=128
    "prefill_8k": NSAConfig("prefill_8k", "prefill", 1, 8192, 64, 4, 192, 128, seed=1001),
    # 64K prefill, same heads
    "prefill_64k": NSAConfig("prefill_64k", "prefill", 1, 65536, 64, 4, 192, 128, seed=1002),
    # decode: 32 sequences, one query each, 64K cache
    "decode_64k": NSAConfig("decode_64k", "decode", 32, 65536, 64, 4, 192, 128, seed=1003),
    # varlen decode: 64 sequences, cache lengths ~ U[8192, 131072]
    "decode_varlen": NSAConfig("decode_varlen", "decode", 64, 131072, 64, 4, 192, 128,
                               len_lo=8192, len_hi=131072, seed=1004),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, g, device, std=1.0):
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * std


def make_weights(l: int, d_k: int, d_v: int, g, device):
    w_ck = _normal((l * d_k, d_k), g, device, 1.0 / math.sqrt(l * d_k))
    pe_k = _normal((l, d_k), g, device, 0.02)
    w_cv = _normal((l * d_v, d_v), g, device, 1.0 / math.sqrt(l * d_v))
    pe_v = _normal((l, d_v), g, device, 0.02)
    return w_ck, pe_k, w_cv, pe_v


def make_prefill_inputs(cfg: NSAConfig, device="cpu", seqlens=None, seed=None):
    """Packed varlen prefill inputs. `seqlens` defaults to [cfg.T] * cfg.B.

    Returns a dict of torch tensors: q [N,H_q,d_k], k [N,H_kv,d_k], v [N,H_kv,d_v]
    (bf16), w_ck, pe_k, w_cv, pe_v (fp32), gates [N,H_q,3] (fp32) and cu_seqlens
    (int32, host) where N = sum(seqlens).
    """
    seqlens = list(seqlens) if seqlens is not None else [cfg.T] * cfg.B
    N = int(sum(seqlens))
    g = _gen(cfg.seed if seed is None else seed, device)
    q = _normal((N, cfg.H_q, cfg.d_k), g, device).to(torch.bfloat16)
    k = _normal((N, cfg.H_kv, cfg.d_k), g, device).to(torch.bfloat16)
    v = _normal((N, cfg.H_kv, cfg.d_v), g, device).to(torch.bfloat16)
    w_ck, pe_k, w_cv, pe_v = make_weights(cfg.l_cmp, cfg.d_k, cfg.d_v, g, device)
    gates = torch.sigmoid(_normal((N, cfg.H_q, 3), g, device))
    cu = [0]
    for s in seqlens:
        cu.append(cu[-1] + int(s))
    return dict(q=q, k=k, v=v, w_ck=w_ck, pe_k=pe_k, w_cv=w_cv, pe_v=pe_v, gates=gates,
                cu_seqlens=torch.tensor(cu, dtype=torch.int32))


def make_decode_inputs(cfg: NSAConfig, device="cpu", seed=None, lens=None, Lmax=None):
    """Decode inputs: one new query per sequence, K/V caches [B, Lmax, H_kv, d].

    The caches already hold the new token, so the query sits at position len-1.
    Returns q [B,H_q,d_k], k_cache, v_cache (bf16), cache_lens (int32, host),
    the compression weights (fp32) and gates [B,H_q,3].
    """
    g = _gen(cfg.seed if seed is None else seed, device)
    if lens is None:
        if cfg.len_lo is not None:
            lens = torch.randint(cfg.len_lo, cfg.len_hi + 1, (cfg.B,), generator=g, device=device)
            lens = lens.to("cpu").to(torch.int32)
        else:
            lens = torch.full((cfg.B,), cfg.T, dtype=torch.int32)
    else:
        lens = torch.as_tensor(lens, dtype=torch.int32)
    B = int(lens.numel())
    if Lmax is None:
        Lmax = int(lens.max())
    q = _normal((B, cfg.H_q, cfg.d_k), g, device).to(torch.bfloat16)
    k_cache = _normal((B, Lmax, cfg.H_kv, cfg.d_k), g, device).to(torch.bfloat16)
    v_cache = _normal((B, Lmax, cfg.H_kv, cfg.d_v), g, device).to(torch.bfloat16)
    w_ck, pe_k, w_cv, pe_v = make_weights(cfg.l_cmp, cfg.d_k, cfg.d_v, g, device)
    gates = torch.sigmoid(_normal((B, cfg.H_q, 3), g, device))
    return dict(q=q, k_cache=k_cache, v_cache=v_cache, cache_lens=lens, w_ck=w_ck, pe_k=pe_k,
                w_cv=w_cv, pe_v=pe_v, gates=gates)


def small_config(name="small", T=256, H_q=4, H_kv=1, d_k=64, d_v=64, **kw) -> NSAConfig:
    """A small prefill configuration for tests (same method parameters as given)."""
    base = dict(kind="prefill", B=1, T=T, H_q=H_q, H_kv=H_kv, d_k=d_k, d_v=d_v)
    base.update(kw)
    return NSAConfig(name=name, **base)


@dataclasses.dataclass(frozen=True)
class DSAConfig:
    """A DSA workload (lightning indexer + token top-k + attention over the kept
    tokens). H_I, d_I: indexer heads and head size; top_k: tokens kept per query."""
    name: str
    kind: str
    B: int
    T: int
    H_q: int
    H_kv: int
    d_k: int
    d_v: int
    H_I: int = 8
    d_I: int = 128
    top_k: int = 2048
    len_lo: Optional[int] = None
    len_hi: Optional[int] = None
    seed: int = 2000

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d_k)


DSA_CONFIGS = {
    "dsa_prefill_tiny": DSAConfig("dsa_prefill_tiny", "prefill", 1, 1024, 4, 1, 64, 64, H_I=4, d_I=64, top_k=256,
                                  seed=2000),
    "dsa_prefill_8k": DSAConfig("dsa_prefill_8k", "prefill", 1, 8192, 64, 4, 192, 128, seed=2001),
    "dsa_decode_64k": DSAConfig("dsa_decode_64k", "decode", 32, 65536, 64, 4, 192, 128, seed=2002),
}


def _fp8(x):
    return x.to(torch.float8_e4m3fn)


def make_dsa_prefill_inputs(cfg: DSAConfig, device="cpu", seqlens=None, seed=None):
    """Packed DSA prefill inputs: q, k, v (bf16) as make_prefill_inputs, then qi
    [N, H_I, d_I] and ki [N, d_I] (FP8 E4M3), wi [N, H_I] (fp32), cu_seqlens (host)."""
    seqlens = list(seqlens) if seqlens is not None else [cfg.T] * cfg.B
    N = int(sum(seqlens))
    g = _gen(cfg.seed if seed is None else seed, device)
    q = _normal((N, cfg.H_q, cfg.d_k), g, device).to(torch.bfloat16)
    k = _normal((N, cfg.H_kv, cfg.d_k), g, device).to(torch.bfloat16)
    v = _normal((N, cfg.H_kv, cfg.d_v), g, device).to(torch.bfloat16)
    qi = _fp8(_normal((N, cfg.H_I, cfg.d_I), g, device))
    ki = _fp8(_normal((N, cfg.d_I), g, device))
    wi = _normal((N, cfg.H_I), g, device)
    cu = [0]
    for x in seqlens:
        cu.append(cu[-1] + int(x))
    return dict(q=q, k=k, v=v, qi=qi, ki=ki, wi=wi, cu_seqlens=torch.tensor(cu, dtype=torch.int32))


def make_dsa_decode_inputs(cfg: DSAConfig, device="cpu", seed=None, lens=None, Lmax=None):
    """DSA decode inputs: cache lengths (varlen draws first), q [B, H_q, d_k], the K/V
    caches [B, Lmax, H_kv, d] (bf16), qi [B, H_I, d_I] and the indexer key cache
    ki [B, Lmax, d_I] (FP8 E4M3), wi [B, H_I] (fp32)."""
    g = _gen(cfg.seed if seed is None else seed, device)
    if lens is None:
        if cfg.len_lo is not None:
            lens = torch.randint(cfg.len_lo, cfg.len_hi + 1, (cfg.B,), generator=g, device=device)
            lens = lens.to("cpu").to(torch.int32)
        else:
            lens = torch.full((cfg.B,), cfg.T, dtype=torch.int32)
    else:
        lens = torch.as_tensor(lens, dtype=torch.int32)
    B = int(lens.numel())
    if Lmax is None:
        Lmax = int(lens.max())
    q = _normal((B, cfg.H_q, cfg.d_k), g, device).to(torch.bfloat16)
    k_cache = _normal((B, Lmax, cfg.H_kv, cfg.d_k), g, device).to(torch.bfloat16)
    v_cache = _normal((B, Lmax, cfg.H_kv, cfg.d_v), g, device).to(torch.bfloat16)
    qi = _fp8(_normal((B, cfg.H_I, cfg.d_I), g, device))
    ki_cache = _fp8(_normal((B, Lmax, cfg.d_I), g, device))
    wi = _normal((B, cfg.H_I), g, device)
    return dict(q=q, k_cache=k_cache, v_cache=v_cache, qi=qi, ki_cache=ki_cache, wi=wi, cache_lens=lens)
