"""Brute-force NSA formulation with dense boolean masks (tiny inputs only).

TEST INFRASTRUCTURE ONLY (see nsa_oracle.py header for who may use it).

This is a second, independent way to write the same definition, used to pin the
structured oracle in nsa_oracle.py. Every branch is expressed as a boolean mask
over (query, key) pairs followed by masked attention exactly as the practice
section of "Разреженное внимание — NSA и DSA" (ai.flicky.cc, section "Практика")
describes it: scores q.k / sqrt(d), -inf where the mask is False, softmax with
the row maximum subtracted, then weights times V. Importance is computed by
spreading each compressed token's probability evenly over the s-token slices of
its span and summing token mass per selection block; selection enumerates every
admissible subset. It shares nothing with nsa_oracle.py but numpy.
"""
from __future__ import annotations

import itertools

import numpy as np


def window_mask(T: int, w: int) -> np.ndarray:
    """mask[i, j] = key j visible to query i: j <= i and i - j < w."""
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    return (j <= i) & (i - j < w)


def cmp_mask(T: int, l: int, s: int) -> np.ndarray:
    """mask[t, c] = compressed token c (tokens c*s .. c*s+l-1) lies entirely at or
    before t. Only blocks fully inside the sequence exist."""
    n = (T - l) // s + 1 if T >= l else 0
    t = np.arange(T)[:, None]
    c = np.arange(n)[None, :]
    return (c * s + l - 1) <= t


def masked_attention(Q, K, V, mask, scale):
    """Q [T, d], K [n, d], V [n, dv], mask [T, n] -> [T, dv]; rows with no key -> 0."""
    S = (Q @ K.T) * scale
    S = np.where(mask, S, -np.inf)
    out = np.zeros((Q.shape[0], V.shape[1]))
    P = np.zeros_like(S)
    has = mask.any(axis=1)
    if has.any():
        Sm = S[has]
        Sm = Sm - Sm.max(axis=1, keepdims=True)
        E = np.exp(Sm)
        Pm = E / E.sum(axis=1, keepdims=True)
        P[has] = Pm
        out[has] = Pm @ V
    return out, P


def compress_brute(x, W, pe, l, s):
    """Explicit sum c[i, h, :] = sum_r sum_e (x[i*s+r, h, e] + pe[r, e]) W[r*d+e, :]."""
    T, H, d = x.shape
    n = (T - l) // s + 1 if T >= l else 0
    Wr = W.reshape(l, d, W.shape[1])
    out = np.zeros((n, H, W.shape[1]))
    for i in range(n):
        for h in range(H):
            acc = np.zeros(W.shape[1])
            for r in range(l):
                acc += (x[i * s + r, h] + pe[r]) @ Wr[r]
            out[i, h] = acc
    return out


def importance_brute(P_group_sum, T, l, s, l_sel):
    """P_group_sum [T, n_cmp] (probabilities summed over the group's heads) ->
    imp [T, n_blk]: compressed token c spreads p/s onto every token of its span;
    a block's importance is the total token mass inside it."""
    n = P_group_sum.shape[1]
    span = np.zeros((n, T))
    for c in range(n):
        span[c, c * s:c * s + l] = 1.0 / s
    nb = -(-T // l_sel)
    blk = np.zeros((T, nb))
    for tau in range(T):
        blk[tau, tau // l_sel] = 1.0
    return P_group_sum @ span @ blk


def select_brute(imp_row, t, l_sel, top_n, force_first, force_local):
    """Enumerate every admissible set: forced blocks plus a free subset of the
    remaining size; keep the largest total importance, ties to the
    lexicographically smallest ascending index list."""
    jt = t // l_sel
    cand = list(range(jt + 1))
    if len(cand) <= top_n:
        return cand
    forced = set(range(min(force_first, jt + 1))) | set(range(max(0, jt - force_local + 1), jt + 1))
    free = [j for j in cand if j not in forced]
    k = top_n - len(forced)
    best, best_key = None, None
    for comb in itertools.combinations(free, k):
        total = sum(float(imp_row[j]) for j in comb)
        chosen = sorted(forced | set(comb))
        key = (-total, chosen)
        if best_key is None or key < best_key:
            best, best_key = chosen, key
    return best


def selection_mask(sel_rows, T, l_sel):
    """sel_rows[t] = block list -> mask[t, tau]: tau in a chosen block and tau <= t."""
    m = np.zeros((T, T), dtype=bool)
    for t in range(T):
        for j in sel_rows[t]:
            lo, hi = j * l_sel, min((j + 1) * l_sel, t + 1)
            m[t, lo:hi] = True
    return m


def nsa_prefill_brute(q, k, v, kc, vc, gates, p):
    """Whole-sequence NSA prefill by masks. Returns (out [T,H_q,dv], sel, imp)."""
    l, s, ls = p["l_cmp"], p["stride"], p["l_sel"]
    T, H_q, _ = q.shape
    H_kv = k.shape[1]
    G = H_q // H_kv
    scale = p["scale"]
    cm = cmp_mask(T, l, s)
    wm = window_mask(T, p["window"])
    out = np.zeros((T, H_q, v.shape[2]))
    sel_all, imp_all = {}, {}
    for g in range(H_kv):
        Psum = np.zeros((T, kc.shape[0]))
        ocs, ows = [], []
        for hh in range(G):
            h = g * G + hh
            oc, Pc = masked_attention(q[:, h], kc[:, g], vc[:, g], cm, scale)
            Psum += Pc
            ow, _ = masked_attention(q[:, h], k[:, g], v[:, g], wm, scale)
            ocs.append(oc)
            ows.append(ow)
        imp = importance_brute(Psum, T, l, s, ls)
        sel_rows = [select_brute(imp[t], t, ls, p["top_n"], p["force_first"], p["force_local"])
                    for t in range(T)]
        sm = selection_mask(sel_rows, T, ls)
        for hh in range(G):
            h = g * G + hh
            osl, _ = masked_attention(q[:, h], k[:, g], v[:, g], sm, scale)
            out[:, h] = (gates[:, h, 0:1] * ocs[hh] + gates[:, h, 1:2] * osl
                         + gates[:, h, 2:3] * ows[hh])
        for t in range(T):
            sel_all[(t, g)] = sel_rows[t]
            imp_all[(t, g)] = imp[t, :t // ls + 1]
    return out, sel_all, imp_all


# ---------------------------------------------------------------------------
# DSA variant, dense formulation (tiny inputs only)
# ---------------------------------------------------------------------------

def dsa_brute(q, k, v, qi, wi, ki, top_k, scale):
    """Second formulation of the DSA variant (dsa_oracle.py): the full score
    matrix I = ReLU(einsum over indexer heads) weighted and summed, a causal mask,
    a rank matrix from a lexicographic sort (score descending, index ascending),
    the keep mask rank < top_k, then masked attention per head (-inf outside the
    mask, max-subtracted softmax). Returns (out [T, H_q, d_v], keep [T, T] bool)."""
    q, k, v, qi, wi, ki = (np.asarray(x, dtype=np.float64) for x in (q, k, v, qi, wi, ki))
    T, H_q, _ = q.shape
    H_kv = k.shape[1]
    G = H_q // H_kv
    dots = np.einsum("thd,sd->tsh", qi, ki)                 # [T, T, H_I]
    I = np.einsum("tsh,th->ts", np.maximum(dots, 0.0), wi)  # [T, T]
    causal = np.arange(T)[None, :] <= np.arange(T)[:, None]
    keep = np.zeros((T, T), dtype=bool)
    for t in range(T):
        cand = np.nonzero(causal[t])[0]
        order = np.lexsort((cand, -I[t, cand]))             # last key primary: score desc, then index
        keep[t, cand[order[:top_k]]] = True
    out = np.zeros((T, H_q, v.shape[2]))
    for h in range(H_q):
        g = h // G
        o, _ = masked_attention(q[:, h], k[:, g], v[:, g], keep, scale)
        out[:, h] = o
    return out, keep
