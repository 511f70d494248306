"""Plain float64 CPU oracle for the DSA variant: lightning indexer + token-level
top-k + attention over the selected tokens.

TEST INFRASTRUCTURE ONLY (the same rule as nsa_oracle.py: only the tests, the
package's smoke check and the bench's CPU-baseline leg may import it). It shares
no code with the CUDA path.

Source: "Разреженное внимание — NSA и DSA" (ai.flicky.cc), section "DSA:
молниеносный индексатор": for query t a small attention model scores every past
token s as I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]) over H_I indexer heads
(each head compares its own query with the one shared key of token s; no
softmax; FP8); for each query the k = 2048 tokens with the largest I are kept and
ordinary attention runs over them only; one selection serves all heads. At 128K
the main attention reads 2048 / 131072 (about 1.6 %) of the keys. "web3.okx.com"
DSA-vs-NSA post: fused index-score + top-k.

Readings (the page leaves these open):
  D1 "past tokens" includes the query's own position: s <= t (causal, as in the
     NSA branches here).
  D2 ties of I go to the lower token index (the tie rule of the NSA selection);
     when t + 1 <= k every token 0..t is taken.
  D3 the main attention is the same GQA attention as the NSA branches (query head
     h uses KV head h / G, softmax scale 1/sqrt(d_k)) over the raw keys/values of
     the selected tokens; one selection per query token serves all heads.
  D4 the indexer's query, key and weights are inputs: q_I [T, H_I, d_I] and k_I
     [T, d_I] in FP8 (E4M3) as the page says, w [T, H_I] in fp32; the oracle
     computes exactly on those values in float64.
"""
from __future__ import annotations

import numpy as np

from . import nsa_oracle as O


def index_scores(qi_t, wi_t, ki):
    """I[s] = sum_j w_j * ReLU(q_j . k_s) for the keys ki [n, d_I]; qi_t [H_I, d_I],
    wi_t [H_I]. Returns [n]."""
    qi_t = np.asarray(qi_t, dtype=np.float64)
    wi_t = np.asarray(wi_t, dtype=np.float64)
    ki = np.asarray(ki, dtype=np.float64)
    if ki.shape[0] == 0:
        return np.zeros(0)
    dots = ki @ qi_t.T                        # [n, H_I]
    return np.maximum(dots, 0.0) @ wi_t       # [n]


def select_tokens(scores, t: int, top_k: int):
    """Tokens kept for query t (D1, D2): all of 0..t when t + 1 <= top_k, else the
    top_k largest scores among s <= t, ties to the lower index; ascending."""
    if t + 1 <= top_k:
        return list(range(t + 1))
    order = sorted(range(t + 1), key=lambda s: (-float(scores[s]), s))
    return sorted(order[:top_k])


def near_tie(scores, sel, t: int, rel: float = 1e-5) -> bool:
    """True when the smallest kept score and the largest dropped one are within
    `rel` (relative): more than one selection is then acceptable."""
    kept = set(sel)
    a = min(float(scores[s]) for s in sel)
    rest = [float(scores[s]) for s in range(t + 1) if s not in kept]
    if not rest:
        return False
    b = max(rest)
    return abs(a - b) <= rel * max(abs(a), abs(b), 1e-30)


def dsa_row(t, q_t, k, v, qi_t, wi_t, ki, top_k, scale, sel_override=None):
    """DSA output for query position t of one sequence: q_t [H_q, d_k], k [T, H_kv,
    d_k], v [T, H_kv, d_v] (rows <= t are read), qi_t [H_I, d_I], wi_t [H_I], ki
    [T, d_I]. Returns (out [H_q, d_v], sel, scores [t + 1])."""
    scores = index_scores(qi_t, wi_t, ki[:t + 1])
    sel = list(sel_override) if sel_override is not None else select_tokens(scores, t, top_k)
    H_q = q_t.shape[0]
    H_kv = k.shape[1]
    G = H_q // H_kv
    out = np.zeros((H_q, v.shape[2]))
    idx = np.asarray(sel, dtype=np.int64)
    for g in range(H_kv):
        out[g * G:(g + 1) * G], _ = O.attend(np.asarray(q_t[g * G:(g + 1) * G], dtype=np.float64),
                                             O._take(k, idx, g), O._take(v, idx, g), scale)
    return out, sel, scores


def prefill(q, k, v, qi, wi, ki, top_k, scale, rows=None, sel_override=None):
    """Causal DSA over one sequence: q [T, H_q, d_k], k, v [T, H_kv, *], qi [T, H_I,
    d_I], wi [T, H_I], ki [T, d_I]. `rows` restricts the query positions;
    `sel_override` maps t -> token list. Returns dict(out, sel {t: list},
    scores {t: array}, rows)."""
    T = q.shape[0]
    rows = list(range(T)) if rows is None else [int(r) for r in rows]
    ki = O._f64(ki)
    out = np.zeros((len(rows), q.shape[1], v.shape[2]))
    sel, sc = {}, {}
    for n, t in enumerate(rows):
        ov = sel_override.get(t) if sel_override is not None else None
        o, s_, i_ = dsa_row(t, O._f64(q[t]), k, v, O._f64(qi[t]), O._f64(wi[t]), ki, top_k, scale, ov)
        out[n] = o
        sel[t] = s_
        sc[t] = i_
    return dict(out=out, sel=sel, scores=sc, rows=rows)


def decode(q, k_cache, v_cache, qi, wi, ki_cache, lens, top_k, scale, batch_rows=None, sel_override=None):
    """DSA decode: one query per sequence at position len-1 (the cache holds the new
    token). q [B, H_q, d_k], caches [B, Lmax, ...], qi [B, H_I, d_I], wi [B, H_I],
    ki_cache [B, Lmax, d_I]."""
    lens = [int(x) for x in (lens.tolist() if hasattr(lens, "tolist") else lens)]
    batch_rows = list(range(len(lens))) if batch_rows is None else [int(b) for b in batch_rows]
    outs, sels, scs = [], {}, {}
    for b in batch_rows:
        L = lens[b]
        ov = sel_override.get(b) if sel_override is not None else None
        o, s_, i_ = dsa_row(L - 1, O._f64(q[b]), k_cache[b, :L], v_cache[b, :L], O._f64(qi[b]), O._f64(wi[b]),
                            O._f64(ki_cache[b, :L]), top_k, scale, ov)
        outs.append(o)
        sels[b] = s_
        scs[b] = i_
    return dict(out=np.stack(outs) if outs else np.zeros((0,)), sel=sels, scores=scs, rows=batch_rows)
