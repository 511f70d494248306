"""Plain float64 CPU oracle for the NSA (Native Sparse Attention) forward pass.

TEST INFRASTRUCTURE ONLY. This module is the reference the kernels are checked
against, not the product: only the tests, the package's smoke check and the
bench's CPU-baseline leg may import it.
It shares no code with the CUDA path (no kernels, headers, helpers or tables) and
imports nothing from it.

Sources (web pages describing the method; cited by title and section):
  [NSA-lesson] "मूल स्पारस ध्यान (डीपसेक एनएसए)" / Native Sparse Attention lesson,
      aiengineeringfromscratch.com, Phase 10 lesson 17: sections "Concept / three
      parallel branches" (compressed, selected, sliding-window branches, gated sum
      out = g_cmp*out_cmp + g_sel*out_sel + g_win*out_win, gates need not sum to 1),
      "Compute budget" (keys per query N/l + k*b + w), "Build it" steps 1-6.
  [NSA-ru] "Разреженное внимание — NSA и DSA", ai.flicky.cc stage 5.5 lesson 02:
      section "NSA: три ветви" (equation for o_t as a gated sum of three attentions,
      gates in [0,1] from a sigmoid; compression blocks l=32 with stride d=16 giving
      about t/16 summaries; selection blocks l'=64 scored from the compressed-branch
      weights, top n=16 with the initial block and two local blocks always taken;
      all heads of a GQA group pick the same blocks; window w=512), section
      "Практика" (mask rule j <= i and i - j < w; masked attention with -inf,
      row-max-subtracted softmax and scale 1/sqrt(d)).

Readings where the pages leave a step open (each restated where it is used):
  R1 compressor: one linear map W [l*d, d_out] of the flattened block plus a learned
     intra-block position embedding pe [l, d] added to each token before flattening;
     flatten order is token-major (row r*d + e).
  R2 only full blocks are compressed: block i covers tokens [i*s, i*s + l), i*s+l <= T.
  R3 query t sees compressed token i iff its whole block lies at or before t.
  R4 an empty compressed set gives o_cmp = 0 and zero importance.
  R5 importance of selection block j = sum over the group's heads and visible
     compressed tokens of p * |span_i ∩ block_j| / s (overlap weighting).
  R6 "two local blocks" = the block holding t and its predecessor; forced blocks
     count toward n; when all candidate blocks fit in n, all are taken; remaining
     slots go to the highest importance, ties to the lower block index.
  R7 inside the selected blocks keys after t are masked (causal).
  R8 window = the w keys ending at t (fewer near the start).
  R9 each branch is its own softmax; the three are not de-duplicated.
  R10 scale 1/sqrt(d_k) in all three branches; gates are given per (token, head,
     branch) in the order (cmp, slc, win).
  R11 decode: the cache already holds the new token, whose position is L-1.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# counts (NSA-ru "NSA: три ветви"; NSA-lesson "Compute budget")
# ---------------------------------------------------------------------------


def n_cmp(T: int, l: int, s: int) -> int:
    """Number of compressed tokens of a length-T sequence (R2: full blocks only)."""
    return (T - l) // s + 1 if T >= l else 0


def n_blk(T: int, l_sel: int) -> int:
    """Number of selection blocks covering T tokens."""
    return -(-T // l_sel)


def cmp_visible(t: int, l: int, s: int) -> int:
    """How many compressed tokens query t may attend to (R3): i*s + l - 1 <= t."""
    return (t - l + 1) // s + 1 if t >= l - 1 else 0


# ---------------------------------------------------------------------------
# step 1: block compression (NSA-ru "Сжатая ветвь"; R1, R2)
# ---------------------------------------------------------------------------


def compress(x, W, pe, l: int, s: int) -> np.ndarray:
    """Compress x [T, H, d] into [n_cmp, H, d_out].

    Each block of l consecutive tokens starting at i*s gets the position
    embedding pe[r] added to its r-th token, is flattened token-major and mapped
    by W [l*d, d_out]. The blocks are independent; they are evaluated a chunk of
    blocks at a time (the same formula per block, gathered by token index).
    """
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    pe = np.asarray(pe, dtype=np.float64)
    T, H, d = x.shape
    n = n_cmp(T, l, s)
    out = np.zeros((n, H, W.shape[1]))
    chunk = 256
    for i0 in range(0, n, chunk):
        i = np.arange(i0, min(n, i0 + chunk))
        tok = i[:, None] * s + np.arange(l)[None, :]          # [c, l] token of row r of block i
        blk = x[tok] + pe[None, :, None, :]                    # [c, l, H, d]
        flat = blk.transpose(0, 2, 1, 3).reshape(len(i), H, l * d)   # row r*d + e
        out[i0:i0 + len(i)] = flat @ W
    return out


# ---------------------------------------------------------------------------
# attention over an index set (NSA-ru "Практика": scale 1/sqrt(d), max-subtract)
# ---------------------------------------------------------------------------


def attend(qh, K, V, scale: float):
    """Softmax attention of query rows qh [H, d] over keys K [n, d], values V [n, dv].

    Returns (o [H, dv], p [H, n]). With n == 0 the output is zero (R4).
    """
    qh = np.asarray(qh, dtype=np.float64)
    H = qh.shape[0]
    if K.shape[0] == 0:
        return np.zeros((H, V.shape[1])), np.zeros((H, 0))
    z = scale * (qh @ np.asarray(K, dtype=np.float64).T)
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    p = e / e.sum(axis=1, keepdims=True)
    return p @ np.asarray(V, dtype=np.float64), p


# ---------------------------------------------------------------------------
# step 3: importance of selection blocks (NSA-ru "Ветвь отбора"; R5)
# ---------------------------------------------------------------------------


def omega(i: int, j: int, l: int, s: int, l_sel: int) -> float:
    """Weight of compressed token i in selection block j: overlap of the token
    span [i*s, i*s+l) with the block span [j*l', (j+1)*l'), divided by s."""
    lo = max(i * s, j * l_sel)
    hi = min(i * s + l, (j + 1) * l_sel)
    return max(0, hi - lo) / s


_OMEGA_CACHE: dict = {}


def omega_matrix(n_c: int, n_b: int, l: int, s: int, l_sel: int) -> np.ndarray:
    """[n_c, n_b] matrix of omega(i, j), the same overlap formula evaluated on
    index grids (cached per (l, s, l') and grown on demand)."""
    key = (l, s, l_sel)
    Om = _OMEGA_CACHE.get(key)
    if Om is None or Om.shape[0] < n_c or Om.shape[1] < n_b:
        nc2 = max(n_c, 0 if Om is None else Om.shape[0])
        nb2 = max(n_b, 0 if Om is None else Om.shape[1])
        i = np.arange(nc2)[:, None]
        j = np.arange(nb2)[None, :]
        lo = np.maximum(i * s, j * l_sel)
        hi = np.minimum(i * s + l, (j + 1) * l_sel)
        Om = np.maximum(0, hi - lo) / s
        _OMEGA_CACHE[key] = Om
    return Om[:n_c, :n_b]


def importance(p_group, t: int, l: int, s: int, l_sel: int) -> np.ndarray:
    """Block importance for query t from the compressed probabilities of the
    group's heads p_group [G, n_visible]; returns [j_t + 1] (R5, heads summed)."""
    jt = t // l_sel
    n_c = p_group.shape[1]
    if n_c == 0:
        return np.zeros(jt + 1)
    return p_group.sum(axis=0) @ omega_matrix(n_c, jt + 1, l, s, l_sel)


# ---------------------------------------------------------------------------
# step 4: top-n selection (NSA-lesson step 3; NSA-ru "Ветвь отбора"; R6)
# ---------------------------------------------------------------------------


def forced_blocks(t: int, l_sel: int, force_first: int, force_local: int) -> set:
    jt = t // l_sel
    f = set(range(min(force_first, jt + 1)))
    f |= set(range(max(0, jt - force_local + 1), jt + 1))
    return f


def select(imp_row, t: int, l_sel: int, top_n: int, force_first: int, force_local: int):
    """Selected block indices for query t, ascending (R6)."""
    jt = t // l_sel
    if jt + 1 <= top_n:
        return list(range(jt + 1))
    forced = forced_blocks(t, l_sel, force_first, force_local)
    free = [j for j in range(jt + 1) if j not in forced]
    free.sort(key=lambda j: (-float(imp_row[j]), j))
    chosen = forced | set(free[:top_n - len(forced)])
    return sorted(chosen)


def near_tie(imp_row, sel, t: int, l_sel: int, force_first: int, force_local: int,
             rel: float = 1e-5) -> bool:
    """True when the last chosen free score and the first unchosen one are within
    `rel` (relative): more than one selection is then acceptable."""
    jt = t // l_sel
    forced = forced_blocks(t, l_sel, force_first, force_local)
    chosen_free = [float(imp_row[j]) for j in sel if j not in forced]
    rest = [float(imp_row[j]) for j in range(jt + 1) if j not in forced and j not in sel]
    if not chosen_free or not rest:
        return False
    a, b = min(chosen_free), max(rest)
    return abs(a - b) <= rel * max(abs(a), abs(b), 1e-30)


# ---------------------------------------------------------------------------
# steps 5-6: selected-block and window key sets (R7, R8)
# ---------------------------------------------------------------------------


def selected_keys(sel, t: int, l_sel: int) -> np.ndarray:
    idx = []
    for j in sel:
        idx.extend(range(j * l_sel, min((j + 1) * l_sel, t + 1)))
    return np.asarray(idx, dtype=np.int64)


def window_keys(t: int, w: int) -> np.ndarray:
    return np.arange(max(0, t - w + 1), t + 1, dtype=np.int64)


# ---------------------------------------------------------------------------
# one query position: all branches and the gated sum
# ---------------------------------------------------------------------------


def nsa_row(t, q_t, k, v, kc, vc, gates_t, p, sel_override=None):
    """NSA output for query position t of one sequence.

    q_t [H_q, d_k]; k [T, H_kv, d_k], v [T, H_kv, d_v] (raw keys/values, only
    positions <= t are read); kc, vc [n_cmp, H_kv, *] compressed keys/values;
    gates_t [H_q, 3]; p a dict with l_cmp, stride, l_sel, top_n, window,
    force_first, force_local, scale. `sel_override` maps kv-head -> block list to
    use instead of the oracle's own choice.

    Returns (out [H_q, d_v], sel list per kv-head, imp list per kv-head,
    branch outputs (o_cmp, o_slc, o_win) each [H_q, d_v]).
    """
    l, s, ls = p["l_cmp"], p["stride"], p["l_sel"]
    scale = p["scale"]
    H_q = q_t.shape[0]
    H_kv = k.shape[1]
    G = H_q // H_kv
    d_v = v.shape[2]
    nvis = cmp_visible(t, l, s)
    o_cmp = np.zeros((H_q, d_v))
    o_slc = np.zeros((H_q, d_v))
    o_win = np.zeros((H_q, d_v))
    sels, imps = [], []
    for g in range(H_kv):
        qg = np.asarray(q_t[g * G:(g + 1) * G], dtype=np.float64)
        oc, pc = attend(qg, kc[:nvis, g], vc[:nvis, g], scale)
        o_cmp[g * G:(g + 1) * G] = oc
        imp = importance(pc, t, l, s, ls)
        if sel_override is not None and g in sel_override:
            sel = list(sel_override[g])
        else:
            sel = select(imp, t, ls, p["top_n"], p["force_first"], p["force_local"])
        idx = selected_keys(sel, t, ls)
        o_slc[g * G:(g + 1) * G], _ = attend(qg, _take(k, idx, g), _take(v, idx, g), scale)
        widx = window_keys(t, p["window"])
        o_win[g * G:(g + 1) * G], _ = attend(qg, _take(k, widx, g), _take(v, widx, g), scale)
        sels.append(sel)
        imps.append(imp)
    gt = np.asarray(gates_t, dtype=np.float64)
    out = gt[:, 0:1] * o_cmp + gt[:, 1:2] * o_slc + gt[:, 2:3] * o_win
    return out, sels, imps, (o_cmp, o_slc, o_win)


def _f64(x):
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def _take(x, idx, g):
    """Rows idx of head g of x [T, H, d] as float64 (x a numpy array, or a torch
    tensor of which only these rows are converted)."""
    if hasattr(x, "detach"):
        import torch
        return _f64(x[torch.as_tensor(idx, dtype=torch.long, device=x.device), g])
    return np.asarray(x[idx, g], dtype=np.float64)


def prefill(q, k, v, kc, vc, gates, p, rows=None, sel_override=None):
    """Causal NSA prefill of ONE sequence with given compressed keys/values.

    q [T, H_q, d_k], k/v [T, H_kv, *], kc/vc [n_cmp, H_kv, *], gates [T, H_q, 3].
    `rows` restricts the query positions computed (default: all).
    `sel_override` maps (t, kv-head) -> block list.
    Returns dict(out [len(rows), H_q, d_v], sel {(t,g): list}, imp {(t,g): array},
    rows).
    """
    # q and gates are read row by row (only the requested rows are converted)
    k, v, kc, vc = (_f64(a) for a in (k, v, kc, vc))
    T = q.shape[0]
    rows = list(range(T)) if rows is None else [int(r) for r in rows]
    out = np.zeros((len(rows), q.shape[1], v.shape[2]))
    sel, imp = {}, {}
    for n, t in enumerate(rows):
        ov = None
        if sel_override is not None:
            ov = {g: sel_override[(t, g)] for g in range(k.shape[1]) if (t, g) in sel_override}
        o, sels, imps, _ = nsa_row(t, _f64(q[t]), k, v, kc, vc, _f64(gates[t]), p, ov)
        out[n] = o
        for g in range(k.shape[1]):
            sel[(t, g)] = sels[g]
            imp[(t, g)] = imps[g]
    return dict(out=out, sel=sel, imp=imp, rows=rows)


def prefill_full(q, k, v, w_ck, pe_k, w_cv, pe_v, gates, p, rows=None):
    """Prefill of one sequence including the oracle's own fp64 compression."""
    kc = compress(_f64(k), _f64(w_ck), _f64(pe_k), p["l_cmp"], p["stride"])
    vc = compress(_f64(v), _f64(w_cv), _f64(pe_v), p["l_cmp"], p["stride"])
    r = prefill(q, k, v, kc, vc, gates, p, rows=rows)
    r["k_cmp"], r["v_cmp"] = kc, vc
    return r


def decode(q, k_cache, v_cache, kc_cache, vc_cache, lens, gates, p, batch_rows=None,
           sel_override=None):
    """NSA decode: one query per sequence at position len-1 (R11).

    q [B, H_q, d_k]; k_cache/v_cache [B, Lmax, H_kv, *]; kc_cache/vc_cache
    [B, Lmax_cmp, H_kv, *] (only the first n_cmp(len) entries are used);
    lens [B]; gates [B, H_q, 3]. `batch_rows` restricts the sequences computed.
    """
    lens = [int(x) for x in (lens.tolist() if hasattr(lens, "tolist") else lens)]
    B = len(lens)
    batch_rows = list(range(B)) if batch_rows is None else [int(b) for b in batch_rows]
    outs, sels, imps = [], {}, {}
    for b in batch_rows:
        L = lens[b]
        t = L - 1
        nc = n_cmp(L, p["l_cmp"], p["stride"])
        # raw keys/values stay in their own dtype; nsa_row converts the rows it reads
        kb, vb = k_cache[b, :L], v_cache[b, :L]
        kcb, vcb = _f64(kc_cache[b, :nc]), _f64(vc_cache[b, :nc])
        ov = None
        if sel_override is not None:
            ov = {g: sel_override[(b, g)] for g in range(kb.shape[1]) if (b, g) in sel_override}
        o, s_, i_, _ = nsa_row(t, _f64(q[b]), kb, vb, kcb, vcb, _f64(gates[b]), p, ov)
        outs.append(o)
        for g in range(kb.shape[1]):
            sels[(b, g)] = s_[g]
            imps[(b, g)] = i_[g]
    return dict(out=np.stack(outs) if outs else np.zeros((0,)), sel=sels, imp=imps,
                rows=batch_rows)
