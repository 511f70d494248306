"""Plain float64 CPU oracle for the NSA backward pass (gradients of the forward
in nsa_oracle.py).

TEST INFRASTRUCTURE ONLY (the same rule as nsa_oracle.py: only the tests, the
package's smoke check and the bench's CPU-baseline leg may import it). It shares
no code with the CUDA path and imports only numpy and the forward oracle.

Source: "Native Sparse Attention" lesson (aiengineeringfromscratch.com), section
"why it is natively trainable": the top-n step is not differentiable and is a
no-op on the computation graph (it only decides which blocks are loaded);
gradients flow through the compressed branch (whose scores feed both its output
and the selection) and through the contributions of the selected blocks to the
output. "Разреженное внимание — NSA и DSA" (ai.flicky.cc), "Сколько это
экономит": the NSA kernels have forward and backward versions.

Reading B1: the backward differentiates the forward of nsa_oracle.py with the
selection held at the forward's choice (or a given one). The importance scores
and the selection receive no gradient; everything else does: the query, the raw
keys/values (through the selected and window branches and, through the
compression, the compressed branch), the compression weights W and position
embeddings pe of K and V, and the gates.

For a loss L with dL/dout = dout, per query t and head h of group g, branch b
with key set K_b(t), probabilities p and output o_b:
    dgate[t,h,b] = <dout[t,h], o_b[t,h]>
    dO_b        = gate[t,h,b] * dout[t,h]
    dV[j]      += p_j * dO_b                  (j in K_b(t))
    dp_j        = <dO_b, V[j]>
    dz_j        = p_j * (dp_j - <dO_b, o_b>)  (softmax backward)
    dq[t,h]    += scale * sum_j dz_j K[j]
    dK[j]      += scale * dz_j q[t,h]
and the compression c_i = vec(x[i*s : i*s+l] + pe) . W (token-major flattening)
sends dc_i back as dW += vec(x_blk + pe)^T dc_i, d vec(x_blk + pe) = dc_i W^T,
which lands on the block's tokens and on pe.
"""
from __future__ import annotations

import numpy as np

from . import nsa_oracle as O


def attend_backward(qh, K, V, o, p, dO, scale):
    """Backward of attend(): qh [H, d], K [n, d], V [n, dv], its outputs o [H, dv]
    and p [H, n], upstream dO [H, dv]. Returns (dq [H, d], dK [n, d], dV [n, dv])."""
    qh = np.asarray(qh, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros_like(qh), np.zeros_like(K), np.zeros_like(V)
    dV = p.T @ dO                                   # [n, dv]
    dp = dO @ V.T                                   # [H, n]
    D = np.sum(dO * o, axis=1, keepdims=True)       # [H, 1] = sum_j p_j dp_j
    dz = p * (dp - D)                               # [H, n]
    dq = scale * (dz @ K)
    dK = scale * (dz.T @ qh)
    return dq, dK, dV


def compress_backward(x, W, pe, dc, l: int, s: int):
    """Backward of nsa_oracle.compress(): x [T, H, d], W [l*d, d_out], pe [l, d],
    dc [n_cmp, H, d_out]. Returns (dx [T, H, d], dW [l*d, d_out], dpe [l, d])."""
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    pe = np.asarray(pe, dtype=np.float64)
    T, H, d = x.shape
    n = dc.shape[0]
    dx = np.zeros_like(x)
    dW = np.zeros_like(W)
    dpe = np.zeros_like(pe)
    for i in range(n):
        blk = x[i * s:i * s + l] + pe[:, None, :]           # [l, H, d]
        flat = blk.transpose(1, 0, 2).reshape(H, l * d)     # row r*d + e
        dW += flat.T @ dc[i]
        dflat = (dc[i] @ W.T).reshape(H, l, d).transpose(1, 0, 2)   # [l, H, d]
        dx[i * s:i * s + l] += dflat
        dpe += dflat.sum(axis=1)
    return dx, dW, dpe


def backward(q, k, v, w_ck, pe_k, w_cv, pe_v, gates, dout, p, sel=None, kc=None, vc=None):
    """Gradients of one causal NSA prefill sequence (Reading B1).

    q [T, H_q, d_k], k [T, H_kv, d_k], v [T, H_kv, d_v], compression weights as in
    nsa_oracle.prefill_full, gates [T, H_q, 3], dout [T, H_q, d_v]; `sel` maps
    (t, kv head) -> block list (default: the forward's own selection). `kc`, `vc`
    (optional) are the compressed keys/values the attention steps use (stage-wise
    checks feed the GPU's rounded ones, as the forward oracle takes them); the
    compression's own backward always follows its definition from x, W and pe.
    Returns a dict with out, sel and the gradients dq, dk, dv, dw_ck, dpe_k,
    dw_cv, dpe_v, dgates.
    """
    f = O._f64
    q, k, v, gates, dout = f(q), f(k), f(v), f(gates), f(dout)
    w_ck, pe_k, w_cv, pe_v = f(w_ck), f(pe_k), f(w_cv), f(pe_v)
    l, s, ls, scale = p["l_cmp"], p["stride"], p["l_sel"], p["scale"]
    T, H_q, d_k = q.shape
    H_kv, d_v = k.shape[1], v.shape[2]
    G = H_q // H_kv
    kc = O.compress(k, w_ck, pe_k, l, s) if kc is None else f(kc)
    vc = O.compress(v, w_cv, pe_v, l, s) if vc is None else f(vc)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dkc = np.zeros_like(kc)
    dvc = np.zeros_like(vc)
    dgates = np.zeros_like(gates)
    out = np.zeros((T, H_q, d_v))
    sel_used = {}
    for t in range(T):
        nvis = O.cmp_visible(t, l, s)
        for g in range(H_kv):
            hs = slice(g * G, (g + 1) * G)
            qg = q[t, hs]
            # compressed branch (its probabilities also give the selection, which is fixed)
            oc, pc = O.attend(qg, kc[:nvis, g], vc[:nvis, g], scale)
            if sel is not None and (t, g) in sel:
                chosen = list(sel[(t, g)])
            else:
                chosen = O.select(O.importance(pc, t, l, s, ls), t, ls, p["top_n"], p["force_first"],
                                  p["force_local"])
            sel_used[(t, g)] = chosen
            idx = O.selected_keys(chosen, t, ls)
            widx = O.window_keys(t, p["window"])
            os_, ps_ = O.attend(qg, k[idx, g], v[idx, g], scale)
            ow, pw = O.attend(qg, k[widx, g], v[widx, g], scale)
            gt = gates[t, hs]
            dO = dout[t, hs]
            out[t, hs] = gt[:, 0:1] * oc + gt[:, 1:2] * os_ + gt[:, 2:3] * ow
            dgates[t, hs, 0] = np.sum(dO * oc, axis=1)
            dgates[t, hs, 1] = np.sum(dO * os_, axis=1)
            dgates[t, hs, 2] = np.sum(dO * ow, axis=1)
            a, bK, bV = attend_backward(qg, kc[:nvis, g], vc[:nvis, g], oc, pc, gt[:, 0:1] * dO, scale)
            dq[t, hs] += a
            dkc[:nvis, g] += bK
            dvc[:nvis, g] += bV
            a, bK, bV = attend_backward(qg, k[idx, g], v[idx, g], os_, ps_, gt[:, 1:2] * dO, scale)
            dq[t, hs] += a
            np.add.at(dk[:, g], idx, bK)
            np.add.at(dv[:, g], idx, bV)
            a, bK, bV = attend_backward(qg, k[widx, g], v[widx, g], ow, pw, gt[:, 2:3] * dO, scale)
            dq[t, hs] += a
            np.add.at(dk[:, g], widx, bK)
            np.add.at(dv[:, g], widx, bV)
    dxk, dw_ck, dpe_k = compress_backward(k, w_ck, pe_k, dkc, l, s)
    dxv, dw_cv, dpe_v = compress_backward(v, w_cv, pe_v, dvc, l, s)
    dk += dxk
    dv += dxv
    return dict(out=out, sel=sel_used, dq=dq, dk=dk, dv=dv, dw_ck=dw_ck, dpe_k=dpe_k, dw_cv=dw_cv, dpe_v=dpe_v,
                dgates=dgates, dk_cmp=dkc, dv_cmp=dvc)


def loss_forward(q, k, v, w_ck, pe_k, w_cv, pe_v, gates, dout, p, sel):
    """<dout, out> of the forward with the selection fixed to `sel` (the scalar the
    gradients above belong to; used by the finite-difference pins)."""
    f = O._f64
    kc = O.compress(f(k), f(w_ck), f(pe_k), p["l_cmp"], p["stride"])
    vc = O.compress(f(v), f(w_cv), f(pe_v), p["l_cmp"], p["stride"])
    r = O.prefill(q, k, v, kc, vc, gates, p, sel_override=sel)
    return float(np.sum(np.asarray(dout, dtype=np.float64) * r["out"]))
