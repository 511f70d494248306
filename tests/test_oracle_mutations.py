"""Planted mistakes in the CPU oracle must be caught by the pins.

Each case patches one plausible error into the oracle (on the CPU, inside the
test only) and checks that at least one pin from test_oracle_pins fails. This is
evidence that the pins constrain every step of the oracle."""
import numpy as np
import pytest

from oracle import nsa_oracle as O
import tests.test_oracle_pins as P


def _fails(fn, *a):
    with pytest.raises(AssertionError):
        fn(*a)


def test_unit_weight_omega_is_caught(monkeypatch):
    orig = O.omega_matrix

    def unit(n_c, n_b, l, s, l_sel):
        return (orig(n_c, n_b, l, s, l_sel) > 0).astype(float)
    monkeypatch.setattr(O, "omega_matrix", unit)
    _fails(P.test_importance_mass_invariant)


def test_window_off_by_one_is_caught(monkeypatch):
    monkeypatch.setattr(O, "window_keys",
                        lambda t, w: np.arange(max(0, t - w), t + 1, dtype=np.int64))
    _fails(P.test_window_mask_matches_page_example)
    _fails(P.test_window_plus_sink_pair_fraction_matches_page)


def test_compressed_visibility_off_by_one_is_caught(monkeypatch):
    monkeypatch.setattr(O, "cmp_visible",
                        lambda t, l, s: (t - l) // s + 1 if t >= l else 0)
    _fails(P.test_counts_closed_form_grid)
    _fails(P.test_compute_budget_of_lesson)


def test_ties_to_higher_index_are_caught(monkeypatch):
    def bad_select(imp_row, t, l_sel, top_n, ff, fl):
        jt = t // l_sel
        if jt + 1 <= top_n:
            return list(range(jt + 1))
        forced = O.forced_blocks(t, l_sel, ff, fl)
        free = [j for j in range(jt + 1) if j not in forced]
        free.sort(key=lambda j: (-float(imp_row[j]), -j))
        return sorted(forced | set(free[:top_n - len(forced)]))
    monkeypatch.setattr(O, "select", bad_select)
    _fails(P.test_select_ties_go_to_lower_index)
    _fails(P.test_select_vs_enumeration, 0)


def test_missing_local_block_is_caught(monkeypatch):
    monkeypatch.setattr(O, "forced_blocks",
                        lambda t, ls, ff, fl: set(range(min(ff, t // ls + 1))) | {t // ls})
    _fails(P.test_structured_vs_brute, 8, 4, 16, 4, 20, 2, 2, 100)


def test_transposed_flatten_is_caught(monkeypatch):
    def bad_compress(x, W, pe, l, s):
        x = np.asarray(x, float)
        T, H, d = x.shape
        n = O.n_cmp(T, l, s)
        out = np.zeros((n, H, W.shape[1]))
        for i in range(n):
            blk = x[i * s:i * s + l] + pe[:, None, :]
            out[i] = blk.transpose(1, 2, 0).reshape(H, l * d) @ W   # e-major: wrong
        return out
    monkeypatch.setattr(O, "compress", bad_compress)
    _fails(P.test_compress_vs_explicit_sum, 32, 16)


def test_missing_softmax_scale_is_caught(monkeypatch):
    orig = O.attend
    monkeypatch.setattr(O, "attend", lambda qh, K, V, scale: orig(qh, K, V, 1.0))
    _fails(P.test_dense_reduction, "win")


def test_noncausal_current_block_is_caught(monkeypatch):
    def leaky(sel, t, l_sel):
        idx = []
        for j in sel:
            idx.extend(range(j * l_sel, (j + 1) * l_sel))
        return np.asarray(idx, dtype=np.int64)
    monkeypatch.setattr(O, "selected_keys", leaky)
    with pytest.raises(Exception):
        P.test_dense_reduction("slc")


def test_swapped_gate_order_is_caught(monkeypatch):
    orig = O.nsa_row

    def swapped(t, q_t, k, v, kc, vc, gates_t, p, sel_override=None):
        return orig(t, q_t, k, v, kc, vc, np.asarray(gates_t)[:, ::-1], p, sel_override)
    monkeypatch.setattr(O, "nsa_row", swapped)
    _fails(P.test_structured_vs_brute, 8, 4, 16, 4, 20, 2, 2, 100)
