"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins of ``test_oracle_pins`` catch them.

Each case swaps one oracle function for a subtly wrong copy via ``monkeypatch`` and runs the pin that is meant to
guard it; the pin must fail.  Nothing here touches the CUDA path.
"""

from __future__ import annotations

import math

import numpy as np
import pytest

from oracle import lighthouse as O
from tests import test_oracle_pins as pins


def _attention_without_scale(qg, kg, vg):
    S, d = qg.shape
    logits = qg @ kg.T
    logits[np.triu_indices(S, 1)] = -np.inf
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    return (e / e.sum(axis=1, keepdims=True)) @ vg, (mx + np.log(e.sum(axis=1, keepdims=True)))[:, 0]


def _attention_mask_excludes_diagonal(qg, kg, vg):
    S, d = qg.shape
    logits = (qg @ kg.T) / math.sqrt(d)
    logits[np.triu_indices(S, 0)] = -np.inf
    logits[0, 0] = 0.0
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    return (e / e.sum(axis=1, keepdims=True)) @ vg, (mx + np.log(e.sum(axis=1, keepdims=True)))[:, 0]


def _scatter_offset_by_w(og, slots, P):
    out = np.zeros((P.N, og.shape[1]))
    t = np.arange(P.N)
    for lev in range(P.L):
        j = t // P.window(lev) - 1          # shift by w instead of w - 1
        ok = (j >= 0) & (j < P.level_size(lev))
        s = np.full(P.N, -1)
        s[ok] = slots[lev][j[ok]]
        ok &= s >= 0
        out[t[ok]] += og[s[ok]]
    return out


def _order_finer_first(sel, P):
    levs = np.concatenate([np.full(len(sel[lev]), lev) for lev in range(P.L)])
    js = np.concatenate(sel)
    ends = (js + 1) * (P.p ** levs) - 1
    order = np.lexsort((levs, ends))
    lev_g, j_g = levs[order], js[order]
    slots = [np.full(P.level_size(lev), -1) for lev in range(P.L)]
    for s, (lev, j) in enumerate(zip(lev_g, j_g)):
        slots[lev][j] = s
    return lev_g, j_g, slots


def _select_ties_to_higher_index(scores, P):
    sel = []
    for lev in range(P.L):
        n = P.level_size(lev)
        if lev == P.L - 1 or P.picks(lev) == n:
            sel.append(np.arange(n))
            continue
        n_c, m = n // P.C, P.picks(lev) // P.C
        parts = []
        for c in range(P.C):
            j = np.arange(c * n_c, (c + 1) * n_c)
            order = np.lexsort((-j, -scores[lev][j].astype(np.float64)))
            parts.append(np.sort(j[order[:m]]))
        sel.append(np.concatenate(parts))
    return sel


def _unpool_without_division(dxg, slots, P):
    dx = np.zeros((P.N, dxg.shape[1]))
    t = np.arange(P.N)
    for lev in range(P.L):
        s = slots[lev][t // P.window(lev)]
        ok = s >= 0
        dx[t[ok]] += dxg[s[ok]]
    return dx


def _pool_dropping_last_child(x, P):
    sums = [np.asarray(x, dtype=np.float64)]
    for lev in range(1, P.L):
        ch = sums[-1].reshape(P.level_size(lev), P.p, P.d)
        acc = ch[:, 0, :].copy()
        for c in range(1, P.p - 1):
            acc = acc + ch[:, c, :]
        sums.append(acc)
    return sums


def _scores_dropping_one_feature(kpyr, P):
    out = []
    for lev in range(P.L - 1):
        sq = kpyr[lev] * kpyr[lev]
        sq[:, -1] = 0
        out.append(O.fp32_round(sq.sum(axis=1)))
    return out


def _attention_backward_transposed_dk(qg, kg, vg, og, lse, dog):
    dq, dk, dv = O.__dict__["_orig_attn_bwd"](qg, kg, vg, og, lse, dog)
    return dq, dk[::-1].copy(), dv


CASES = [
    ("causal_attention", _attention_without_scale, lambda: pins.test_single_level_reduces_to_dense_causal_attention(7)),
    ("causal_attention", _attention_mask_excludes_diagonal,
     lambda: pins.test_single_level_reduces_to_dense_causal_attention(7)),
    ("scatter", _scatter_offset_by_w, lambda: pins.test_full_selection_equals_hand_built_pyramid_attention(2, 3)),
    ("gathered_order", _order_finer_first, lambda: pins.test_full_selection_equals_hand_built_pyramid_attention(2, 3)),
    ("select", _select_ties_to_higher_index, lambda: pins.test_select_matches_brute_force_sort_per_chunk(True)),
    ("unpool_backward", _unpool_without_division, pins.test_backward_matches_central_finite_differences),
    ("pool_sums", _pool_dropping_last_child, lambda: pins.test_pool_is_exact_block_mean_rounded_once(4, 3)),
    ("norm_scores", _scores_dropping_one_feature, lambda: pins.test_scores_are_exact_squared_norm_rounded_to_fp32(8)),
    ("causal_attention_backward", _attention_backward_transposed_dk,
     pins.test_backward_matches_central_finite_differences),
]


@pytest.mark.parametrize("name,bad,pin", CASES, ids=[f"{c[0]}-{c[1].__name__}" for c in CASES])
def test_pin_catches_planted_mistake(monkeypatch, name, bad, pin):
    monkeypatch.setitem(O.__dict__, "_orig_attn_bwd", O.causal_attention_backward)
    monkeypatch.setattr(O, name, bad)
    with pytest.raises(AssertionError):
        pin()


# ---- children-expansion variant ------------------------------------------------------------------------------

def _expand_select_children_shifted(scores, P):
    sel = _REAL_SELECT(scores, P)
    return [np.minimum(s + 1, P.level_size(lev) - 1) if lev < P.L - 1 else s for lev, s in enumerate(sel)]


def _expand_select_lowest_parents(scores, P):
    """Ranks the parents by ascending score (a dropped minus sign in the sort key)."""
    out = []
    for lev in range(P.L - 1):
        n_par = P.level_size(lev + 1)
        if P.parent_picks(lev + 1) == n_par:
            out.append(np.arange(P.level_size(lev)))
            continue
        J = O.chunked_top(-np.asarray(scores[lev], dtype=np.float64), P.parent_picks(lev + 1), P)
        out.append((J[:, None] * P.p + np.arange(P.p)[None, :]).reshape(-1))
    out.append(np.arange(P.level_size(P.L - 1)))
    return out


_REAL_SELECT = O.select


@pytest.mark.parametrize("mutant", [_expand_select_children_shifted, _expand_select_lowest_parents])
def test_expand_pins_catch_selection_mutants(monkeypatch, mutant):
    def patched(scores, P):
        return mutant(scores, P) if P.expand else _REAL_SELECT(scores, P)

    monkeypatch.setattr(O, "select", patched)
    failed = 0
    for fn, args in ((pins.test_expand_selection_is_the_children_of_the_per_level_selection_one_level_up,
                      (3, 4, 8, 2)),
                     (pins.test_expand_selection_comes_in_sibling_groups_with_equal_counts_per_chunk, ())):
        try:
            fn(*args)
        except AssertionError:
            failed += 1
    assert failed >= 1
