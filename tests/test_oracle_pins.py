"""Pins of the CPU oracle against references other than itself (no GPU needed).

Each test checks one oracle function against exact rational arithmetic, a textbook loop, brute force, a closed
form or finite differences.  ``test_oracle_mutations.py`` plants plausible mistakes in the oracle and checks that
these pins catch them.
"""

from __future__ import annotations

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import lighthouse as O
from tests import _exact as X

HERE = os.path.dirname(os.path.abspath(__file__))


def rand_bf16(rng, shape, scale=1.0):
    """Random bf16 values (float64) with lognormal row scaling, exact in fp64."""
    z = rng.standard_normal(shape) * np.exp(0.5 * rng.standard_normal(shape[:-1] + (1,))) * scale
    return O.bf16_round(z)


# ----------------------------------------------------------------------------------------------------------------
# Rounding helpers
# ----------------------------------------------------------------------------------------------------------------

def test_bf16_round_matches_exact_nearest_even():
    rng = np.random.default_rng(1)
    xs = list(rng.standard_normal(2000) * np.exp(rng.uniform(-30, 30, 2000)))
    # exact midpoints between neighbouring bf16 values (ties), both parities
    for b in [0x3F80, 0x3F81, 0x0001, 0x0002, 0x007F, 0x0080, 0x7F7E, 0x4000, 0x1234, 0x8F01]:
        lo, hi = X.bf16_value_of_bits(b), X.bf16_value_of_bits(b + 1)
        xs += [(lo + hi) / 2, -(lo + hi) / 2, np.nextafter((lo + hi) / 2, 0), np.nextafter((lo + hi) / 2, 10)]
    # subnormal range and overflow edge
    xs += [2.0 ** -140, 3 * 2.0 ** -134, 2.0 ** -133 * 0.5, 3.3e38, 3.39e38, 3.4e38, -3.395e38, 1e-45]
    got = O.bf16_round(np.array(xs))
    for x, g in zip(xs, got):
        want = X.to_bf16_exact(x)
        assert g == want or (math.isinf(want) and g == want), (x, g, want)


def test_bf16_bits_roundtrip_all_patterns():
    bits = np.array([b for b in range(1 << 16) if (b & 0x7F80) != 0x7F80], dtype=np.uint16)  # skip inf/nan
    vals = O.bf16_from_bits(bits)
    for b in [0, 1, 0x3F80, 0x8001, 0x7F7F, 0x4049]:
        assert vals[np.searchsorted(bits, b)] == X.bf16_value_of_bits(b)
    assert np.array_equal(O.bf16_bits(vals), bits)
    assert np.array_equal(O.bf16_round(vals), vals)


# ----------------------------------------------------------------------------------------------------------------
# Pool
# ----------------------------------------------------------------------------------------------------------------

def test_pool_constant_input_reproduces_itself():
    P = O.Params(1, 1, 64, 8, 4, 4, 4, 1)
    x = np.full((64, 8), X.bf16_value_of_bits(0x3FA0))
    for lev, level in enumerate(O.pyramid(x, P)):
        assert level.shape == (P.level_size(lev), 8)
        assert np.all(level == x[0, 0])


@pytest.mark.parametrize("p,L", [(2, 4), (4, 3), (3, 3)])
def test_pool_is_exact_block_mean_rounded_once(p, L):
    rng = np.random.default_rng(p * 10 + L)
    N, d = p ** (L - 1) * 3, 8
    P = O.Params(1, 1, N, d, L, p, 1, 1)
    x = rand_bf16(rng, (N, d))
    pyr = O.pyramid(x, P)
    for lev in range(1, L):
        w = p ** lev
        for j in range(N // w):
            for i in range(d):
                mean = sum(Fraction(float(x[t, i])) for t in range(j * w, (j + 1) * w)) / w
                assert pyr[lev][j, i] == X.to_bf16_exact(mean), (lev, j, i)


def test_pool_negative_zero_block_stays_negative_zero():
    P = O.Params(1, 1, 16, 8, 3, 4, 1, 1)
    x = np.full((16, 8), -0.0)
    for level in O.pyramid(x, P)[1:]:
        assert np.all(np.signbit(level))


# ----------------------------------------------------------------------------------------------------------------
# Score
# ----------------------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("d", [8, 16, 64])
def test_scores_are_exact_squared_norm_rounded_to_fp32(d):
    rng = np.random.default_rng(d)
    P = O.Params(1, 1, 64, d, 3, 4, 4, 1)
    k = rand_bf16(rng, (64, d))
    kp = O.pyramid(k, P)
    sc = O.norm_scores(kp, P)
    assert len(sc) == P.L - 1 and all(s.dtype == np.float32 for s in sc)
    for lev in range(P.L - 1):
        for j in range(P.level_size(lev)):
            exact = sum(Fraction(float(v)) ** 2 for v in kp[lev][j])
            assert float(sc[lev][j]) == X.to_fp32_exact(exact), (lev, j)


# ----------------------------------------------------------------------------------------------------------------
# Top-K
# ----------------------------------------------------------------------------------------------------------------

def brute_select(scores, P):
    out = []
    for lev in range(P.L):
        n = P.level_size(lev)
        if lev == P.L - 1 or min(P.k, n) == n:
            out.append(list(range(n)))
            continue
        n_c, m = n // P.C, min(P.k, n) // P.C
        chosen = []
        for c in range(P.C):
            js = range(c * n_c, (c + 1) * n_c)
            chosen += sorted(sorted(js, key=lambda j: (-float(scores[lev][j]), j))[:m])
        out.append(chosen)
    return out


@pytest.mark.parametrize("ties", [False, True])
def test_select_matches_brute_force_sort_per_chunk(ties):
    rng = np.random.default_rng(7)
    P = O.Params(1, 1, 256, 8, 4, 2, 16, 4)
    scores = []
    for lev in range(P.L - 1):
        n = P.level_size(lev)
        s = rng.integers(0, 3, n) if ties else rng.random(n)
        scores.append(np.asarray(s, dtype=np.float32))
    sel = O.select(scores, P)
    want = brute_select(scores, P)
    for lev in range(P.L):
        assert sel[lev].tolist() == want[lev]
        n = P.level_size(lev)
        if lev < P.L - 1:
            n_c, m = n // P.C, P.picks(lev) // P.C
            counts = np.bincount(sel[lev] // n_c, minlength=P.C)
            assert np.all(counts == m)
    assert sel[P.L - 1].tolist() == list(range(P.level_size(P.L - 1)))  # coarsest level kept whole


def test_select_all_equal_scores_takes_lowest_indices():
    P = O.Params(1, 1, 64, 8, 2, 4, 8, 2)
    sel = O.select([np.ones(64, dtype=np.float32)], P)
    assert sel[0].tolist() == [0, 1, 2, 3, 32, 33, 34, 35]


def test_select_k_at_least_level_size_takes_whole_level():
    P = O.Params(1, 1, 64, 8, 3, 4, 16, 4)      # level 1 has 16 entries = k
    rng = np.random.default_rng(3)
    sel = O.select([rng.random(64).astype(np.float32), rng.random(16).astype(np.float32)], P)
    assert sel[1].tolist() == list(range(16))
    assert len(sel[0]) == 16


# ----------------------------------------------------------------------------------------------------------------
# Ordering, slots, S
# ----------------------------------------------------------------------------------------------------------------

def test_order_is_sorted_by_end_then_coarser_and_slots_invert_it():
    rng = np.random.default_rng(11)
    P = O.Params(1, 1, 128, 8, 4, 2, 8, 2)
    scores = [rng.random(P.level_size(lev)).astype(np.float32) for lev in range(P.L - 1)]
    sel = O.select(scores, P)
    lev_g, j_g, slots = O.gathered_order(sel, P)
    assert len(lev_g) == P.gathered_length() == sum(len(s) for s in sel)
    keys = [((int(j) + 1) * P.p ** int(lev) - 1, -int(lev)) for lev, j in zip(lev_g, j_g)]
    assert all(a < b for a, b in zip(keys, keys[1:]))
    for s, (lev, j) in enumerate(zip(lev_g, j_g)):
        assert slots[lev][j] == s
    for lev in range(P.L):
        chosen = set(sel[lev].tolist())
        assert all((slots[lev][j] >= 0) == (j in chosen) for j in range(P.level_size(lev)))
    ids = O.global_ids(lev_g, j_g, P)
    assert np.array_equal(O.slot_map(slots)[ids], np.arange(len(ids)))


@pytest.mark.parametrize("cfg,S", [
    ((1, 2, 4096, 64, 3, 4, 256, 8), 768),
    ((1, 16, 32768, 64, 4, 4, 2048, 16), 6656),
    ((1, 16, 98304, 64, 4, 4, 2048, 16), 7680),
    ((1, 16, 524288, 128, 4, 4, 4096, 32), 20480),
    ((1, 8, 1048576, 128, 4, 4, 4096, 32), 28672),
])
def test_gathered_length_formula(cfg, S):
    P = O.Params(*cfg)
    P.validate()
    assert P.gathered_length() == S
    # the formula counts what the selection actually returns (level sizes only; no data needed)
    assert sum(P.picks(lev) for lev in range(P.L)) == S


def test_pages_size_example_is_not_reproduced_by_the_per_level_reading():
    g = json.load(open(os.path.join(HERE, "golden", "pages_size_example.json")))
    N, L, p, k = g["N"], g["L"], g["p"], g["k"]
    P = O.Params(1, 1, N, 8, L, p, k, 1)
    ours = P.gathered_length()
    children_variant = N // p ** (L - 1) + (L - 1) * p * k
    assert ours == 27913
    assert abs(children_variant - g["gathered_about"]) < 0.01 * g["gathered_about"]
    assert abs(ours - g["gathered_about"]) > 0.5 * g["gathered_about"]


# ----------------------------------------------------------------------------------------------------------------
# The children-expansion variant ([E] "Какво точно промени Nous Research в attention пътя?": the size example)
# ----------------------------------------------------------------------------------------------------------------

def test_expand_gathered_length_reproduces_the_pages_size_example():
    g = json.load(open(os.path.join(HERE, "golden", "pages_size_example.json")))
    N, L, p, k = g["N"], g["L"], g["p"], g["k"]
    P = O.Params(1, 1, N, 8, L, p, k, 1, expand=True)
    assert P.gathered_length() == 64777                      # 15,625 coarsest entries + 3 levels x 4 x 4,096
    assert abs(P.gathered_length() - g["gathered_about"]) < 0.01 * g["gathered_about"]
    assert O.Params(1, 8, 1 << 20, 128, 4, 4, 4096, 32, expand=True).gathered_length() == 65536


def _expand_case(rng, N=1024, d=8, L=3, p=4, k=8, C=2):
    kx = rand_bf16(rng, (N, d))
    Pe = O.Params(1, 1, N, d, L, p, k, C, expand=True)
    Pp = O.Params(1, 1, N, d, L + 1, p, k, C)                # one level more: level L-1 is ranked, not kept whole
    return kx, Pe, Pp


@pytest.mark.parametrize("L,p,k,C", [(3, 4, 8, 2), (4, 2, 16, 4), (2, 4, 16, 4), (3, 2, 64, 1)])
def test_expand_selection_is_the_children_of_the_per_level_selection_one_level_up(L, p, k, C):
    """The parents the variant picks at level lev+1 are exactly what the per-level reading picks at that level
    (same scores, chunks and k), given one more level so that level L-1 is ranked too."""
    rng = np.random.default_rng(L * 100 + p * 10 + C)
    N = p ** L * 16
    kx, Pe, Pp = _expand_case(rng, N=N, L=L, p=p, k=k, C=C)
    Pe.validate()
    Pp.validate()
    sel_e = O.select(O.norm_scores(O.pyramid(kx, Pe), Pe), Pe)
    sel_p = O.select(O.norm_scores(O.pyramid(kx, Pp), Pp), Pp)
    for lev in range(L - 1):
        parents = sel_p[lev + 1]
        want = sorted(int(J) * p + c for J in parents for c in range(p))
        assert sel_e[lev].tolist() == want, lev
        assert len(sel_e[lev]) == Pe.picks(lev)
    assert sel_e[L - 1].tolist() == list(range(Pe.level_size(L - 1)))


def test_expand_selection_comes_in_sibling_groups_with_equal_counts_per_chunk():
    rng = np.random.default_rng(5)
    P = O.Params(1, 1, 2048, 8, 4, 2, 32, 4, expand=True)
    scores = [rng.random(P.level_size(lev)).astype(np.float32) for lev in P.scored_levels()]
    sel = O.select(scores, P)
    for lev in range(P.L - 1):
        chosen = set(sel[lev].tolist())
        assert all((j ^ 1) in chosen for j in chosen)        # p = 2: every entry with its sibling
        n_c = P.level_size(lev) // P.C
        counts = np.bincount(sel[lev] // n_c, minlength=P.C)
        assert np.all(counts == P.picks(lev) // P.C)
        # brute force: the parents are the top (k/C) of each chunk of level lev+1 by (score desc, index asc)
        par = scores[lev]                                   # scored level lev+1 is entry lev of the list
        m, pc = P.parent_picks(lev + 1) // P.C, P.level_size(lev + 1) // P.C
        want = []
        for c in range(P.C):
            js = sorted(range(c * pc, (c + 1) * pc), key=lambda j: (-float(par[j]), j))[:m]
            want += [2 * j + e for j in sorted(js) for e in range(2)]
        assert sel[lev].tolist() == want


def test_expand_with_k_covering_every_parent_level_is_the_whole_pyramid():
    rng = np.random.default_rng(9)
    N, d = 256, 8
    q, k, v = (rand_bf16(rng, (N, d)) for _ in range(3))
    Pe = O.Params(1, 1, N, d, 3, 4, 64, 2, expand=True)       # N_1 = 64 = k: every level whole
    Pw = O.Params(1, 1, N, d, 3, 4, 256, 2)                   # per-level reading with k = N: every level whole
    assert Pe.gathered_length() == Pw.gathered_length() == 256 + 64 + 16
    fe, fw = O.forward_head(q, k, v, Pe), O.forward_head(q, k, v, Pw)
    assert np.array_equal(fe["idx_g"], fw["idx_g"])
    _close(fe["out"], fw["out"], tol=0)


# ----------------------------------------------------------------------------------------------------------------
# Attention and the whole layer
# ----------------------------------------------------------------------------------------------------------------

def _close(a, b, tol=1e-12):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape
    assert np.all(np.abs(a - b) <= tol * (1 + np.abs(b))), np.max(np.abs(a - b))


@pytest.mark.parametrize("k", [1, 7, 24])
def test_single_level_reduces_to_dense_causal_attention(k):
    rng = np.random.default_rng(5)
    N, d = 24, 8
    P = O.Params(1, 1, N, d, 1, 2, k, 1)
    q, kk, v = (rand_bf16(rng, (N, d)) for _ in range(3))
    res = O.forward_head(q, kk, v, P)
    want = X.textbook_causal_attention(q.tolist(), kk.tolist(), v.tolist())
    _close(res["out"], want)
    assert P.gathered_length() == N


def _full_pyramid_layer_by_hand(q, k, v, P):
    """Independent construction when every entry is selected: exact pooled means rounded to bf16, entries sorted
    by (end, coarser first), textbook causal attention, and each entry's output added to tokens E..E+w-1."""
    N, d = q.shape
    entries = []
    for lev in range(P.L):
        w = P.p ** lev
        for j in range(N // w):
            rows = []
            for x in (q, k, v):
                rows.append([X.to_bf16_exact(sum(Fraction(float(x[t, i])) for t in range(j * w, (j + 1) * w)) / w)
                             for i in range(d)])
            entries.append(((j + 1) * w - 1, -lev, lev, j, rows))
    entries.sort(key=lambda e: (e[0], e[1]))
    og = X.textbook_causal_attention([e[4][0] for e in entries], [e[4][1] for e in entries],
                                     [e[4][2] for e in entries])
    out = [[0.0] * d for _ in range(N)]
    for e, row in zip(entries, og):
        end, lev = e[0], e[2]
        for t in range(end, min(end + P.p ** lev - 1, N - 1) + 1):
            out[t] = [a + b for a, b in zip(out[t], row)]
    return out


@pytest.mark.parametrize("p,L", [(2, 3), (4, 2), (2, 4)])
def test_full_selection_equals_hand_built_pyramid_attention(p, L):
    rng = np.random.default_rng(p + 3 * L)
    N, d = p ** (L - 1) * 4, 8
    P = O.Params(1, 1, N, d, L, p, N, 1)     # k >= every level size: the whole pyramid is selected
    q, k, v = (rand_bf16(rng, (N, d)) for _ in range(3))
    res = O.forward_head(q, k, v, P)
    _close(res["out"], _full_pyramid_layer_by_hand(q, k, v, P), 1e-11)


def test_causality_under_frozen_selection():
    rng = np.random.default_rng(9)
    P = O.Params(1, 1, 64, 8, 3, 2, 4, 2)
    q, k, v = (rand_bf16(rng, (64, 8)) for _ in range(3))
    base = O.forward_head(q, k, v, P)
    for t in [0, 5, 17, 40, 63]:
        q2, k2, v2 = q.copy(), k.copy(), v.copy()
        for x in (q2, k2, v2):
            x[t] = rand_bf16(rng, (1, 8))[0]
        pert = O.forward_head(q2, k2, v2, P, selection=base["sel"])
        _close(pert["out"][:t], base["out"][:t], 1e-13)
        if t < 63:
            assert not np.allclose(pert["out"][t:], base["out"][t:])
        # gradient form: an upstream gradient supported before t gives no gradient at or after t
        dout = np.zeros((64, 8))
        dout[:t] = rng.standard_normal((t, 8))
        dq, dk, dv, _ = O.backward_head(dout, base, P)
        for g in (dq, dk, dv):
            assert np.all(g[t:] == 0)


def test_backward_matches_central_finite_differences():
    rng = np.random.default_rng(13)
    P = O.Params(1, 1, 16, 8, 3, 2, 2, 2)
    q, k, v = (rng.standard_normal((16, 8)) for _ in range(3))
    frozen = O.forward_head(q, k, v, P)["sel"]
    G = rng.standard_normal((16, 8))

    def f(q_, k_, v_):
        return float(np.sum(O.forward_head(q_, k_, v_, P, selection=frozen, round_pool=False)["out"] * G))

    fwd = O.forward_head(q, k, v, P, selection=frozen, round_pool=False)
    grads = O.backward_head(G, fwd, P)[:3]
    h = 1e-6
    for which in range(3):
        for t, i in itertools.product(range(16), range(8)):
            args = [q.copy(), k.copy(), v.copy()]
            args[which][t, i] += h
            fp = f(*args)
            args[which][t, i] -= 2 * h
            fm = f(*args)
            fd = (fp - fm) / (2 * h)
            an = grads[which][t, i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (which, t, i, fd, an)


def test_scatter_backward_is_adjoint_of_scatter():
    rng = np.random.default_rng(17)
    P = O.Params(1, 1, 64, 8, 3, 4, 4, 2)
    scores = [rng.random(P.level_size(lev)).astype(np.float32) for lev in range(P.L - 1)]
    lev_g, j_g, slots = O.gathered_order(O.select(scores, P), P)
    og = rng.standard_normal((len(lev_g), 8))
    dO = rng.standard_normal((64, 8))
    lhs = np.sum(O.scatter(og, slots, P) * dO)
    rhs = np.sum(og * O.scatter_backward(dO, lev_g, j_g, P))
    assert abs(lhs - rhs) <= 1e-12 * (1 + abs(lhs))
