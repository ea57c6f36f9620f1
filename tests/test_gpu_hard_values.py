"""Bit-exact parity of the exact steps (pool, score, selection, gather) on adversarial values.

The pool and gather kernels sum in fp32 with two directed roundings and fall back to fp64 where the two differ or the
pooled value would be subnormal; the scores are fp64 sums of squares rounded once to fp32.  These inputs mix zeros of
both signs, bf16 subnormals and exponents spread over 2^-140 .. 2^3, so that every fallback runs: entries whose fp32
sum is inexact, entries whose sum is exact but subnormal, and rows whose score lies in the fp32 subnormal range.
The recomputed levels cover 8 (p=8), 16 (p=4, level 2), 64 (p=4, level 3: child by child) and 2..8 (p=2) raw
rows."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from hierarchical_sparse_attention_avg_b200.inputs import make_hard_inputs
from oracle import lighthouse as O
from tests._parity import bits16, f64

pytestmark = pytest.mark.gpu

CASES = {
    "hard-d128-p4-L4": (1, 2, 4096, 128, 4, 4, 64, 4),  # levels 1 and 2 recomputed (4 and 16 raw rows)
    "hard-d64-p4-L5": (1, 1, 4096, 64, 5, 4, 32, 2),    # level 3 recomputed from 64 raw rows
    "hard-d128-p8-L3": (1, 1, 4096, 128, 3, 8, 64, 4),  # level 1 from 8 raw rows
    "hard-d64-p2-L5": (1, 1, 2048, 64, 5, 2, 64, 4),    # levels 1..3 from 2, 4 and 8 raw rows
}


@pytest.fixture(scope="module", params=list(CASES), ids=list(CASES))
def case(request, cuda_device):
    from hierarchical_sparse_attention_avg_b200 import lh

    cfg = CASES[request.param]
    P, Q = lh.Params(*cfg), O.Params(*cfg)
    q, k, v = make_hard_inputs(Q.B, Q.H, Q.N, Q.d, seed=11)
    heads = [(b, h) for b in range(Q.B) for h in range(Q.H)]
    ref = {bh: O.forward_head(f64(q[bh]), f64(k[bh]), f64(v[bh]), Q) for bh in heads}
    dev = cuda_device
    return dict(lh=lh, P=P, Q=Q, heads=heads, ref=ref, q=q.to(dev), k=k.to(dev), v=v.to(dev))


def _fp16(a):
    return np.asarray(a, dtype=np.float64).astype(np.float16).astype(np.float64)


def test_inputs_reach_the_fallbacks(case):
    """The inputs do hold what the docstring promises (checked on the oracle's own pyramid)."""
    Q = case["Q"]
    k = f64(case["k"].cpu())
    assert np.any(k == 0) and np.any(np.signbit(k) & (k == 0)), "zeros of both signs"
    assert np.any((k != 0) & (np.abs(k) < 2.0 ** -126)), "bf16 subnormals"
    pyr = np.concatenate(case["ref"][case["heads"][0]]["pyr_k"][1:])
    assert np.any((pyr != 0) & (np.abs(pyr) < 2.0 ** -126)), "subnormal pooled values"
    sc = np.concatenate(case["ref"][case["heads"][0]]["scores"])
    assert np.any((sc != 0) & (sc < np.float32(2.0 ** -126))), "subnormal scores"


def test_pool_bit_exact_hard(case):
    lh, P = case["lh"], case["P"]
    for name, key in (("q", "pyr_q"), ("k", "pyr_k"), ("v", "pyr_v")):
        got = bits16(lh.lh_pool(P, case[name]))
        for (b, h) in case["heads"]:
            want = np.concatenate(case["ref"][(b, h)][key][1:])
            assert np.array_equal(got[b, h], O.bf16_bits(want)), (name, b, h)


def test_scores_and_selection_bit_exact_hard(case):
    lh, P, Q = case["lh"], case["P"], case["Q"]
    scores = torch.empty((Q.B, Q.H, lh.lh_score_rows(P)), dtype=torch.float32, device=case["q"].device)
    idx_g, _ = lh.lh_score_topk(P, case["k"], scores_out=scores)
    got = scores.cpu().numpy()
    for (b, h) in case["heads"]:
        want = np.concatenate(case["ref"][(b, h)]["scores"])
        assert np.array_equal(got[b, h].view(np.uint32), want.view(np.uint32)), (b, h)
        assert np.array_equal(idx_g[b, h].cpu().numpy(), case["ref"][(b, h)]["idx_g"]), (b, h)


def test_forward_gathered_rows_bit_exact_hard(case):
    """lh_forward stores only the coarsest level, so the gather recomputes every other pooled row."""
    lh, P = case["lh"], case["P"]
    _, ctx = lh.lh_forward(P, case["q"], case["k"], case["v"])
    views = lh.ctx_views(P, ctx)
    for (b, h) in case["heads"]:
        r = case["ref"][(b, h)]
        assert np.array_equal(views["idx_g"][b, h].cpu().numpy(), r["idx_g"]), (b, h)
        for key in ("qg", "kg", "vg"):
            assert np.array_equal(f64(views[key][b, h]), _fp16(r[key])), (key, b, h)
