"""The device status paths of the library, each driven to its error on purpose without faulting the GPU.

- LH_ERR_TIMEOUT: every device-side wait of the attention kernels is bounded.  ``lh_set_wait_limit_ns(1)`` makes
  each wait that finds its barrier phase incomplete give up at once; the kernels then drain the copies and
  tensor-core products they issued, free their tensor memory and return, and ``lh_get_status`` reports the timeout.
  The next call, with the default limit restored, must be clean and match the oracle.
- LH_ERR_RANGE: the attention takes fp16 operands; a bf16 input beyond 65504 in a selected row is reported.
- Tiny upstream gradients: the backward scales dO_g per head by a power of two before rounding it to fp16; the
  scale is capped so that it and its inverse stay finite.  A gradient 2^-100 times smaller gives results 2^-100
  times smaller (compared against the oracle after scaling back), and one near 1e-38 stays finite.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from hierarchical_sparse_attention_avg_b200.inputs import make_inputs
from oracle import lighthouse as O
from tests._parity import assert_close, f64

pytestmark = pytest.mark.gpu

CFG = (1, 2, 4096, 64, 3, 4, 256, 8)  # the 4K correctness configuration


@pytest.fixture(scope="module")
def setup(cuda_device):
    from hierarchical_sparse_attention_avg_b200 import lh

    P, Q = lh.Params(*CFG), O.Params(*CFG)
    q, k, v, dout = make_inputs(Q.B, Q.H, Q.N, Q.d, seed=0, device="cpu")
    ref = {h: O.forward_head(f64(q[0, h]), f64(k[0, h]), f64(v[0, h]), Q) for h in range(Q.H)}
    dev = cuda_device
    return dict(lh=lh, P=P, Q=Q, ref=ref, q=q, k=k, v=v, dout=dout, dev=dev)


def _check_layer(s, o, dq, dk, dv, dout):
    Q = s["Q"]
    for h in range(Q.H):
        r = s["ref"][h]
        assert_close(f64(o[0, h]), r["out"], what=f"O{h}")
        rq, rk, rv, _ = O.backward_head(f64(dout[0, h]), r, Q)
        assert_close(f64(dq[0, h]), rq, what=f"dQ{h}")
        assert_close(f64(dk[0, h]), rk, what=f"dK{h}")
        assert_close(f64(dv[0, h]), rv, what=f"dV{h}")


def _step(s, q=None, dout=None):
    lh, P, dev = s["lh"], s["P"], s["dev"]
    q = s["q"] if q is None else q
    dout = s["dout"] if dout is None else dout
    o, ctx = lh.lh_forward(P, q.to(dev), s["k"].to(dev), s["v"].to(dev))
    dq, dk, dv = lh.lh_backward(P, dout.to(dev), ctx)
    return o, dq, dk, dv


@pytest.mark.parametrize("d", [64, 128])
def test_wait_timeout_is_reported_and_the_next_call_is_clean(setup, d):
    lh = setup["lh"]
    cfg = (1, 2, 4096, d, 3, 4, 256, 8)
    P = lh.Params(*cfg)
    q, k, v, dout = (t.to(setup["dev"]) for t in make_inputs(1, 2, 4096, d, seed=0, device="cpu"))
    assert lh.lh_get_status() == 0
    lh.lh_set_wait_limit_ns(1)
    try:
        o, ctx = lh.lh_forward(P, q, k, v)
        lh.lh_backward(P, dout, ctx)
        status = lh.lh_get_status()
    finally:
        lh.lh_set_wait_limit_ns(0)
    assert status == lh.LH_ERR_TIMEOUT, lh.error_string(status)
    assert lh.lh_get_status() == 0  # reading the status cleared it
    if d == 64:
        o, dq, dk, dv = _step(setup)
        assert lh.lh_get_status() == 0
        _check_layer(setup, o, dq, dk, dv, setup["dout"])


def test_short_wait_limit_aborts_anywhere_and_the_next_call_is_clean(setup):
    """A limit of a few microseconds lets some waits finish and makes others give up wherever they are."""
    lh = setup["lh"]
    for ns in (2000, 8000, 30000):
        lh.lh_set_wait_limit_ns(ns)
        try:
            _step(setup)
            status = lh.lh_get_status()
        finally:
            lh.lh_set_wait_limit_ns(0)
        assert status in (0, lh.LH_ERR_TIMEOUT), lh.error_string(status)
    o, dq, dk, dv = _step(setup)
    assert lh.lh_get_status() == 0
    _check_layer(setup, o, dq, dk, dv, setup["dout"])


def test_value_beyond_fp16_range_is_reported(setup):
    lh = setup["lh"]
    for which in ("q", "k", "v"):
        x = setup[which].clone()
        x[0, 1, 777, 5] = 7.0e6  # its level-0 row and the coarsest entry holding it leave the fp16 range
        args = {n: setup[n] for n in ("q", "k", "v")}
        args[which] = x
        o, ctx = lh.lh_forward(setup["P"], *(args[n].to(setup["dev"]) for n in ("q", "k", "v")))
        assert lh.lh_get_status() == lh.LH_ERR_RANGE, which
    o, dq, dk, dv = _step(setup)
    assert lh.lh_get_status() == 0
    _check_layer(setup, o, dq, dk, dv, setup["dout"])


def test_small_gradient_scales_exactly(setup):
    """bf16(2^-100 dO) = 2^-100 bf16(dO) exactly, and the oracle is linear in dO: the gradients scaled back by
    2^100 must meet the usual tolerance against the oracle's."""
    lh = setup["lh"]
    c = 2.0 ** -100
    dout_small = (setup["dout"].to(torch.float32) * c).to(torch.bfloat16)
    assert torch.equal(dout_small.to(torch.float32) / c, setup["dout"].to(torch.float32))
    o, dq, dk, dv = _step(setup, dout=dout_small)
    assert lh.lh_get_status() == 0
    up = lambda t: (t.to(torch.float32) / c)
    for t in (dq, dk, dv):
        assert torch.isfinite(t.to(torch.float32)).all()
    _check_layer(setup, o, up(dq), up(dk), up(dv), setup["dout"])


def test_gradient_near_1e_minus_38_stays_finite(setup):
    """A head whose window-summed gradient is below 2^-116 gets the capped scale 2^126: results stay finite and
    within the tolerance of the oracle's (which are themselves ~1e-38)."""
    lh, Q = setup["lh"], setup["Q"]
    dout_tiny = (setup["dout"].to(torch.float32) * 1e-38).to(torch.bfloat16)
    o, dq, dk, dv = _step(setup, dout=dout_tiny)
    assert lh.lh_get_status() == 0
    for t in (dq, dk, dv):
        assert torch.isfinite(t.to(torch.float32)).all()
    for h in range(Q.H):
        rq, rk, rv, _ = O.backward_head(f64(dout_tiny[0, h]), setup["ref"][h], Q)
        for got, want, n in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV")):
            assert_close(f64(got[0, h]), want, what=f"{n}{h}")
            assert np.max(np.abs(f64(got[0, h]))) <= 1e-30
