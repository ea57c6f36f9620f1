"""lh_step_host (host tensors in and out, copies pipelined by head chunks) against the device entry points.

O, dK and dV are bit-identical to lh_forward / lh_backward on the same data: every chunk computes its heads exactly
as the call over all heads does.  dQ sums the key tiles' contributions with floating-point reduce-adds whose order
is not fixed, so it is compared within the layer's tolerance |d| <= 2e-2 + 2e-2 |ref| (and almost always agrees
to the bit)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from hierarchical_sparse_attention_avg_b200.inputs import make_inputs
from tests._parity import assert_close, bits16, f64

pytestmark = pytest.mark.gpu

CASES = {
    "tiny-d64-one-head-chunks": ((1, 2, 4096, 64, 3, 4, 256, 8), 1),
    "B2-d128-p8": ((2, 2, 4096, 128, 3, 8, 64, 4), 1),
    "H4-d128-two-head-chunks": ((1, 4, 8192, 128, 4, 4, 256, 8), 2),
}


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("pinned", [True, False], ids=["pinned", "pageable"])
def test_step_host_matches_device_path(name, pinned, cuda_device):
    from hierarchical_sparse_attention_avg_b200 import lh

    cfg, hc = CASES[name]
    P = lh.Params(*cfg)
    q, k, v, dout = make_inputs(P.B, P.H, P.N, P.d, seed=5, device="cpu")
    dev = cuda_device
    o_ref, ctx = lh.lh_forward(P, q.to(dev), k.to(dev), v.to(dev))
    dq_ref, dk_ref, dv_ref = lh.lh_backward(P, dout.to(dev), ctx)
    host = [t.pin_memory() if pinned else t.clone() for t in (q, k, v, dout)]
    outs = None if pinned else [torch.empty_like(q) for _ in range(4)]
    kw = {} if outs is None else dict(o=outs[0], dq=outs[1], dk=outs[2], dv=outs[3])
    o, dq, dk, dv = lh.lh_step_host(P, *host, heads_per_chunk=hc, device=dev, **kw)
    torch.cuda.current_stream(dev).synchronize()
    assert lh.lh_get_status(dev) == 0
    for got, want, what in ((o, o_ref, "o"), (dk, dk_ref, "dk"), (dv, dv_ref, "dv")):
        assert np.array_equal(bits16(got), bits16(want)), what
    assert_close(f64(dq), f64(dq_ref), what="dq")
