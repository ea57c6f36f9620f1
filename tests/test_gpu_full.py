"""GPU parity at the full benchmark configurations, in the launch configuration ``bench.py`` times
(``lh_forward`` + ``lh_backward`` over [B, H, N, d] inputs generated on the device).

* pooled scores and the selection (idx_g, slot) are checked bit-exact for EVERY head;
* the gathered rows are checked bit-exact, and O, dQ, dK, dV within |d| <= 2e-2 + 2e-2 |ref|, on the first and
  last head (the oracle runs the whole head in float64)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from hierarchical_sparse_attention_avg_b200.inputs import make_inputs
from oracle import lighthouse as O
from tests._parity import assert_close, f64

pytestmark = [pytest.mark.gpu, pytest.mark.full]

FULL = {
    "train32K": (1, 16, 32768, 64, 4, 4, 2048, 16),
    "ctx98K": (1, 16, 98304, 64, 4, 4, 2048, 16),
    "long512K": (1, 16, 524288, 128, 4, 4, 4096, 32),
    "stress1M": (1, 8, 1048576, 128, 4, 4, 4096, 32),
}


@pytest.mark.parametrize("name", list(FULL))
def test_full_configuration(name, cuda_device):
    from hierarchical_sparse_attention_avg_b200 import lh

    cfg = FULL[name]
    P, Q = lh.Params(*cfg), O.Params(*cfg)
    dev = cuda_device
    q, k, v, dout = make_inputs(Q.B, Q.H, Q.N, Q.d, seed=0, device=dev)
    o, ctx = lh.lh_forward(P, q, k, v)
    dq, dk, dv = lh.lh_backward(P, dout, ctx)
    assert lh.lh_get_status(dev) == 0
    views = lh.ctx_views(P, ctx)
    idx_all = views["idx_g"].cpu().numpy()
    slot_all = views["slot"].cpu().numpy()
    k_cpu = k.cpu()
    assert Q.gathered_length() == lh.lh_S(P)

    # selection on every head: pool the keys, score, select, order (oracle) vs the GPU context
    for h in range(Q.H):
        kp = O.pyramid(f64(k_cpu[0, h]), Q)
        sel = O.select(O.norm_scores(kp, Q), Q)
        lev_g, j_g, slots = O.gathered_order(sel, Q)
        assert np.array_equal(idx_all[0, h], O.global_ids(lev_g, j_g, Q)), f"{name}: selection of head {h}"
        assert np.array_equal(slot_all[0, h], O.slot_map(slots)), f"{name}: slot map of head {h}"
    del k_cpu

    for h in sorted({0, Q.H - 1}):
        ref = O.forward_head(f64(q[0, h].cpu()), f64(k[0, h].cpu()), f64(v[0, h].cpu()), Q)
        for key in ("qg", "kg", "vg"):
            want = ref[key].astype(np.float16).astype(np.float64)  # the documented fp16 operand conversion
            assert np.array_equal(f64(views[key][0, h]), want), f"{name}: {key} of head {h}"
        assert_close(f64(o[0, h]), ref["out"], what=f"{name} O head {h}")
        gq, gk, gv, _ = O.backward_head(f64(dout[0, h].cpu()), ref, Q)
        assert_close(f64(dq[0, h]), gq, what=f"{name} dQ head {h}")
        assert_close(f64(dk[0, h]), gk, what=f"{name} dK head {h}")
        assert_close(f64(dv[0, h]), gv, what=f"{name} dV head {h}")
        del ref, gq, gk, gv
    torch.cuda.synchronize(dev)


def test_expand_variant_at_one_million_tokens(cuda_device):
    """The children-expansion variant at the pages' size example (N = 2^20, L = 4, p = 4, k = 4096: S = 65,536).
    Selection bit-exact on every head; on the first and last head the gathered rows bit-exact and, on sampled rows
    (the oracle computes one attention row at a time, O(S d) each), O_g and LSE within the tolerance, and O at
    sampled tokens as the sum of the oracle's rows of their contributing entries."""
    from hierarchical_sparse_attention_avg_b200 import lh

    cfg = (1, 8, 1048576, 128, 4, 4, 4096, 32, True)
    P, Q = lh.Params(*cfg), O.Params(*cfg)
    dev = cuda_device
    assert lh.lh_S(P) == Q.gathered_length() == 65536
    q, k, v, dout = make_inputs(Q.B, Q.H, Q.N, Q.d, seed=0, device=dev)
    o, ctx = lh.lh_forward(P, q, k, v)
    lh.lh_backward(P, dout, ctx)
    assert lh.lh_get_status(dev) == 0
    views = lh.ctx_views(P, ctx)
    idx_all = views["idx_g"].cpu().numpy()
    slot_all = views["slot"].cpu().numpy()
    k_cpu = k.cpu()
    for h in range(Q.H):
        sel = O.select(O.norm_scores(O.pyramid(f64(k_cpu[0, h]), Q), Q), Q)
        lev_g, j_g, slots = O.gathered_order(sel, Q)
        assert np.array_equal(idx_all[0, h], O.global_ids(lev_g, j_g, Q)), f"selection of head {h}"
        assert np.array_equal(slot_all[0, h], O.slot_map(slots)), f"slot map of head {h}"
    del k_cpu
    rng = np.random.default_rng(1)
    scale = 1.0 / np.sqrt(Q.d)
    for h in sorted({0, Q.H - 1}):
        pyr = [O.pyramid(f64(t[0, h].cpu()), Q) for t in (q, k, v)]
        sel = O.select(O.norm_scores(pyr[1], Q), Q)
        lev_g, j_g, slots = O.gathered_order(sel, Q)
        qg, kg, vg = (O.gather(pp, lev_g, j_g) for pp in pyr)
        for key, ref in (("qg", qg), ("kg", kg), ("vg", vg)):
            assert np.array_equal(f64(views[key][0, h]), ref.astype(np.float16).astype(np.float64)), (key, h)
        og_gpu, lse_gpu, o_gpu = f64(views["og"][0, h]), f64(views["lse"][0, h]), f64(o[0, h])

        def og_row(s):  # one row of causal attention over the gathered sequence, float64
            logits = kg[: s + 1] @ qg[s] * scale
            mx = logits.max()
            e = np.exp(logits - mx)
            return (e @ vg[: s + 1]) / e.sum(), mx + np.log(e.sum())

        rows = np.unique(np.concatenate([[0, 1, 65535], rng.integers(0, 65536, 48)]))
        for s in rows:
            want, lse = og_row(int(s))
            assert_close(og_gpu[s], want, what=f"O_g row {s} head {h}")
            assert_close(lse_gpu[s], lse, atol=2e-3, rtol=1e-4, what=f"LSE row {s} head {h}")
        for t in np.unique(np.concatenate([[0, 3, 63, Q.N - 1], rng.integers(0, Q.N, 32)])):
            want = np.zeros(Q.d)
            for lev in range(Q.L):
                j = (int(t) + 1) // Q.window(lev) - 1
                if j >= 0 and slots[lev][j] >= 0:
                    want += og_row(int(slots[lev][j]))[0]
            assert_close(o_gpu[t], want, what=f"O token {t} head {h}")
    torch.cuda.synchronize(dev)
