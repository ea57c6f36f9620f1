"""Context parallelism through the C ABI on one GPU: the G ranks of a split are run one after another in this
process (every exchange done by copying each rank's buffer into the others', in rank order), so no kernel ever
waits for another rank.  The assembled outputs and gradients must match the oracle on the whole sequence within the
layer's tolerance, and the selection and gathered rows must equal those of ``lh_forward`` on the whole sequence bit
for bit.  G = 1 runs the same entry points with no neighbour and must reproduce ``lh_forward``/``lh_backward``."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from hierarchical_sparse_attention_avg_b200.inputs import make_inputs
from oracle import lighthouse as O
from tests._parity import assert_close, f64

pytestmark = pytest.mark.gpu

CASES = {
    # (global parameters, G); every shard's gathered length is a multiple of 128
    "L3-d64-G2": ((1, 2, 8192, 64, 3, 4, 256, 8), 2),                # S = 1024, 512 per rank
    "L3-d64-G4": ((1, 2, 8192, 64, 3, 4, 256, 8), 4),                # 256 per rank
    "L4-d128-G2": ((1, 2, 16384, 128, 4, 4, 512, 8), 2),             # S = 1792, 896 per rank
    "expand-L3-d64-G2": ((1, 2, 8192, 64, 3, 4, 64, 4, True), 2),    # S = 1024, 512 per rank
    "L3-d64-G1": ((1, 2, 8192, 64, 3, 4, 256, 8), 1),
}


def _shard(x, r, G):
    n = x.shape[2] // G
    return x[:, :, r * n:(r + 1) * n].contiguous()


def _run_split(cfg, G, q, k, v, dout):
    from hierarchical_sparse_attention_avg_b200 import cp, lh

    P = lh.Params(*cfg)
    sp = cp.split(P, G)
    dev = q.device
    st = [cp.new_state(sp, r, dev) for r in range(G)]
    shards = [[_shard(t, r, G) for t in (q, k, v, dout)] for r in range(G)]
    o = [torch.empty_like(s[0]) for s in shards]
    grads = [[torch.empty_like(s[0]) for _ in range(3)] for s in shards]

    def all_gather(parts, field):
        full = torch.stack(parts)
        for s in st:
            getattr(s, field).copy_(full)

    for r in range(G):
        cp.forward_select(st[r], *shards[r][:3])
    all_gather([cp.kv_chunk(sp, s.ctx) for s in st], "kv_all")
    halo = [torch.empty((sp.halo_bytes // 4,), dtype=torch.float32, device=dev) for _ in range(G)]
    for r in range(G):
        cp.forward_attend(st[r], halo[r])
    all_gather(halo, "halos")
    for r in range(G):
        cp.forward_scatter(st[r], o[r])
    for r in range(G):
        cp.backward_halo(st[r], shards[r][3], halo[r])
    all_gather(halo, "halos")
    for r in range(G):
        cp.backward_attend(st[r], shards[r][3])
    for r in range(G):  # reduce-scatter: rank r receives the sum of every rank's block r
        st[r].dkv.copy_(torch.stack([st[g].dkv_part[r] for g in range(G)]).sum(dim=0))
    for r in range(G):
        cp.backward_unpool(st[r], *grads[r])
    cat = lambda ts: torch.cat(ts, dim=2)
    return sp, st, cat(o), tuple(cat([g[i] for g in grads]) for i in range(3))


@pytest.mark.parametrize("name", list(CASES))
def test_split_matches_the_whole_sequence(name, cuda_device):
    from hierarchical_sparse_attention_avg_b200 import lh

    cfg, G = CASES[name]
    P, Q = lh.Params(*cfg), O.Params(*cfg)
    q, k, v, dout = (t.to(cuda_device) for t in make_inputs(Q.B, Q.H, Q.N, Q.d, seed=0, device="cpu"))
    sp, st, o, (dq, dk, dv) = _run_split(cfg, G, q, k, v, dout)
    assert lh.lh_get_status() == 0
    # the whole sequence through the ordinary entry points
    o1, ctx1 = lh.lh_forward(P, q, k, v)
    dq1, dk1, dv1 = lh.lh_backward(P, dout, ctx1)
    whole = lh.ctx_views(P, ctx1)
    S_r = sp.S_local
    for r in range(G):
        loc = lh.ctx_views(sp.local, st[r].ctx)
        rows = slice(r * S_r, (r + 1) * S_r)
        for key in ("qg", "kg", "vg"):
            assert torch.equal(loc[key], whole[key][:, :, rows]), (key, r)
        # local pyramid ids = global ids shifted by the shard's first entry of each level
        gid = whole["idx_g"][:, :, rows].cpu().numpy().astype(np.int64)
        lev = np.searchsorted([Q.level_offset(l) for l in range(1, Q.L)], gid, side="right")
        j = gid - np.array([Q.level_offset(l) for l in range(Q.L)])[lev]
        shift = np.array([r * Q.level_size(l) // G for l in range(Q.L)])[lev]
        loff = np.array([Q.level_offset(l) // G for l in range(Q.L)])[lev]
        assert np.array_equal(loc["idx_g"].cpu().numpy(), loff + j - shift), r
    if G == 1:
        assert torch.equal(o, o1) and torch.equal(dk, dk1) and torch.equal(dv, dv1)
    for (b, h) in [(b, h) for b in range(Q.B) for h in range(Q.H)]:
        ref = O.forward_head(f64(q[b, h].cpu()), f64(k[b, h].cpu()), f64(v[b, h].cpu()), Q)
        assert_close(f64(o[b, h]), ref["out"], what=f"{name} O{(b, h)}")
        gq, gk, gv, _ = O.backward_head(f64(dout[b, h].cpu()), ref, Q)
        assert_close(f64(dq[b, h]), gq, what=f"{name} dQ{(b, h)}")
        assert_close(f64(dk[b, h]), gk, what=f"{name} dK{(b, h)}")
        assert_close(f64(dv[b, h]), gv, what=f"{name} dV{(b, h)}")
