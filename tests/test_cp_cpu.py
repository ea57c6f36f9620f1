"""Context parallelism on the CPU: two (and four) gloo ranks run the library's exchanges (``cp.TorchDistExchange``,
the halo and chunk conventions of ``cp``) with the oracle's arithmetic standing in for each rank's kernels, and the
assembled forward and backward must equal the oracle on the whole sequence.

This pins the decomposition the GPU path implements: every rank selects within its own shard (G | C, G | k), its
gathered rows are rows r S/G .. of the global gathered sequence, its queries attend the keys of ranks 0..r, one
halo row per (head, level) crosses each shard edge (forward: the previous rank's last entry's output; backward: the
next rank's part of the last window), and dK_g/dV_g contributions are reduce-scattered to the key's owner."""

from __future__ import annotations

import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

# (global parameters, G): every shard's gathered length is a multiple of 128 rows, as the kernels require
CFGS = {
    "L3-G2": ((1, 1, 2048, 64, 3, 4, 64, 4, False), 2),         # S = 256, 128 rows per rank
    "L3-p2-G4": ((1, 1, 4096, 64, 3, 2, 512, 8, False), 4),     # S = 2048, 512 rows per rank
    "expand-L3-G2": ((1, 1, 4096, 64, 3, 4, 32, 4, True), 2),   # S = 512, 256 rows per rank
}


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(cfg, seed=3):
    from oracle import lighthouse as O

    P = O.Params(*cfg)
    rng = np.random.default_rng(seed)
    f = lambda: O.bf16_round(rng.standard_normal((P.N, P.d)) * np.exp(0.5 * rng.standard_normal((P.N, 1))))
    q, k, v = f(), f(), f()
    dout = O.bf16_round(rng.standard_normal((P.N, P.d)))
    return P, q, k, v, dout


def _rank(rank: int, world: int, port: int, name: str, out):
    import datetime

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        out.put((rank, _run_rank(rank, world, name)))
    except Exception as e:  # reported to the parent at once (the other ranks then fail on their next collective)
        out.put((rank, f"{type(e).__name__}: {e}"))
        raise
    finally:
        torch.distributed.destroy_process_group()


def _run_rank(r: int, G: int, name: str):
    from hierarchical_sparse_attention_avg_b200 import cp, lh
    from oracle import lighthouse as O

    cfg, _ = CFGS[name]
    P, q, k, v, dout = _inputs(cfg)
    sp = cp.split(lh.Params(*cfg), G)
    Pl = O.Params(*[getattr(sp.local, f) for f in ("B", "H", "N", "d", "L", "p", "k", "C", "expand")])
    n = Pl.N
    sl = slice(r * n, (r + 1) * n)
    ex = cp.TorchDistExchange()

    # ---- forward: local selection and gather (what lh_cp_forward_select computes)
    pyr = [O.pyramid(x[sl], Pl) for x in (q, k, v)]
    sel = O.select(O.norm_scores(pyr[1], Pl), Pl)
    lev_g, j_g, slots = O.gathered_order(sel, Pl)
    qg, kg, vg = (O.gather(p_, lev_g, j_g) for p_ in pyr)
    S_r = len(lev_g)
    assert S_r == sp.S_local
    # K_g/V_g exchange: one chunk per rank, rank order
    chunk = torch.from_numpy(np.stack([kg, vg]))
    kv_all = torch.empty((G,) + tuple(chunk.shape), dtype=chunk.dtype)
    ex.all_gather(kv_all, chunk)
    K = np.concatenate([kv_all[g, 0].numpy() for g in range(r + 1)])  # keys of ranks 0..r
    V = np.concatenate([kv_all[g, 1].numpy() for g in range(r + 1)])
    # attention of the local queries (global rows r S_r ..) over those keys
    off = r * S_r
    logits = qg @ K.T / math.sqrt(Pl.d)
    logits[np.arange(S_r)[:, None] + off < np.arange(len(K))[None, :]] = -np.inf
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    og = (e @ V) / e.sum(axis=1, keepdims=True)
    lse = (mx + np.log(e.sum(axis=1, keepdims=True)))[:, 0]
    # forward halo: the output row of the shard's last entry of every level (zeros when not selected)
    halo = np.zeros((Pl.L, Pl.d))
    for lev in range(Pl.L):
        s = slots[lev][Pl.level_size(lev) - 1]
        if s >= 0:
            halo[lev] = og[s]
    halos = torch.empty((G, Pl.L * Pl.d), dtype=torch.float64)
    ex.all_gather(halos, torch.from_numpy(halo.reshape(-1)))
    o = O.scatter(og, slots, Pl)
    prev = cp.halo_prev(halos, r)
    if prev is not None:
        prev = prev.numpy().reshape(Pl.L, Pl.d)
        for lev in range(Pl.L):
            o[: Pl.window(lev) - 1] += prev[lev]

    # ---- backward
    dl = dout[sl]
    hb = np.zeros((Pl.L, Pl.d))
    for lev in range(Pl.L):
        hb[lev] = dl[: Pl.window(lev) - 1].sum(axis=0)
    ex.all_gather(halos, torch.from_numpy(hb.reshape(-1)))
    dog = O.scatter_backward(dl, lev_g, j_g, Pl)
    nxt = cp.halo_next(halos, r, G)
    if nxt is not None:
        nxt = nxt.numpy().reshape(Pl.L, Pl.d)
        for lev in range(Pl.L):
            s = slots[lev][Pl.level_size(lev) - 1]
            if s >= 0:
                dog[s] += nxt[lev]
    scale = 1.0 / math.sqrt(Pl.d)
    prob = np.exp(logits - lse[:, None])
    dV = prob.T @ dog
    dprob = dog @ V.T
    delta = (dog * og).sum(axis=1, keepdims=True)
    dlog = prob * (dprob - delta)
    dQ = dlog @ K * scale
    dK = dlog.T @ qg * scale
    part = np.zeros((G, 2, S_r, Pl.d))  # this rank's contribution to every rank's keys (zeros after rank r)
    for g in range(r + 1):
        part[g, 0] = dK[g * S_r:(g + 1) * S_r]
        part[g, 1] = dV[g * S_r:(g + 1) * S_r]
    mine = torch.empty((2, S_r, Pl.d), dtype=torch.float64)
    ex.reduce_scatter(mine, torch.from_numpy(part))
    dq = O.unpool_backward(dQ, slots, Pl)
    dk = O.unpool_backward(mine[0].numpy(), slots, Pl)
    dv = O.unpool_backward(mine[1].numpy(), slots, Pl)
    return dict(idx_g=O.global_ids(lev_g, j_g, Pl), o=o, dq=dq, dk=dk, dv=dv, S_r=S_r)


@pytest.mark.parametrize("name", list(CFGS))
def test_context_parallel_split_equals_the_whole_sequence(name):
    from oracle import lighthouse as O

    cfg, world = CFGS[name]
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, name, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, got = out.get(timeout=240)
        assert not isinstance(got, str), f"rank {r}: {got}"
        res[r] = got
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    P, q, k, v, dout = _inputs(cfg)
    ref = O.forward_head(q, k, v, P)
    grads = O.backward_head(dout, ref, P)
    S = P.gathered_length()
    assert sum(res[r]["S_r"] for r in range(world)) == S
    n = P.N // world
    for r in range(world):
        # the shard's gathered rows are the global sequence's rows r S/G .. (entry ids shifted to global)
        lev_g = ref["lev_g"][r * (S // world):(r + 1) * (S // world)]
        j_g = ref["j_g"][r * (S // world):(r + 1) * (S // world)]
        Pl = O.Params(P.B, P.H, n, P.d, P.L, P.p, P.k // world, P.C // world, P.expand)
        local_ids = O.global_ids(lev_g, j_g - np.array([r * Pl.level_size(int(l)) for l in lev_g]), Pl)
        assert np.array_equal(res[r]["idx_g"], local_ids), r
        sl = slice(r * n, (r + 1) * n)
        for key, want in (("o", ref["out"]), ("dq", grads[0]), ("dk", grads[1]), ("dv", grads[2])):
            np.testing.assert_allclose(res[r][key], want[sl], rtol=1e-10, atol=1e-12, err_msg=f"{key} rank {r}")


def test_split_sizes_and_rejections():
    from hierarchical_sparse_attention_avg_b200 import cp, lh

    P = lh.Params(1, 16, 524288, 128, 4, 4, 4096, 32)
    sp = cp.split(P, 8)
    assert (sp.local.N, sp.local.k, sp.local.C, sp.S_local) == (65536, 512, 4, 2560)
    assert sp.halo_bytes == 16 * 4 * 128 * 4 and sp.dkv_bytes == 2 * 16 * 2560 * 128 * 4
    assert sp.kv_bytes >= 2 * 16 * 2560 * 128 * 2 and sp.v_offset >= 16 * 2560 * 128 * 2
    assert cp.split(lh.Params(1, 8, 1048576, 128, 4, 4, 4096, 32), 8).S_local == 3584
    for G, code in ((3, lh.LH_ERR_INVALID_ARG),   # 3 does not divide C = 32
                    (64, lh.LH_ERR_INVALID_ARG),  # 64 does not divide C = 32
                    (0, lh.LH_ERR_INVALID_ARG)):
        with pytest.raises(lh.LighthouseError) as e:
            cp.split(P, G)
        assert e.value.status == code
    with pytest.raises(lh.LighthouseError) as e:  # S/G = 7680/8 = 960 is not a multiple of 128
        cp.split(lh.Params(1, 16, 98304, 64, 4, 4, 2048, 16), 8)
    assert e.value.status == lh.LH_ERR_UNSUPPORTED
    halos = torch.arange(12.0).view(3, 4)
    assert cp.halo_prev(halos, 0) is None and torch.equal(cp.halo_prev(halos, 2), halos[1])
    assert cp.halo_next(halos, 2, 3) is None and torch.equal(cp.halo_next(halos, 0, 3), halos[1])
