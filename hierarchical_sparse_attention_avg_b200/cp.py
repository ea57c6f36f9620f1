"""Context parallelism: one sequence split across G ranks (one process per GPU), through the C ABI of ``liblh.so``.

The pages' scaling path ([E] "Може ли този подход да скалира отвъд един GPU…"): pooling, scoring and top-K stay
local to each shard; the gathered subsequence is dense, so the attention over it is ordinary causal attention across
ranks.  Rank r holds tokens [r N/G, (r+1) N/G) of every head.  Each rank computes its shard's selection and gathered
rows, the K_g/V_g chunks are all-gathered, every rank attends its own gathered queries over the keys of ranks
0..r, one halo row per (head, level) crosses each shard edge in each direction, and the dK_g/dV_g contributions are
reduce-scattered back to the rank that owns the keys.  All arithmetic runs in the library's kernels; this module
only sizes buffers and issues the exchanges.

``Exchange`` is the collective interface: ``TorchDistExchange`` runs it with ``torch.distributed`` (NCCL between
GPUs, each rank receiving into its own device memory).
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import lh

_lib = lh.library()


class LhCpLayout(ctypes.Structure):
    _fields_ = [("local", lh.LhParams), ("S_local", ctypes.c_int64), ("kv_offset", ctypes.c_uint64),
                ("kv_bytes", ctypes.c_uint64), ("v_offset", ctypes.c_uint64), ("halo_bytes", ctypes.c_uint64),
                ("dkv_bytes", ctypes.c_uint64)]


_P = ctypes.POINTER(lh.LhParams)
_vp = ctypes.c_void_p
_i = ctypes.c_int
_SIGS = {
    "lh_cp_layout": (_i, [_P, _i, ctypes.POINTER(LhCpLayout)]),
    "lh_cp_forward_select": (_i, [_P, _i, _i, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "lh_cp_forward_attend": (_i, [_P, _i, _i, _vp, _vp, _vp, _vp]),
    "lh_cp_forward_scatter": (_i, [_P, _i, _i, _vp, _vp, _vp, _vp]),
    "lh_cp_backward_halo": (_i, [_P, _i, _i, _vp, _vp, _vp]),
    "lh_cp_backward_attend": (_i, [_P, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "lh_cp_backward_unpool": (_i, [_P, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


@dataclass(frozen=True)
class Split:
    """Sizes of the split of global parameters ``P`` over ``G`` ranks (from ``lh_cp_layout``)."""

    P: lh.Params
    G: int
    local: lh.Params
    S_local: int
    kv_offset: int
    kv_bytes: int
    v_offset: int
    halo_bytes: int
    dkv_bytes: int


def split(P: lh.Params, G: int) -> Split:
    out = LhCpLayout()
    lh._check(_lib.lh_cp_layout(ctypes.byref(P.c()), int(G), ctypes.byref(out)), "lh_cp_layout")
    lp = out.local
    local = lh.Params(lp.B, lp.H, lp.N, lp.d, lp.L, lp.p, lp.k, lp.C, bool(lp.flags & lh.LH_EXPAND_CHILDREN))
    return Split(P, int(G), local, int(out.S_local), int(out.kv_offset), int(out.kv_bytes), int(out.v_offset),
                 int(out.halo_bytes), int(out.dkv_bytes))


def halo_prev(halos: torch.Tensor, rank: int):
    """Rank ``rank - 1``'s block of an all-gathered halo exchange ``[G, halo_bytes]`` (None on rank 0)."""
    return halos[rank - 1] if rank > 0 else None


def halo_next(halos: torch.Tensor, rank: int, G: int):
    """Rank ``rank + 1``'s block of an all-gathered halo exchange (None on the last rank)."""
    return halos[rank + 1] if rank < G - 1 else None


def kv_chunk(sp: Split, ctx: torch.Tensor) -> torch.Tensor:
    """The bytes of a rank's context that it contributes to the K_g/V_g all-gather."""
    return ctx[sp.kv_offset: sp.kv_offset + sp.kv_bytes]


class Exchange:
    """Collectives of one rank: ``all_gather(out, inp)`` writes every rank's ``inp`` (same size) into ``out``
    ``[G, n]`` in rank order; ``reduce_scatter(out, inp)`` sums block ``rank`` of every rank's ``inp`` ``[G, n]``
    into ``out`` ``[n]``."""

    def all_gather(self, out: torch.Tensor, inp: torch.Tensor) -> None:
        raise NotImplementedError

    def reduce_scatter(self, out: torch.Tensor, inp: torch.Tensor) -> None:
        raise NotImplementedError


class TorchDistExchange(Exchange):
    def __init__(self, group=None):
        self.group = group

    def all_gather(self, out, inp):
        torch.distributed.all_gather_into_tensor(out.view(-1), inp.contiguous().view(-1), group=self.group)

    def reduce_scatter(self, out, inp):
        torch.distributed.reduce_scatter_tensor(out.view(-1), inp.contiguous().view(-1),
                                                op=torch.distributed.ReduceOp.SUM, group=self.group)


def _ptr(t):
    return None if t is None else lh._ptr(t)


@dataclass
class RankState:
    """Buffers of one rank between the stages (all on its device)."""

    sp: Split
    rank: int
    ctx: torch.Tensor
    ws: torch.Tensor
    kv_all: torch.Tensor
    halos: torch.Tensor
    dkv_part: torch.Tensor
    dkv: torch.Tensor


def new_state(sp: Split, rank: int, device) -> RankState:
    u8 = dict(dtype=torch.uint8, device=device)
    return RankState(sp, rank, lh.new_ctx(sp.local, device), lh.new_workspace(sp.local, device),
                     torch.empty((sp.G, sp.kv_bytes), **u8),
                     torch.empty((sp.G, sp.halo_bytes // 4), dtype=torch.float32, device=device),
                     torch.empty((sp.G, sp.dkv_bytes // 4), dtype=torch.float32, device=device),
                     torch.empty((sp.dkv_bytes // 4,), dtype=torch.float32, device=device))


def _cp(st: RankState):
    return ctypes.byref(st.sp.P.c()), st.sp.G, st.rank


def _stream(t):
    return lh._stream(t.device)


# ---- the stages (each one library call on the rank's current stream) ------------------------------------------

def forward_select(st: RankState, q, k, v):
    rc = _lib.lh_cp_forward_select(*_cp(st), _ptr(q), _ptr(k), _ptr(v), _ptr(st.ctx), _ptr(st.ws), st.ws.numel(),
                                   _stream(q))
    lh._check(rc, "lh_cp_forward_select")


def forward_attend(st: RankState, halo_out: torch.Tensor):
    rc = _lib.lh_cp_forward_attend(*_cp(st), _ptr(st.ctx), _ptr(st.kv_all), _ptr(halo_out), _stream(st.ctx))
    lh._check(rc, "lh_cp_forward_attend")


def forward_scatter(st: RankState, o):
    prev = halo_prev(st.halos, st.rank)
    rc = _lib.lh_cp_forward_scatter(*_cp(st), _ptr(st.ctx), _ptr(prev), _ptr(o), _stream(o))
    lh._check(rc, "lh_cp_forward_scatter")


def backward_halo(st: RankState, dout, halo_out: torch.Tensor):
    rc = _lib.lh_cp_backward_halo(*_cp(st), _ptr(dout), _ptr(halo_out), _stream(dout))
    lh._check(rc, "lh_cp_backward_halo")


def backward_attend(st: RankState, dout):
    nxt = halo_next(st.halos, st.rank, st.sp.G)
    rc = _lib.lh_cp_backward_attend(*_cp(st), _ptr(dout), _ptr(st.ctx), _ptr(st.kv_all), _ptr(nxt),
                                    _ptr(st.dkv_part), _ptr(st.ws), st.ws.numel(), _stream(dout))
    lh._check(rc, "lh_cp_backward_attend")


def backward_unpool(st: RankState, dq, dk, dv):
    rc = _lib.lh_cp_backward_unpool(*_cp(st), _ptr(st.ctx), _ptr(st.dkv), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(st.ws),
                                    st.ws.numel(), _stream(dq))
    lh._check(rc, "lh_cp_backward_unpool")


# ---- one rank's forward and backward with its exchanges ----------------------------------------------------------

def forward(st: RankState, q, k, v, ex: Exchange, o=None):
    """Rank ``st.rank``'s forward: q, k, v bf16 ``[B, H, N/G, d]`` (its shard) -> o (its shard)."""
    o = torch.empty_like(q) if o is None else o
    forward_select(st, q, k, v)
    ex.all_gather(st.kv_all, kv_chunk(st.sp, st.ctx))
    mine = torch.empty((st.sp.halo_bytes // 4,), dtype=torch.float32, device=q.device)
    forward_attend(st, mine)
    ex.all_gather(st.halos, mine)
    forward_scatter(st, o)
    return o


def backward(st: RankState, dout, ex: Exchange, dq=None, dk=None, dv=None):
    """Rank ``st.rank``'s backward (after ``forward`` on the same state): dout of its shard -> dq, dk, dv."""
    dq = torch.empty_like(dout) if dq is None else dq
    dk = torch.empty_like(dout) if dk is None else dk
    dv = torch.empty_like(dout) if dv is None else dv
    mine = torch.empty((st.sp.halo_bytes // 4,), dtype=torch.float32, device=dout.device)
    backward_halo(st, dout, mine)
    ex.all_gather(st.halos, mine)
    backward_attend(st, dout)
    ex.reduce_scatter(st.dkv, st.dkv_part)
    backward_unpool(st, dq, dk, dv)
    return dq, dk, dv
