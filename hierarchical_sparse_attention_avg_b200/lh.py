"""Thin Python binding of ``liblh.so`` (the C ABI declared in ``include/lh.h``).

Only argument marshalling happens here: every step of the layer runs in the library's CUDA kernels.  PyTorch
provides device memory and the current stream.  Function names match the C entry points.  Importing this module
raises when the library has not been built; there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblh.so")

LH_OK = 0
LH_ERR_INVALID_ARG = 1
LH_ERR_UNSUPPORTED = 2
LH_ERR_CUDA = 3
LH_ERR_TIMEOUT = 4
LH_ERR_WORKSPACE = 5
LH_ERR_RANGE = 6

LH_EXPAND_CHILDREN = 1


class LhParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "H", "N", "d", "L", "p", "k", "C", "flags")]


class LhCtxLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in ("qg", "kg", "vg", "og", "lse", "idx_g", "slot", "total")]


class LhKernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int32), ("ms", ctypes.c_double)]


class LighthouseError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {error_string(status)} (status {status})")


_P = ctypes.POINTER(LhParams)
_vp = ctypes.c_void_p
_SIGS = {
    "lh_error_string": (ctypes.c_char_p, [ctypes.c_int]),
    "lh_validate": (ctypes.c_int, [_P]),
    "lh_S": (ctypes.c_int64, [_P]),
    "lh_level_size": (ctypes.c_int64, [_P, ctypes.c_int]),
    "lh_level_offset": (ctypes.c_int64, [_P, ctypes.c_int]),
    "lh_pyramid_rows": (ctypes.c_int64, [_P]),
    "lh_score_rows": (ctypes.c_int64, [_P]),
    "lh_slot_rows": (ctypes.c_int64, [_P]),
    "lh_ctx_bytes": (ctypes.c_size_t, [_P]),
    "lh_ctx_layout": (ctypes.c_int, [_P, ctypes.POINTER(LhCtxLayout)]),
    "lh_workspace_bytes": (ctypes.c_size_t, [_P]),
    "lh_pool": (ctypes.c_int, [_P, _vp, _vp, _vp]),
    "lh_score_topk": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "lh_gather": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "lh_attend": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp]),
    "lh_scatter": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp]),
    "lh_forward": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "lh_backward": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "lh_scatter_bwd": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp]),
    "lh_attend_bwd": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "lh_get_status": (ctypes.c_int, [_vp]),
    "lh_set_wait_limit_ns": (ctypes.c_int, [ctypes.c_uint64]),
    "lh_score_topk_static": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp]),
    "lh_profile_enable": (ctypes.c_int, [ctypes.c_int]),
    "lh_profile_read": (ctypes.c_int, [ctypes.POINTER(LhKernelTime), ctypes.c_int]),
    "lh_step_host_bytes": (ctypes.c_size_t, [_P, ctypes.c_int]),
    "lh_step_host": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int, _vp, ctypes.c_size_t, _vp,
                                    _vp, _vp]),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m hierarchical_sparse_attention_avg_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def library() -> ctypes.CDLL:
    return _lib


# ------------------------------------------------------------------------------------------------------------
# Parameters and host-only queries
# ------------------------------------------------------------------------------------------------------------

@dataclass(frozen=True)
class Params:
    B: int
    H: int
    N: int
    d: int
    L: int
    p: int
    k: int
    C: int
    expand: bool = False  # LH_EXPAND_CHILDREN

    def c(self) -> LhParams:
        return LhParams(self.B, self.H, self.N, self.d, self.L, self.p, self.k, self.C,
                        LH_EXPAND_CHILDREN if self.expand else 0)


def error_string(status: int) -> str:
    return _lib.lh_error_string(status).decode()


def _check(rc: int, where: str) -> None:
    if rc != LH_OK:
        raise LighthouseError(rc, where)


def lh_validate(P: Params) -> int:
    return _lib.lh_validate(ctypes.byref(P.c()))


def lh_S(P: Params) -> int:
    return _lib.lh_S(ctypes.byref(P.c()))


def lh_level_size(P: Params, level: int) -> int:
    return _lib.lh_level_size(ctypes.byref(P.c()), level)


def lh_level_offset(P: Params, level: int) -> int:
    return _lib.lh_level_offset(ctypes.byref(P.c()), level)


def lh_pyramid_rows(P: Params) -> int:
    return _lib.lh_pyramid_rows(ctypes.byref(P.c()))


def lh_score_rows(P: Params) -> int:
    return _lib.lh_score_rows(ctypes.byref(P.c()))


def lh_slot_rows(P: Params) -> int:
    return _lib.lh_slot_rows(ctypes.byref(P.c()))


def lh_ctx_bytes(P: Params) -> int:
    return _lib.lh_ctx_bytes(ctypes.byref(P.c()))


def lh_workspace_bytes(P: Params) -> int:
    return _lib.lh_workspace_bytes(ctypes.byref(P.c()))


def lh_ctx_layout(P: Params) -> LhCtxLayout:
    out = LhCtxLayout()
    _check(_lib.lh_ctx_layout(ctypes.byref(P.c()), ctypes.byref(out)), "lh_ctx_layout")
    return out


# ------------------------------------------------------------------------------------------------------------
# Device entry points (torch tensors in, torch tensors out)
# ------------------------------------------------------------------------------------------------------------

def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors must be contiguous CUDA tensors")
    return t.data_ptr()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _valid(P: Params, where: str) -> None:
    """Raise the library's own status for invalid or unsupported parameters before sizing any buffer."""
    _check(lh_validate(P), where)


def _typed(t, shape, name, dtype=torch.bfloat16):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


def _bf16(t, shape, name):
    _typed(t, shape, name, torch.bfloat16)


def new_workspace(P: Params, device) -> torch.Tensor:
    return torch.empty(lh_workspace_bytes(P), dtype=torch.uint8, device=device)


def new_ctx(P: Params, device) -> torch.Tensor:
    return torch.empty(lh_ctx_bytes(P), dtype=torch.uint8, device=device)


def ctx_views(P: Params, ctx: torch.Tensor) -> dict:
    """Typed views of the saved-context buffer written by ``lh_forward``."""
    lay = lh_ctx_layout(P)
    S, rows = lh_S(P), P.B * P.H

    def view(off, n, dtype, shape):
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        return ctx[off: off + nbytes].view(dtype).view(*shape)

    g = (P.B, P.H, S, P.d)
    return dict(qg=view(lay.qg, rows * S * P.d, torch.float16, g), kg=view(lay.kg, rows * S * P.d, torch.float16, g),
                vg=view(lay.vg, rows * S * P.d, torch.float16, g), og=view(lay.og, rows * S * P.d, torch.float32, g),
                lse=view(lay.lse, rows * S, torch.float32, (P.B, P.H, S)),
                idx_g=view(lay.idx_g, rows * S, torch.int32, (P.B, P.H, S)),
                slot=view(lay.slot, rows * lh_slot_rows(P), torch.int32, (P.B, P.H, lh_slot_rows(P))))


def lh_pool(P: Params, x, pyr=None):
    _valid(P, "lh_pool")
    _bf16(x, (P.B, P.H, P.N, P.d), "x")
    if pyr is None:
        pyr = torch.empty((P.B, P.H, lh_pyramid_rows(P), P.d), dtype=torch.bfloat16, device=x.device)
    _check(_lib.lh_pool(ctypes.byref(P.c()), _ptr(x), _ptr(pyr), _stream(x.device)), "lh_pool")
    return pyr


def lh_score_topk(P: Params, k, scores_in=None, scores_out=None, idx_g=None, slot=None, ws=None):
    _valid(P, "lh_score_topk")
    dev = k.device
    _bf16(k, (P.B, P.H, P.N, P.d), "k")
    if idx_g is None:
        idx_g = torch.empty((P.B, P.H, lh_S(P)), dtype=torch.int32, device=dev)
    if slot is None:
        slot = torch.empty((P.B, P.H, lh_slot_rows(P)), dtype=torch.int32, device=dev)
    if ws is None:
        ws = new_workspace(P, dev)
    for t in (scores_in, scores_out):
        if t is not None and (t.dtype != torch.float32 or tuple(t.shape) != (P.B, P.H, lh_score_rows(P))):
            raise ValueError("scores must be fp32 [B, H, lh_score_rows]")
    rc = _lib.lh_score_topk(ctypes.byref(P.c()), _ptr(k), _ptr(scores_in), _ptr(scores_out), _ptr(idx_g), _ptr(slot),
                            _ptr(ws), ws.numel(), _stream(dev))
    _check(rc, "lh_score_topk")
    return idx_g, slot


def lh_gather(P: Params, q, k, v, q_pyr, k_pyr, v_pyr, idx_g, out=None):
    _valid(P, "lh_gather")
    dev = q.device
    S = lh_S(P)
    if out is None:
        out = tuple(torch.empty((P.B, P.H, S, P.d), dtype=torch.float16, device=dev) for _ in range(3))
    qg, kg, vg = out
    rc = _lib.lh_gather(ctypes.byref(P.c()), _ptr(q), _ptr(k), _ptr(v), _ptr(q_pyr), _ptr(k_pyr), _ptr(v_pyr),
                        _ptr(idx_g), _ptr(qg), _ptr(kg), _ptr(vg), _stream(dev))
    _check(rc, "lh_gather")
    return qg, kg, vg


def lh_attend(P: Params, qg, kg, vg, og=None, lse=None):
    _valid(P, "lh_attend")
    dev = qg.device
    S = lh_S(P)
    for t, n in ((qg, "qg"), (kg, "kg"), (vg, "vg")):
        _typed(t, (P.B, P.H, S, P.d), n, torch.float16)
    if og is None:
        og = torch.empty(qg.shape, dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((P.B, P.H, S), dtype=torch.float32, device=dev)
    _check(_lib.lh_attend(ctypes.byref(P.c()), _ptr(qg), _ptr(kg), _ptr(vg), _ptr(og), _ptr(lse), _stream(dev)),
           "lh_attend")
    return og, lse


def lh_scatter(P: Params, og, slot, o=None):
    _valid(P, "lh_scatter")
    dev = og.device
    if o is None:
        o = torch.empty((P.B, P.H, P.N, P.d), dtype=torch.bfloat16, device=dev)
    _check(_lib.lh_scatter(ctypes.byref(P.c()), _ptr(og), _ptr(slot), _ptr(o), _stream(dev)), "lh_scatter")
    return o


def lh_forward(P: Params, q, k, v, o=None, ctx=None, ws=None):
    _valid(P, "lh_forward")
    dev = q.device
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _bf16(t, (P.B, P.H, P.N, P.d), n)
    if o is None:
        o = torch.empty_like(q)
    if ctx is None:
        ctx = new_ctx(P, dev)
    if ws is None:
        ws = new_workspace(P, dev)
    rc = _lib.lh_forward(ctypes.byref(P.c()), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(ctx), _ptr(ws), ws.numel(),
                         _stream(dev))
    _check(rc, "lh_forward")
    return o, ctx


def lh_backward(P: Params, dout, ctx, dq=None, dk=None, dv=None, ws=None):
    _valid(P, "lh_backward")
    dev = dout.device
    _bf16(dout, (P.B, P.H, P.N, P.d), "dout")
    dq = torch.empty_like(dout) if dq is None else dq
    dk = torch.empty_like(dout) if dk is None else dk
    dv = torch.empty_like(dout) if dv is None else dv
    if ws is None:
        ws = new_workspace(P, dev)
    rc = _lib.lh_backward(ctypes.byref(P.c()), _ptr(dout), _ptr(ctx), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
                          ws.numel(), _stream(dev))
    _check(rc, "lh_backward")
    return dq, dk, dv


# ------------------------------------------------------------------------------------------------------------
# Host-resident step (host tensors in, host tensors out; the copies are pipelined inside the library)
# ------------------------------------------------------------------------------------------------------------

_copy_streams: dict = {}


def default_heads_per_chunk(P: Params) -> int:
    """The largest divisor of H that still gives at least sixteen chunks per batch row (one head when H < 16): the
    first chunk's host-to-device copy and the last chunk's device-to-host copy are not overlapped, so small chunks
    pay less for them."""
    best = 1
    for hc in range(1, P.H + 1):
        if P.H % hc == 0 and P.H // hc >= 16:
            best = hc
    return best


def lh_step_host_bytes(P: Params, heads_per_chunk: int) -> int:
    return _lib.lh_step_host_bytes(ctypes.byref(P.c()), int(heads_per_chunk))


def _host_bf16(t, shape, name):
    _typed(t, shape, name, torch.bfloat16)
    if t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous host (CPU) tensor")
    return t.data_ptr()


def lh_step_host(P: Params, q, k, v, dout, o=None, dq=None, dk=None, dv=None, heads_per_chunk=None, dev_buf=None,
                 device=None):
    """lh_forward + lh_backward on HOST bf16 tensors [B,H,N,d] (page-locked for overlap), returning host (o, dq, dk,
    dv).  Runs on `device` (default: the current CUDA device): the compute on its current stream, the copies on two
    streams of this module; returns once everything is enqueued (synchronise the current stream before reading the
    outputs, and keep the input tensors alive until then: the library copies from them asynchronously)."""
    _valid(P, "lh_step_host")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    hc = default_heads_per_chunk(P) if heads_per_chunk is None else int(heads_per_chunk)
    shape = (P.B, P.H, P.N, P.d)
    ins = [_host_bf16(t, shape, n) for t, n in ((q, "q"), (k, "k"), (v, "v"), (dout, "dout"))]
    outs = []
    for t, n in ((o, "o"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        outs.append(torch.empty(shape, dtype=torch.bfloat16, pin_memory=True) if t is None else t)
    out_ptrs = [_host_bf16(t, shape, n) for t, n in zip(outs, ("o", "dq", "dk", "dv"))]
    need = lh_step_host_bytes(P, hc)
    if need == 0:
        raise LighthouseError(LH_ERR_INVALID_ARG, "lh_step_host_bytes")
    if dev_buf is None:
        dev_buf = torch.empty(need, dtype=torch.uint8, device=dev)
    if dev_buf.device != dev:
        raise ValueError("dev_buf must live on the step's device")
    key = dev.index
    if key not in _copy_streams:
        _copy_streams[key] = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
    h2d, d2h = _copy_streams[key]
    with torch.cuda.device(dev):
        rc = _lib.lh_step_host(ctypes.byref(P.c()), *ins, *out_ptrs, hc, _ptr(dev_buf), dev_buf.numel(),
                               torch.cuda.current_stream(dev).cuda_stream, h2d.cuda_stream, d2h.cuda_stream)
    _check(rc, "lh_step_host")
    return tuple(outs)


def lh_scatter_bwd(P: Params, dout, idx_g, dog=None):
    _valid(P, "lh_scatter_bwd")
    dev = dout.device
    if dog is None:
        dog = torch.empty((P.B, P.H, lh_S(P), P.d), dtype=torch.float32, device=dev)
    _check(_lib.lh_scatter_bwd(ctypes.byref(P.c()), _ptr(dout), _ptr(idx_g), _ptr(dog), _stream(dev)),
           "lh_scatter_bwd")
    return dog


def lh_attend_bwd(P: Params, qg, kg, vg, og, lse, dog, ws=None):
    _valid(P, "lh_attend_bwd")
    dev = qg.device
    S = lh_S(P)
    for t, n in ((qg, "qg"), (kg, "kg"), (vg, "vg")):
        _typed(t, (P.B, P.H, S, P.d), n, torch.float16)
    for t, n in ((og, "og"), (dog, "dog")):
        _typed(t, (P.B, P.H, S, P.d), n, torch.float32)
    dqg = torch.empty(qg.shape, dtype=torch.float32, device=dev)
    dkg = torch.empty(qg.shape, dtype=torch.float32, device=dev)
    dvg = torch.empty(qg.shape, dtype=torch.float32, device=dev)
    if ws is None:
        ws = new_workspace(P, dev)
    rc = _lib.lh_attend_bwd(ctypes.byref(P.c()), _ptr(qg), _ptr(kg), _ptr(vg), _ptr(og), _ptr(lse), _ptr(dog),
                            _ptr(dqg), _ptr(dkg), _ptr(dvg), _ptr(ws), ws.numel(), _stream(dev))
    _check(rc, "lh_attend_bwd")
    return dqg, dkg, dvg


def lh_get_status(device=None) -> int:
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    return _lib.lh_get_status(_stream(dev))


def lh_set_wait_limit_ns(ns: int, device=None) -> None:
    """Bound on every device-side wait of later launches on ``device`` (0 restores the default of 2 s)."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        _check(_lib.lh_set_wait_limit_ns(int(ns)), "lh_set_wait_limit_ns")


def lh_profile_enable(on: bool = True) -> None:
    _check(_lib.lh_profile_enable(1 if on else 0), "lh_profile_enable")


def lh_profile_read() -> dict:
    """``{kernel name: (launches, summed device ms)}`` since the last read; clears the record."""
    buf = (LhKernelTime * 64)()
    n = _lib.lh_profile_read(buf, 64)
    if n < 0:
        raise LighthouseError(-n, "lh_profile_read")
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].ms)) for i in range(n)}


LH_STATIC_SCRATCH_BYTES = 16 << 20


def lh_score_topk_static(P: Params, k, scores_in=None, scores_out=None, idx_g=None, slot=None):
    """``lh_score_topk`` without a caller workspace: the library's fixed device scratch array is used instead
    (for callers that cannot allocate device memory where they select).  Output buffers are created here only
    for convenience when not given; the library call itself allocates nothing."""
    _valid(P, "lh_score_topk_static")
    dev = k.device
    _bf16(k, (P.B, P.H, P.N, P.d), "k")
    if idx_g is None:
        idx_g = torch.empty((P.B, P.H, lh_S(P)), dtype=torch.int32, device=dev)
    if slot is None:
        slot = torch.empty((P.B, P.H, lh_slot_rows(P)), dtype=torch.int32, device=dev)
    rc = _lib.lh_score_topk_static(ctypes.byref(P.c()), _ptr(k), _ptr(scores_in), _ptr(scores_out), _ptr(idx_g),
                                   _ptr(slot), _stream(dev))
    _check(rc, "lh_score_topk_static")
    return idx_g, slot
