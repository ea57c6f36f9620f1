"""Helpers shared by the GPU parity tests: conversions between torch tensors and the oracle's float64 arrays, and
the elementwise tolerance of the layer's floating-point outputs."""

from __future__ import annotations

import numpy as np
import torch

ATOL = 2e-2
RTOL = 2e-2


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a bf16/fp32 tensor."""
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def assert_close(got, ref, atol=ATOL, rtol=RTOL, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = ~(err <= bound)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err - bound, -np.inf)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements outside |d| <= {atol} + {rtol}|ref|; "
                             f"worst at {i}: got {got[i]!r}, ref {ref[i]!r}")
