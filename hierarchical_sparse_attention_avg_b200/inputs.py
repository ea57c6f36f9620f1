"""Seeded synthetic inputs for the Lighthouse layer.

This module only draws random numbers; it holds none of the layer's arithmetic.  Both the CUDA path's tests and
benchmark and the CPU oracle's tests take their inputs from here, so both sides see the same bytes.

Recipe (the value distributions of the long-context configurations): every token row of Q, K and V is
``bf16(s * z)`` with ``z ~ N(0, 1)^d`` and one factor ``s = exp(0.5 * n)``, ``n ~ N(0, 1)`` (lognormal(0, 0.5)) per
row; the upstream gradient is ``bf16(N(0, 1))``.  Draws come from one ``torch.Generator`` seeded with ``seed`` on the
requested device, in the order Q, K, V, dO.  CPU and CUDA generators give different (but each reproducible) bytes.
"""

from __future__ import annotations

import torch


def _generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _scaled_rows(shape, g, device) -> torch.Tensor:
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    n = torch.randn(shape[:-1] + (1,), generator=g, device=device, dtype=torch.float32)
    z.mul_(torch.exp(0.5 * n))
    return z.to(torch.bfloat16)


def make_inputs(B: int, H: int, N: int, d: int, seed: int = 0, device="cpu", with_grad: bool = True):
    """Return ``(q, k, v, dout)`` bf16 tensors of shape ``[B, H, N, d]`` (``dout`` is None without grad)."""
    g = _generator(seed, device)
    shape = (B, H, N, d)
    q = _scaled_rows(shape, g, device)
    k = _scaled_rows(shape, g, device)
    v = _scaled_rows(shape, g, device)
    dout = None
    if with_grad:
        dout = torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    return q, k, v, dout


def make_scores(B: int, H: int, rows: int, seed: int = 0, device="cpu", ties: bool = False,
                signed: bool = False) -> torch.Tensor:
    """fp32 scores ``[B, H, rows]`` for feeding the top-K step directly: non-negative by default.

    With ``ties=True`` the values are drawn from a small set so that many scores are equal, which exercises the
    lower-index tie rule.  With ``signed=True`` they are N(0, 1) values of both signs, about one in eight replaced
    by a zero of random sign (so that -0 meets +0) and one in eight by a value repeated across the row."""
    g = _generator(seed, device)
    if ties:
        return torch.randint(0, 4, (B, H, rows), generator=g, device=device).to(torch.float32)
    z = torch.randn((B, H, rows), generator=g, device=device, dtype=torch.float32)
    if signed:
        u = torch.rand((B, H, rows), generator=g, device=device)
        sign = torch.randint(0, 2, (B, H, rows), generator=g, device=device).to(torch.float32) * 2 - 1
        z = torch.where(u < 0.125, sign * 0.0, z)
        z = torch.where((u >= 0.125) & (u < 0.25), torch.full_like(z, -0.75), z)
        return z
    return z * z


def make_hard_inputs(B: int, H: int, N: int, d: int, seed: int = 0, device="cpu", emin: int = -140, emax: int = 3):
    """``(q, k, v)`` bf16 tensors ``[B, H, N, d]`` whose values stress exact summation and the number formats.

    Every value is ``sign * (1 + m/128) * 2^e`` with a random sign, a random 7-bit ``m`` and an exponent ``e``
    drawn per element from ``[emin, emax]`` in half of the rows, and from a three-wide band at a random height in the
    other half (so whole pooled entries can be tiny, with sums in the subnormal range); about one value in eight is a
    zero of either sign.  Values below 2^-126 become bf16 subnormals (or zero) in the final rounding to bf16.  The
    default range keeps every value below 16, inside the fp16 range of the attention operands."""
    g = _generator(seed, device)
    shape = (B, H, N, d)
    rows = shape[:-1] + (1,)

    def one():
        sign = torch.randint(0, 2, shape, generator=g, device=device).to(torch.float64) * 2 - 1
        mant = 1 + torch.randint(0, 128, shape, generator=g, device=device).to(torch.float64) / 128
        e_elem = torch.randint(emin, emax + 1, shape, generator=g, device=device)
        e_band = (torch.randint(emin + 2, emax + 1, rows, generator=g, device=device)
                  - torch.randint(0, 3, shape, generator=g, device=device))
        banded = torch.rand(rows, generator=g, device=device) < 0.5
        e = torch.where(banded, e_band, e_elem).to(torch.float64)
        zero = torch.rand(shape, generator=g, device=device) < 0.125
        x = sign * torch.where(zero, torch.zeros_like(mant), mant * torch.exp2(e))
        return x.to(torch.float32).to(torch.bfloat16)

    return one(), one(), one()
