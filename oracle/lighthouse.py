"""CPU oracle of the Lighthouse selection-and-attend layer (forward and backward).

TEST INFRASTRUCTURE ONLY.  This module is the slow, plain reference that the CUDA path is checked against.
Only the tests, the package's ``smoke()`` entry and the benchmark's CPU-baseline leg may import it; the product
path never calls it and has no CPU fallback.  It shares no code with the CUDA path.

Arithmetic is numpy float64 throughout, except the two roundings the layer's definition fixes: pooled values are
rounded to bf16 and scores to fp32.  One head ``(b, h)`` is processed at a time; heads are independent.

Sources (web pages about Nous Research's Lighthouse Attention), cited by short name:

* [W]  wispaper.ai, "Lighthouse Attention：预训练长文本的高速公路，训练提速 21 倍且无损恢复"
* [E]  encorp.ai, "Услуги по внедряване на AI задават правилния въпрос за Lighthouse Attention"
* [C]  clawdbytes.com, "Lighthouse Attention: the training-time hierarchy that makes quadratic attention …"
* [H]  news.hamidun.com, "Nous Research introduced Lighthouse Attention to accelerate LLM training"

The pages give the method in prose only.  Where they are silent this oracle takes the readings named in each
docstring ("reading: ..."); the same readings are written down in the project's specification.

Parity status: every function below is pinned by a test under ``tests/test_oracle_*.py`` against something other
than itself (exact rational arithmetic, a textbook loop, brute force, finite differences).
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np


# --------------------------------------------------------------------------------------------------------------
# Parameters and sizes
# --------------------------------------------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Params:
    """Layer parameters.

    ``L`` pyramid levels (level 0 = raw tokens), pool factor ``p``, ``k`` picks per level and ``C`` chunks per
    level ([E] "Как four-stage pipeline…": pyramid of several levels, per-level chunked-bitonic top-K;
    [C] "Four-Stage Pipeline…")."""

    B: int
    H: int
    N: int
    d: int
    L: int
    p: int
    k: int
    C: int
    expand: bool = False

    def window(self, lev: int) -> int:
        """Tokens covered by one entry of level ``lev``: ``p**lev``."""
        return self.p ** lev

    def level_size(self, lev: int) -> int:
        """Entries of level ``lev``: ``N / p**lev``."""
        return self.N // self.window(lev)

    def picks(self, lev: int) -> int:
        """Entries kept at level ``lev``: ``min(k, N_lev)`` below the coarsest level, all of the coarsest.

        Reading: "top-K per level" with the coarsest level "always retained in full" ([C] "Four-Stage
        Pipeline…").  With ``expand`` (the children-expansion variant): ``p * min(k, N_{lev+1})`` below the
        coarsest level, the children of the entries picked one level up."""
        if lev == self.L - 1:
            return self.level_size(lev)
        if self.expand:
            return self.p * self.parent_picks(lev + 1)
        return min(self.k, self.level_size(lev))

    def parent_picks(self, lev: int) -> int:
        """Children-expansion variant: entries of level ``lev`` (1 .. L-1) picked by score, ``min(k, N_lev)``."""
        return min(self.k, self.level_size(lev))

    def scored_levels(self) -> list[int]:
        """Levels whose pooled keys are scored: ``0 .. L-2``, or ``1 .. L-1`` in the children-expansion variant."""
        return list(range(1, self.L)) if self.expand else list(range(self.L - 1))

    def gathered_length(self) -> int:
        """``S = sum_{lev <= L-2} min(k, N_lev) + N_{L-1}`` (reading R-S), or, in the children-expansion variant,
        ``S = sum_{lev=1}^{L-1} p * min(k, N_lev) + N_{L-1}``."""
        return sum(self.picks(lev) for lev in range(self.L))

    def score_rows(self) -> int:
        """Rows of one head's score array: the scored levels concatenated, finest first."""
        return sum(self.level_size(x) for x in self.scored_levels())

    def score_offset(self, lev: int) -> int:
        """Row of scored level ``lev``'s first entry in one head's score array."""
        return sum(self.level_size(x) for x in self.scored_levels() if x < lev)

    def level_offset(self, lev: int) -> int:
        """Global pyramid id of entry ``(lev, 0)``: number of entries of all finer levels."""
        return sum(self.level_size(x) for x in range(lev))

    def validate(self) -> None:
        if min(self.B, self.H, self.N, self.d, self.L, self.k, self.C) < 1 or self.p < 2:
            raise ValueError("sizes must be positive and p >= 2")
        if self.N % self.window(self.L - 1):
            raise ValueError("p**(L-1) must divide N")
        if self.d % 8 or (self.d // 8) & (self.d // 8 - 1):
            raise ValueError("d must be 8 times a power of two (score summation order)")
        for lev in range(self.L - 1):
            if self.expand:
                n, kk = self.level_size(lev + 1), self.parent_picks(lev + 1)
            else:
                n, kk = self.level_size(lev), self.picks(lev)
            if kk == n:
                continue
            if n % self.C or kk % self.C:
                raise ValueError(f"C must divide the entries and the picks of every partially picked level")


# --------------------------------------------------------------------------------------------------------------
# Rounding to the storage formats the definition fixes
# --------------------------------------------------------------------------------------------------------------

_BF16_MIN_NORMAL_EXP = -126      # smallest normal binade of bf16 (same exponent range as fp32)
_BF16_FRACTION_BITS = 7


def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 value, ties to even; returns float64 holding bf16 values.

    Done by scaling to the bf16 quantum of each value's binade (an exact power-of-two scaling), rounding to an
    integer with ``np.rint`` (round half to even) and scaling back.  Magnitudes that round to 2**128 or beyond
    become infinities.  NaN is passed through."""
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, copy=True)
    finite = np.isfinite(x) & (x != 0)
    xf = x[finite]
    _, e = np.frexp(xf)                               # |xf| = m * 2**e, m in [0.5, 1)
    binade = np.maximum(e - 1, _BF16_MIN_NORMAL_EXP)  # subnormals share the smallest normal quantum
    quantum_exp = binade - _BF16_FRACTION_BITS
    r = np.ldexp(np.rint(np.ldexp(xf, -quantum_exp)), quantum_exp)
    r = np.where(np.abs(r) >= 2.0 ** 128, np.copysign(np.inf, r), r)
    out[finite] = r
    return out


def bf16_bits(x) -> np.ndarray:
    """uint16 bit patterns of float64 values that are already bf16 values (e.g. ``bf16_round`` output)."""
    f32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    return (f32.view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(bits) -> np.ndarray:
    """float64 values of uint16 bf16 bit patterns (exact)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def fp32_round(x) -> np.ndarray:
    """IEEE round-to-nearest-even conversion of float64 to float32 (numpy's cast)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


# --------------------------------------------------------------------------------------------------------------
# Step 1: symmetric average-pool pyramid
# --------------------------------------------------------------------------------------------------------------

def pool_sums(x: np.ndarray, P: Params) -> list[np.ndarray]:
    """fp64 block sums of one head's rows ``x`` ``[N, d]`` for every level.

    Level 0 is ``x`` itself; level ``lev`` sums the ``p`` children of level ``lev-1`` left to right, starting
    from the first child (reading P1 of the layer's specification; [W] 核心方法 §1 对称金字塔池化: Q, K and V are
    average-pooled alike into a multi-level pyramid)."""
    sums = [np.asarray(x, dtype=np.float64)]
    for lev in range(1, P.L):
        children = sums[-1].reshape(P.level_size(lev), P.p, P.d)
        acc = children[:, 0, :].copy()
        for c in range(1, P.p):
            acc = acc + children[:, c, :]
        sums.append(acc)
    return sums


def pyramid(x: np.ndarray, P: Params, round_pool: bool = True) -> list[np.ndarray]:
    """Pooled values of every level: level 0 = ``x``; level ``lev`` = ``bf16_RN(sum / p**lev)``.

    With ``round_pool=False`` the bf16 rounding is skipped (used only by the finite-difference test, where the
    rounding would make the function piecewise constant)."""
    sums = pool_sums(x, P)
    levels = [sums[0]]
    for lev in range(1, P.L):
        mean = sums[lev] / float(P.window(lev))
        levels.append(bf16_round(mean) if round_pool else mean)
    return levels


# --------------------------------------------------------------------------------------------------------------
# Step 2: parameter-free per-head l2-norm score
# --------------------------------------------------------------------------------------------------------------

def norm_scores(kpyr: list[np.ndarray], P: Params) -> list[np.ndarray]:
    """Squared l2 norm of every pooled key of the scored levels (``P.scored_levels()``), as float32.

    [W] 核心方法 §2 and [E] "Как four-stage pipeline…" score entries with a parameter-free per-head l2 norm.
    Reading P2: the norm of the pooled key, squared (same order as the norm).  Summation order: eight squares
    left to right per group of eight features, then a pairwise tree over the groups; one rounding to fp32."""
    out = []
    for lev in P.scored_levels():
        sq = kpyr[lev] * kpyr[lev]                      # exact in float64 (16-bit significands)
        groups = sq.reshape(sq.shape[0], P.d // 8, 8)
        part = groups[:, :, 0].copy()
        for i in range(1, 8):
            part = part + groups[:, :, i]
        while part.shape[1] > 1:
            part = part[:, 0::2] + part[:, 1::2]
        out.append(fp32_round(part[:, 0]))
    return out


# --------------------------------------------------------------------------------------------------------------
# Step 3: stratified (chunked) top-K per level, coarsest level kept whole
# --------------------------------------------------------------------------------------------------------------

def chunked_top(s: np.ndarray, picks: int, P: Params) -> np.ndarray:
    """Indices, ascending, of the ``picks`` entries of largest score of one level split into ``C`` equal
    contiguous chunks, ``picks / C`` from each chunk, ties to the lower index (found by sorting each chunk)."""
    s = np.asarray(s, dtype=np.float64)
    n = len(s)
    n_c, m = n // P.C, picks // P.C
    chosen = []
    for c in range(P.C):
        j = np.arange(c * n_c, (c + 1) * n_c, dtype=np.int64)
        order = np.lexsort((j, -s[j]))             # primary: score descending; secondary: index ascending
        chosen.append(np.sort(j[order[:m]]))
    return np.concatenate(chosen)


def select(scores: list[np.ndarray], P: Params) -> list[np.ndarray]:
    """Selected entry indices of every level, ascending.  ``scores[i]`` belongs to level ``P.scored_levels()[i]``.

    Levels ``0 .. L-2``: ``C`` equal contiguous chunks, each keeping its ``k_lev / C`` entries with the largest
    score, ties to the lower index, found by sorting each chunk ([W] 核心方法 §2 "Chunked Bitonic Top-K";
    [C] "Four-Stage Pipeline…": stratified rather than global top-K).  When ``k >= N_lev`` the whole level is
    kept.  The coarsest level is always kept whole ([C] "Four-Stage Pipeline…").

    Children-expansion variant (``P.expand``; the reading under which the size example of [E] "Какво точно
    промени Nous Research в attention пътя?" comes out): the chunked top-K runs on the scored levels
    ``1 .. L-1``, and level ``lev <= L-2`` keeps the ``p`` children ``p*J .. p*J + p-1`` of every entry ``J``
    picked at level ``lev + 1``; the coarsest level is still kept whole."""
    if P.expand:
        sel = []
        for lev in range(P.L - 1):
            parent = lev + 1
            n_par = P.level_size(parent)
            if P.parent_picks(parent) == n_par:
                sel.append(np.arange(P.level_size(lev), dtype=np.int64))
                continue
            J = chunked_top(scores[parent - 1], P.parent_picks(parent), P)
            kids = (J[:, None] * P.p + np.arange(P.p, dtype=np.int64)[None, :]).reshape(-1)
            sel.append(kids)
        sel.append(np.arange(P.level_size(P.L - 1), dtype=np.int64))
        return sel
    sel = []
    for lev in range(P.L):
        n = P.level_size(lev)
        if lev == P.L - 1 or P.picks(lev) == n:
            sel.append(np.arange(n, dtype=np.int64))
            continue
        sel.append(chunked_top(scores[lev], P.picks(lev), P))
    return sel


# --------------------------------------------------------------------------------------------------------------
# Step 4a: gathered order and slot maps
# --------------------------------------------------------------------------------------------------------------

def gathered_order(sel: list[np.ndarray], P: Params):
    """Order the selected entries into one position-ordered sequence.

    Reading P4: ascending end token ``E = (j+1)*p**lev - 1``; equal ends go coarser level first.  Returns
    ``(lev_g, j_g, slots)`` where ``lev_g[s], j_g[s]`` name the entry at gathered position ``s`` and
    ``slots[lev][j]`` is that position or -1 ([W] 核心方法 §3: the selected entries form a dense, causality
    preserving subsequence)."""
    levs = np.concatenate([np.full(len(sel[lev]), lev, dtype=np.int64) for lev in range(P.L)])
    js = np.concatenate(sel)
    ends = (js + 1) * (np.int64(P.p) ** levs) - 1
    order = np.lexsort((-levs, ends))
    lev_g, j_g = levs[order], js[order]
    slots = [np.full(P.level_size(lev), -1, dtype=np.int64) for lev in range(P.L)]
    for s, (lev, j) in enumerate(zip(lev_g.tolist(), j_g.tolist())):
        slots[lev][j] = s
    return lev_g, j_g, slots


def global_ids(lev_g: np.ndarray, j_g: np.ndarray, P: Params) -> np.ndarray:
    """Global pyramid id ``off_lev + j`` (levels concatenated finest first)."""
    offs = np.array([P.level_offset(lev) for lev in range(P.L)], dtype=np.int64)
    return offs[lev_g] + j_g


def gather(pyr: list[np.ndarray], lev_g: np.ndarray, j_g: np.ndarray) -> np.ndarray:
    """Rows of the gathered sequence: row ``s`` is ``pyr[lev_g[s]][j_g[s]]``."""
    d = pyr[0].shape[1]
    out = np.empty((len(lev_g), d), dtype=np.float64)
    for lev, level in enumerate(pyr):
        m = lev_g == lev
        out[m] = level[j_g[m]]
    return out


# --------------------------------------------------------------------------------------------------------------
# Step 4b: dense causal attention over the gathered sequence
# --------------------------------------------------------------------------------------------------------------

def _above_diagonal(S: int) -> np.ndarray:
    """Boolean ``[S, S]`` mask of the entries ``b > a`` (key after query)."""
    idx = np.arange(S)
    return idx[None, :] > idx[:, None]


def causal_attention(qg: np.ndarray, kg: np.ndarray, vg: np.ndarray):
    """``softmax(Q K^T / sqrt(d) + causal mask) V`` and the natural-log row LSE, in float64.

    Standard scaled-dot-product attention with the diagonal included ([W] 核心方法 §3 标准 FlashAttention 调用;
    [H] "How Lighthouse Attention Works")."""
    S, d = qg.shape
    logits = (qg @ kg.T) / math.sqrt(d)
    np.putmask(logits, _above_diagonal(S), -np.inf)
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    lsum = e.sum(axis=1, keepdims=True)
    prob = e / lsum
    og = prob @ vg
    lse = (mx + np.log(lsum))[:, 0]
    return og, lse


def causal_attention_backward(qg, kg, vg, og, lse, dog):
    """Gradients of ``causal_attention`` w.r.t. its three inputs (textbook softmax backward), float64."""
    S, d = qg.shape
    scale = 1.0 / math.sqrt(d)
    logits = (qg @ kg.T) * scale
    np.putmask(logits, _above_diagonal(S), -np.inf)
    prob = np.exp(logits - lse[:, None])
    dvg = prob.T @ dog
    dprob = dog @ vg.T
    delta = (dog * og).sum(axis=1, keepdims=True)
    dlogits = prob * (dprob - delta)
    dqg = (dlogits @ kg) * scale
    dkg = (dlogits.T @ qg) * scale
    return dqg, dkg, dvg


# --------------------------------------------------------------------------------------------------------------
# Step 5: causality-preserving offset scatter-back, and the two backward-only steps
# --------------------------------------------------------------------------------------------------------------

def scatter(og: np.ndarray, slots: list[np.ndarray], P: Params) -> np.ndarray:
    """Token outputs: ``O[t] = sum_lev O_g[slot_lev(floor((t+1)/p**lev) - 1)]`` over selected entries.

    Reading P6 ([W] figure caption: scatter-back; [E] "Как four-stage pipeline…": redistributed to the original
    positions with a causality-preserving offset): entry ``(lev, j)`` writes tokens ``E .. E + p**lev - 1``;
    levels are summed; a token without a selected candidate gets 0."""
    out = np.zeros((P.N, og.shape[1]), dtype=np.float64)
    t = np.arange(P.N, dtype=np.int64)
    for lev in range(P.L):
        j = (t + 1) // P.window(lev) - 1
        ok = (j >= 0) & (j < P.level_size(lev))
        s = np.full(P.N, -1, dtype=np.int64)
        s[ok] = slots[lev][j[ok]]
        ok &= s >= 0
        out[t[ok]] += og[s[ok]]
    return out


def scatter_backward(dout: np.ndarray, lev_g, j_g, P: Params) -> np.ndarray:
    """``dO_g[s] = sum_{t=E}^{min(E+w-1, N-1)} dO[t]`` for the entry at gathered position ``s``."""
    dog = np.zeros((len(lev_g), P.d), dtype=np.float64)
    for lev in range(P.L):
        w = P.window(lev)
        shifted = np.zeros((P.N, P.d), dtype=np.float64)
        shifted[: P.N - (w - 1)] = dout[w - 1:]
        windows = shifted.reshape(P.level_size(lev), w, P.d).sum(axis=1)
        m = lev_g == lev
        dog[m] = windows[j_g[m]]
    return dog


def unpool_backward(dxg: np.ndarray, slots: list[np.ndarray], P: Params) -> np.ndarray:
    """``dX[t] = sum_lev dX_g[slot_lev(floor(t/p**lev))] / p**lev`` over selected entries.

    Gradients reach the inputs only through the gathered values; selection gets none ([E] "Как four-stage
    pipeline…": no straight-through estimator, no Gumbel softmax; [W] 深度洞察)."""
    dx = np.zeros((P.N, dxg.shape[1]), dtype=np.float64)
    t = np.arange(P.N, dtype=np.int64)
    for lev in range(P.L):
        w = P.window(lev)
        s = slots[lev][t // w]
        ok = s >= 0
        dx[t[ok]] += dxg[s[ok]] / float(w)
    return dx


# --------------------------------------------------------------------------------------------------------------
# Whole layer, one head
# --------------------------------------------------------------------------------------------------------------

def forward_head(q, k, v, P: Params, selection=None, round_pool: bool = True) -> dict:
    """Forward of one head.  ``q, k, v``: float64 ``[N, d]`` (bf16 values).

    ``selection`` (a list of per-level index arrays) freezes the selection instead of computing it; used by the
    causality and finite-difference tests."""
    qp = pyramid(q, P, round_pool)
    kp = pyramid(k, P, round_pool)
    vp = pyramid(v, P, round_pool)
    scores = norm_scores(kp, P)
    sel = select(scores, P) if selection is None else selection
    lev_g, j_g, slots = gathered_order(sel, P)
    qg, kg, vg = gather(qp, lev_g, j_g), gather(kp, lev_g, j_g), gather(vp, lev_g, j_g)
    og, lse = causal_attention(qg, kg, vg)
    out = scatter(og, slots, P)
    return dict(pyr_q=qp, pyr_k=kp, pyr_v=vp, scores=scores, sel=sel, lev_g=lev_g, j_g=j_g,
                idx_g=global_ids(lev_g, j_g, P), slots=slots, qg=qg, kg=kg, vg=vg, og=og, lse=lse, out=out)


def backward_head(dout, fwd: dict, P: Params):
    """Gradients of one head's output w.r.t. ``q, k, v`` given the upstream gradient ``dout`` ``[N, d]``."""
    dog = scatter_backward(np.asarray(dout, dtype=np.float64), fwd["lev_g"], fwd["j_g"], P)
    dqg, dkg, dvg = causal_attention_backward(fwd["qg"], fwd["kg"], fwd["vg"], fwd["og"], fwd["lse"], dog)
    slots = fwd["slots"]
    return (unpool_backward(dqg, slots, P), unpool_backward(dkg, slots, P), unpool_backward(dvg, slots, P),
            dog)


def slot_map(slots: list[np.ndarray]) -> np.ndarray:
    """Concatenated slot map over all levels (finest first), as stored by the CUDA path."""
    return np.concatenate(slots)


def forward(q, k, v, P: Params, heads=None) -> dict:
    """Forward over ``[B, H, N, d]`` float64 inputs; returns per-head results keyed by ``(b, h)``."""
    P.validate()
    heads = [(b, h) for b in range(P.B) for h in range(P.H)] if heads is None else heads
    return {(b, h): forward_head(q[b, h], k[b, h], v[b, h], P) for (b, h) in heads}
