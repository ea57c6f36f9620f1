"""C-ABI checks that need no GPU: the library loads, exports every entry point declared in ``include/lh.h``, and its
host-only queries (validation, sizes, layouts) agree with the oracle's definitions.  No compute call is made."""

from __future__ import annotations

import ctypes
import os
import re

import pytest

from oracle import lighthouse as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lh.h")


@pytest.fixture(scope="module")
def lh():
    lib_path = os.path.join(ROOT, "hierarchical_sparse_attention_avg_b200", "liblh.so")
    if not os.path.exists(lib_path):
        from hierarchical_sparse_attention_avg_b200 import build

        build.build()
    from hierarchical_sparse_attention_avg_b200 import lh as mod

    return mod


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lh_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ["lh_pool", "lh_score_topk", "lh_gather", "lh_attend", "lh_scatter", "lh_forward", "lh_backward"]:
        assert must in names


def test_library_exports_every_declared_symbol(lh):
    lib = ctypes.CDLL(lh.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


CONFIGS = [
    (1, 2, 4096, 64, 3, 4, 256, 8),
    (1, 16, 32768, 64, 4, 4, 2048, 16),
    (1, 16, 98304, 64, 4, 4, 2048, 16),
    (1, 16, 524288, 128, 4, 4, 4096, 32),
    (1, 8, 1048576, 128, 4, 4, 4096, 32),
    (2, 3, 1024, 128, 1, 4, 100, 1),
    (1, 1, 512, 64, 5, 2, 8, 2),
]


@pytest.mark.parametrize("cfg", CONFIGS)
def test_sizes_match_oracle(lh, cfg):
    P, Q = lh.Params(*cfg), O.Params(*cfg)
    assert lh.lh_validate(P) == lh.LH_OK
    assert lh.lh_S(P) == Q.gathered_length()
    for lev in range(Q.L):
        assert lh.lh_level_size(P, lev) == Q.level_size(lev)
        assert lh.lh_level_offset(P, lev) == Q.level_offset(lev)
    assert lh.lh_level_size(P, Q.L) == -1
    assert lh.lh_pyramid_rows(P) == sum(Q.level_size(lev) for lev in range(1, Q.L))
    assert lh.lh_score_rows(P) == sum(Q.level_size(lev) for lev in range(Q.L - 1))
    assert lh.lh_slot_rows(P) == sum(Q.level_size(lev) for lev in range(Q.L))
    lay = lh.lh_ctx_layout(P)
    S, rows = Q.gathered_length(), Q.B * Q.H
    offs = [lay.qg, lay.kg, lay.vg, lay.og, lay.lse, lay.idx_g, lay.slot, lay.total]
    assert all(o % 256 == 0 for o in offs) and offs == sorted(offs)
    assert lay.kg - lay.qg >= rows * S * Q.d * 2 and lay.total - lay.slot >= rows * lh.lh_slot_rows(P) * 4
    assert lh.lh_ctx_bytes(P) == lay.total
    assert lh.lh_workspace_bytes(P) >= rows * S * Q.d * 4  # at least the fp32 dQ accumulator


@pytest.mark.parametrize("cfg,code", [
    ((1, 1, 100, 64, 3, 4, 8, 2), 1),       # p^(L-1) does not divide N
    ((1, 1, 4096, 64, 3, 4, 100, 8), 1),    # C does not divide k
    ((1, 1, 4096, 64, 3, 4, 96, 7), 1),     # C does not divide N_l
    ((0, 1, 4096, 64, 3, 4, 256, 8), 1),    # empty batch
    ((1, 1, 4096, 64, 3, 1, 256, 8), 1),    # p < 2
    ((1, 1, 4096, 96, 3, 4, 256, 8), 2),    # head dim not built
    ((1, 1, 4096, 64, 3, 3, 256, 8), 1),    # 9 does not divide 4096
    ((1, 1, 4374, 64, 3, 3, 6, 2), 2),      # p = 3 is valid but not built
    ((1, 1, 65536, 64, 6, 4, 64, 2), 2),    # too many levels for the kernels
    ((1, 1, 65536, 64, 2, 4, 4096, 4), 2),  # 1024 picks per chunk
])
def test_validation_codes(lh, cfg, code):
    assert lh.lh_validate(lh.Params(*cfg)) == code


def test_k_at_least_level_size_needs_no_divisibility(lh):
    P = lh.Params(1, 1, 2048, 64, 4, 4, 2048, 16)  # level 0 whole (k = N), level 1..: whole
    assert lh.lh_validate(P) == lh.LH_OK
    assert lh.lh_S(P) == 2048 + 512 + 128 + 32


def test_error_strings(lh):
    for code in range(7):
        assert lh.error_string(code)
    assert lh.error_string(99) == "unknown status"
