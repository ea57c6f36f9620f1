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
    # children-expansion variant: the pages' size example at N = 2^20, the 4K case, a whole-level case
    (1, 8, 1048576, 128, 4, 4, 4096, 32, True),
    (1, 2, 4096, 64, 3, 4, 64, 4, True),
    (1, 1, 1024, 64, 3, 4, 64, 4, True),
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
    assert lh.lh_score_rows(P) == Q.score_rows()
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


def test_expand_variant_sizes_and_validation(lh):
    P = lh.Params(1, 8, 1048576, 128, 4, 4, 4096, 32, True)
    assert lh.lh_S(P) == 65536                                   # 16,384 coarsest + 3 levels x 4 x 4,096
    assert lh.lh_score_rows(P) == 262144 + 65536 + 16384          # levels 1..3 scored
    assert lh.lh_validate(lh.Params(1, 1, 4096, 64, 3, 4, 64, 3, True)) == lh.LH_ERR_INVALID_ARG  # 3 does not divide
    import ctypes as C
    bad = lh.Params(1, 1, 4096, 64, 3, 4, 64, 4).c()
    bad.flags = 2                                                # an unknown flag bit
    assert lh.library().lh_validate(C.byref(bad)) == lh.LH_ERR_INVALID_ARG


def test_k_at_least_level_size_needs_no_divisibility(lh):
    P = lh.Params(1, 1, 2048, 64, 4, 4, 2048, 16)  # level 0 whole (k = N), level 1..: whole
    assert lh.lh_validate(P) == lh.LH_OK
    assert lh.lh_S(P) == 2048 + 512 + 128 + 32


def test_error_strings(lh):
    for code in range(7):
        assert lh.error_string(code)
    assert lh.error_string(99) == "unknown status"


def test_step_host_bytes_and_argument_errors(lh):
    """lh_step_host sizing and the errors it returns on the host, before any CUDA call."""
    P = lh.Params(2, 4, 4096, 64, 3, 4, 256, 8)
    Pc = lh.Params(1, 2, 4096, 64, 3, 4, 256, 8)
    tensor = 2 * 4096 * 64 * 2  # one chunk tensor of two heads, bf16
    need = lh.lh_step_host_bytes(P, 2)
    rnd = lambda x: (x + 255) // 256 * 256
    assert need == 3 * 8 * rnd(tensor) + rnd(lh.lh_ctx_bytes(Pc)) + rnd(lh.lh_workspace_bytes(Pc))
    assert lh.lh_step_host_bytes(P, 3) == 0  # does not divide H
    assert lh.lh_step_host_bytes(P, 0) == 0
    bad = lh.Params(1, 2, 4100, 64, 3, 4, 256, 8)  # p^(L-1) = 16 does not divide N
    assert lh.lh_validate(bad) != 0 and lh.lh_step_host_bytes(bad, 1) == 0
    assert lh.default_heads_per_chunk(lh.Params(1, 16, 524288, 128, 4, 4, 4096, 32)) == 1
    assert lh.default_heads_per_chunk(lh.Params(1, 64, 4096, 64, 3, 4, 256, 8)) == 4
    assert lh.default_heads_per_chunk(lh.Params(1, 2, 4096, 64, 3, 4, 256, 8)) == 1

    lib = lh.library()
    buf = (ctypes.c_uint8 * 64)()
    p = ctypes.addressof(buf)
    c = P.c()
    call = lambda hc, dev, nbytes, ptr=p: lib.lh_step_host(ctypes.byref(c), ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, hc,
                                                           dev, nbytes, None, None, None)
    assert call(3, 256, 1 << 40) == lh.LH_ERR_INVALID_ARG           # heads_per_chunk does not divide H
    assert call(2, None, 1 << 40) == lh.LH_ERR_INVALID_ARG          # no device buffer
    assert call(2, 256 + 16, 1 << 40) == lh.LH_ERR_INVALID_ARG      # misaligned device buffer
    assert call(2, 256, need - 1) == lh.LH_ERR_WORKSPACE            # device buffer too small
    assert call(2, 256, 1 << 40, ptr=None) == lh.LH_ERR_INVALID_ARG  # NULL host tensor
