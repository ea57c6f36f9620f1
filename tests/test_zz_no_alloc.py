"""GPU test of ``lh_score_topk_static``, the selection entry point that takes no caller workspace.

Who needs it: callers that cannot allocate device memory where they run the selection (a runtime whose device
memory is planned once at start-up, a hook that only receives the tensors it reads and writes).  The entry point
keeps its scratch in a fixed device array of the library, so this test checks, through the C ABI, that two calls
in a row (different shapes, so the second one runs over the first one's leftovers) give exactly what the regular
``lh_score_topk`` gives, and that a call needing more than the array holds is refused before any launch.

This file is collected last, so that a run that stops at the first failure has already run every other test.
"""

from __future__ import annotations

import ctypes

import pytest
import torch

from hierarchical_sparse_attention_avg_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

SHAPES = [
    (1, 2, 4096, 64, 3, 4, 256, 8),      # the 4K configuration
    (2, 3, 8192, 128, 4, 4, 512, 16),    # larger, different level structure
]


def _call_static(lh, P, k, scores_in, scores_out, idx_g, slot):
    """Direct C-ABI call (no Python-side allocation on the path)."""
    dev = k.device
    ptr = lambda t: None if t is None else t.data_ptr()
    return lh.library().lh_score_topk_static(ctypes.byref(P.c()), ptr(k), ptr(scores_in), ptr(scores_out),
                                             ptr(idx_g), ptr(slot), torch.cuda.current_stream(dev).cuda_stream)


def test_static_scratch_selection_matches_workspace_selection(cuda_device):
    from hierarchical_sparse_attention_avg_b200 import lh

    for round_ in range(2):  # the second round reuses the array with the other shape's contents left in it
        for cfg in (SHAPES if round_ == 0 else SHAPES[::-1]):
            P = lh.Params(*cfg)
            _, k, _, _ = make_inputs(P.B, P.H, P.N, P.d, seed=11 + round_, device=cuda_device, with_grad=False)
            want_idx, want_slot = lh.lh_score_topk(P, k)
            want_scores = torch.empty((P.B, P.H, lh.lh_score_rows(P)), dtype=torch.float32, device=cuda_device)
            lh.lh_score_topk(P, k, scores_out=want_scores)

            idx_g = torch.full_like(want_idx, -7)
            slot = torch.full_like(want_slot, -7)
            assert _call_static(lh, P, k, None, None, idx_g, slot) == lh.LH_OK
            assert torch.equal(idx_g, want_idx) and torch.equal(slot, want_slot)

            scores = torch.zeros_like(want_scores)
            idx_g.fill_(-7)
            slot.fill_(-7)
            assert _call_static(lh, P, k, None, scores, idx_g, slot) == lh.LH_OK
            assert torch.equal(scores, want_scores)
            assert torch.equal(idx_g, want_idx) and torch.equal(slot, want_slot)

            idx_g.fill_(-7)
            assert _call_static(lh, P, k, want_scores, None, idx_g, slot) == lh.LH_OK
            assert torch.equal(idx_g, want_idx)
    assert lh.lh_get_status(cuda_device) == lh.LH_OK


def test_static_scratch_rejects_calls_beyond_its_size(cuda_device):
    from hierarchical_sparse_attention_avg_b200 import lh

    # 16 heads x 688128 score rows x 4 bytes is about 44 MB of scores alone: more than the 16 MiB array
    P = lh.Params(1, 16, 524288, 128, 4, 4, 4096, 32)
    k = torch.zeros((1, 1, 8), dtype=torch.bfloat16, device=cuda_device)  # never read: refused before launch
    idx_g = torch.empty(8, dtype=torch.int32, device=cuda_device)
    slot = torch.empty(8, dtype=torch.int32, device=cuda_device)
    assert _call_static(lh, P, k, None, None, idx_g, slot) == lh.LH_ERR_WORKSPACE
    assert lh.lh_get_status(cuda_device) == lh.LH_OK
