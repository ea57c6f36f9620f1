"""bench.py's reference arm (the oracle timed on the host cores) on the small workload: one JSON line with the same
metric, unit, direction and config as the GPU arm, the oracle described as its CPU baseline, and an end-to-end
entry with no host-device bytes."""

from __future__ import annotations

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _line(args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [x for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


def test_reference_arm_line():
    import argparse

    import bench

    d = _line(["--impl", "reference", "--workload", "tiny4K", "--steps", "2", "--warmup", "1"])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["value"] > 0 and d["ms_per_step"] > 0
    # the same config dict as the GPU arm's line for this workload on one rank
    w = bench.WORKLOADS["tiny4K"]
    assert d["config"] == bench.arm_config(argparse.Namespace(workload="tiny4K"), w, 1)
    assert d["config"]["S"] == 768
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_oracle_unavailable_above_its_memory():
    import bench

    # the oracle's S x S attention matrices do not fit the host at the expansion variant's S = 65,536
    assert bench.oracle_unavailable(bench.WORKLOADS["stress1M_expand"])
    assert not bench.oracle_unavailable(bench.WORKLOADS["tiny4K"])


def test_algorithmic_work_of_the_configurations():
    """The gathered lengths of the benchmarked configurations and the attention FLOPs at 512K, as the closed forms
    give them: S = sum over ranked levels of min(k, N_l) + N_(L-1) (children expansion: p picks of the level above
    per pick, plus the whole coarsest level); attention 2 S^2 d and 5 S^2 d per head."""
    import bench

    S = {name: bench.kernel_work(w)[1] for name, w in bench.WORKLOADS.items()}
    assert S["tiny4K"] == 768 and S["train32K"] == 6656 and S["ctx98K"] == 7680
    assert S["long512K"] == 3 * 4096 + 524288 // 64 == 20480
    assert S["stress1M"] == 3 * 4096 + 1048576 // 64 == 28672
    assert S["stress1M_expand"] == 3 * 4 * 4096 + 1048576 // 64 == 65536
    assert S["dense512K"] == 524288
    work, _ = bench.kernel_work(bench.WORKLOADS["long512K"])
    assert work["attn_fwd"] == ("tensor", 2.0 * 20480 ** 2 * 128 * 16)  # 1.718 TFLOP
    assert work["attn_bwd"] == ("tensor", 5.0 * 20480 ** 2 * 128 * 16)  # 4.295 TFLOP
    # pool: Q, K and V read once, their coarsest level written, the scores of the ranked levels written
    N, d, BH = 524288, 128, 16
    assert work["pool_score"][1] == BH * (3 * N * d * 2 + 3 * (N // 64) * d * 2 + (N + N // 4 + N // 16) * 4)
