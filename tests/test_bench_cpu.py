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
