"""Benchmark of the Lighthouse selection-and-attend layer: forward + backward tokens/s on one B200 per rank.

One step = ``lh_forward`` + ``lh_backward`` (pool, score, top-K, gather, causal attention, scatter and their
backward) over one batch of synthetic inputs resident in HBM.  Multi-GPU runs are weak-scaled replicas (each rank
its own batch, no collective on the data path); the step time is the max over ranks.

Prints ONE JSON line (rank 0).  ``--impl reference`` times the CPU oracle instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    "tiny4K": dict(B=1, H=2, N=4096, d=64, L=3, p=4, k=256, C=8),
    "train32K": dict(B=1, H=16, N=32768, d=64, L=4, p=4, k=2048, C=16),
    "ctx98K": dict(B=1, H=16, N=98304, d=64, L=4, p=4, k=2048, C=16),
    "long512K": dict(B=1, H=16, N=524288, d=128, L=4, p=4, k=4096, C=32),
    "stress1M": dict(B=1, H=8, N=1048576, d=128, L=4, p=4, k=4096, C=32),
    # a smaller d=128 case with the long-context level structure, for profiler captures that must stay small
    "probe128K": dict(B=1, H=4, N=131072, d=128, L=4, p=4, k=4096, C=32),
    # dense comparator: one level, identity selection (S = N), i.e. plain causal attention through the same kernels
    "dense512K": dict(B=1, H=16, N=524288, d=128, L=1, p=4, k=1, C=1),
    # variant parameters: the recipe's L=3, k=1536, and the ablation grid's L in {3, 4}, k in {1536, 2048} at 98K
    "recipe98K": dict(B=1, H=16, N=98304, d=64, L=3, p=4, k=1536, C=16),
    "ablation98K_L4k1536": dict(B=1, H=16, N=98304, d=64, L=4, p=4, k=1536, C=16),
    # the children-expansion reading at the pages' size example (S = 65,536 at N = 2^20)
    "stress1M_expand": dict(B=1, H=8, N=1048576, d=128, L=4, p=4, k=4096, C=32, expand=True),
}
DEFAULT_WORKLOAD = "long512K"
METRIC = "Lighthouse fwd+bwd tokens/s at N=512K; HBM GB/s and attention TFLOP/s vs peak"
UNIT = "tokens/s"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return dict(hbm=pk["hbm_gbs"], bf16=pk["bf16_tflops"], bf16_sust=pk["bf16_tflops_sustained"], src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, src="fallback")


def kernel_work(w: dict) -> dict:
    """Algorithmic bytes (HBM-bound kernels) or FLOPs (attention) of ONE launch of each kernel, all heads."""
    B, H, N, d, L, p, k = w["B"], w["H"], w["N"], w["d"], w["L"], w["p"], w["k"]
    expand = w.get("expand", False)
    BH = B * H
    Nl = [N // p ** lev for lev in range(L)]
    if expand:  # level lev keeps the p children of the picks of level lev + 1
        kl = [p * min(k, Nl[lev + 1]) if lev < L - 1 else Nl[lev] for lev in range(L)]
        ranked = [lev + 1 for lev in range(L - 1) if kl[lev] < Nl[lev]]
        Rs = sum(Nl[1:])
    else:
        kl = [min(k, Nl[lev]) if lev < L - 1 else Nl[lev] for lev in range(L)]
        ranked = [lev for lev in range(L - 1) if kl[lev] < Nl[lev]]
        Rs = sum(Nl[:-1])
    S = sum(kl)
    R = sum(Nl)
    row = d * 2
    # rows of the raw input that selected entries below the coarsest level cover (read by the gather)
    gather_src = sum(kl[lev] * p ** lev for lev in range(L - 1)) + Nl[-1]
    partial = sum(Nl[lev] for lev in ranked)  # scores read by the top-K
    slots_init = sum(Nl[lev] for lev in range(L - 1) if kl[lev] < Nl[lev])
    return {
        "pool_score": ("hbm", BH * (3 * N * row + 3 * Nl[-1] * row + Rs * 4)),
        "topk": ("hbm", BH * (partial * 4 + slots_init * 4 + sum(kl[:-1]) * 4)),
        "order": ("hbm", BH * (S * 4 * 2 + sum(kl[:-1]) * 4)),
        "gather": ("hbm", BH * 3 * (gather_src + S) * row),
        "attn_fwd": ("tensor", 2.0 * S * S * d * BH),
        "scatter": ("hbm", BH * (N * row + S * row + R * 4)),
        "scatter_bwd": ("hbm", BH * (N * row + S * d * 4)),
        "bwd_prep": ("hbm", BH * S * (d * 4 * 2 + d * 2 + 4 + d * 4)),
        "absmax": ("hbm", BH * S * d * 4),
        "attn_bwd": ("tensor", 5.0 * S * S * d * BH),
        "unpool_bwd": ("hbm", BH * (3 * N * row + S * d * 4 + 2 * S * row + R * 4)),
    }, S


def kernel_bytes(w: dict) -> dict:
    """Algorithmic DRAM bytes of ONE launch of each kernel (all heads): the HBM-bound kernels' bytes as in
    kernel_work, and for the attention kernels the unique bytes of their operands and outputs (fp16 gathered rows,
    fp32 outputs and accumulators, per-row statistics).  Used to scale a DRAM-traffic capture taken on a small
    workload to another workload of the same kernel."""
    work, S = kernel_work(w)
    BH, d = w["B"] * w["H"], w["d"]
    out = {n: amt for n, (bound, amt) in work.items() if bound == "hbm"}
    out["attn_fwd"] = BH * S * (3 * d * 2 + d * 4 + 4)
    out["attn_bwd"] = BH * S * (4 * d * 2 + 2 * 4 + 2 * d * 4 + 2 * d * 4)
    return out


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one-kernel ncu captures on a small
# workload, recorded in profiles/dram_traffic.txt with a digest of the kernel's sources; reported (scaled to the
# bench's workload by the ratio of algorithmic bytes) only while the sources still match.
TRAFFIC_FILE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles", "dram_traffic.txt")
CSRC = os.path.join(os.path.dirname(os.path.abspath(__file__)), "hierarchical_sparse_attention_avg_b200", "csrc")
KERNEL_SOURCES = {"attn_bwd": "attn_bwd.cu", "attn_fwd": "attn_fwd.cu", "pool_score": "pool_gather.cu",
                  "gather": "pool_gather.cu", "unpool_bwd": "scatter.cu", "scatter": "scatter.cu",
                  "scatter_bwd": "scatter.cu", "bwd_prep": "scatter.cu", "absmax": "scatter.cu", "topk": "topk.cu",
                  "order": "topk.cu"}


def source_digest(kernel: str) -> str:
    import hashlib

    h = hashlib.sha256()
    for f in (KERNEL_SOURCES.get(kernel, ""), "lh_common.cuh", "internal.h"):
        path = os.path.join(CSRC, f)
        if f and os.path.exists(path):
            h.update(open(path, "rb").read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, w: dict):
    """(bytes per launch at workload w, capture workload) for `kernel`, or (None, None) when no capture matches the
    current sources.  A capture on another workload is scaled by the ratio of the kernel's algorithmic bytes."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, None
    for line in open(TRAFFIC_FILE):
        f = line.split("#")[0].split()
        if len(f) == 5 and f[0] == kernel and f[1] in WORKLOADS:
            if f[4] != source_digest(kernel):
                continue
            got = int(f[2]) + int(f[3])
            if WORKLOADS[f[1]] == w:
                return got, f[1]
            ratio = kernel_bytes(w)[kernel] / kernel_bytes(WORKLOADS[f[1]])[kernel]
            return int(round(got * ratio)), f[1]
    return None, None


class NvmlClockSampler:
    """SM clock and clock-event reasons read through NVML every 10 ms in a thread while the timed region runs
    (read-only queries; no setting of the GPU is changed)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device):
        import threading

        import pynvml

        self.nv = pynvml
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(device).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode() if isinstance(uuid, str) else uuid)
        self.samples, self.reasons = [], set()
        self.stop_ev = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)

    def _run(self):
        nv = self.nv
        while not self.stop_ev.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, attr in self.REASONS:
                    if bits & getattr(nv, attr):
                        self.reasons.add(name)
            except Exception:
                pass
            self.stop_ev.wait(0.01)

    def start(self):
        self.thread.start()

    def stop(self) -> dict | None:
        self.stop_ev.set()
        self.thread.join(timeout=2)
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


def make_clock_sampler(device):
    try:
        return NvmlClockSampler(device)
    except Exception:
        return ClockSampler(device)


class ClockSampler:
    """nvidia-smi clock/throttle sampling (every 200 ms) while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.sel = []
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            self.sel = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", *self.sel, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[5 + i] and "Not" not in r[5 + i]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(values, world: int, device) -> list:
    """Element-wise max of `values` (floats) over all ranks.  Every rank calls it at the same points, in the same
    order, including on error paths (a device status is reduced with the times, so all ranks raise together)."""
    if world == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_tokens(w: dict, world: int) -> int:
    """Tokens all ranks process in one step: each rank runs its own batch (weak scaling)."""
    return w["B"] * w["N"] * world


def oracle_unavailable(w: dict):
    """Why the oracle cannot time a head of workload w on the host, or None.  It holds several S x S float64
    matrices (8 GB each at S = 32K)."""
    S = kernel_work(w)[1]
    return f"the oracle's S x S attention matrices at S = {S} exceed host memory" if S > 32768 else None


def cpu_baseline(w: dict, seed: int = 0) -> dict:
    """The CPU oracle timed on one head of the workload (forward + backward), scaled to tokens/s of the whole
    workload (heads are independent, so the time of all B*H heads is B*H times one head's)."""
    from oracle import lighthouse as O
    from hierarchical_sparse_attention_avg_b200.inputs import make_inputs

    why = oracle_unavailable(w)
    if why:
        return {"unavailable": why, "kind": "oracle"}
    q, k, v, dout = make_inputs(1, 1, w["N"], w["d"], seed=seed, device="cpu")
    f = lambda t: t[0, 0].float().numpy().astype(np.float64)
    qf, kf, vf, df = f(q), f(k), f(v), f(dout)
    P = O.Params(1, 1, w["N"], w["d"], w["L"], w["p"], w["k"], w["C"], w.get("expand", False))
    t0 = time.perf_counter()
    fwd = O.forward_head(qf, kf, vf, P)
    O.backward_head(df, fwd, P)
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info

        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = 1
    heads = w["B"] * w["H"]
    return {"value": w["B"] * w["N"] / (dt * heads), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"1 of {heads} heads of {w_name(w)} (forward+backward, {dt:.1f} s), scaled by {heads}",
            "seconds": dt}


def w_name(w):
    for n, v in WORKLOADS.items():
        if v == w:
            return n
    return "custom"


def arm_config(args, w, world: int) -> dict:
    """The `config` of the bench line, the same for both arms (the reference arm times a sample of this workload)."""
    S = kernel_work(w)[1]
    l2 = ("inputs larger than L2 (2 GB per tensor), no flush" if w["B"] * w["H"] * w["N"] * w["d"] * 2 > 126e6
          else "inputs smaller than L2, no flush")
    return {"workload": args.workload, **w, "S": S, "parallelism": f"replicas{world}", "l2": l2}


def run_reference(args, w):
    """The oracle as the reference arm: W warm-up steps and K timed steps, each one head of the workload
    (forward + backward) on the host cores; tokens/s of that sample.  Rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    why = oracle_unavailable(w)
    if why:
        print(json.dumps({"impl": "reference", "unavailable": why}), flush=True)
        return
    for _ in range(max(args.warmup, 0)):
        cpu_baseline(w)
    times = [cpu_baseline(w)["seconds"] for _ in range(args.steps)]
    heads = w["B"] * w["H"]
    sec = sum(times) / len(times)
    value = w["B"] * w["N"] / (sec * heads)  # the workload's tokens over the time all its heads take
    try:
        from threadpoolctl import threadpool_info

        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = 1
    sample = f"one head of {heads} per step (forward+backward; heads are independent)"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": arm_config(args, w, int(os.environ.get("WORLD_SIZE", "1"))),
            "scaled_to_all_heads": {"ms_per_step": sec * 1e3 * heads,
                                    "note": f"one head's time x {heads} heads: the time the whole step would take"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_cp(args, w):
    """Context-parallel step: rank r holds tokens [r N/G, (r+1) N/G) of every head of one sequence and runs the
    lh_cp_* stages with NCCL all-gathers and a reduce-scatter (cp.forward / cp.backward); the step time is the max
    over ranks and the tokens are the one sequence's (strong scaling).  A single process forms a group of one."""
    import datetime

    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world == 1:  # a group of one: under torchrun its rendezvous variables are set, else a local port is taken
        if "MASTER_ADDR" not in os.environ:
            import socket

            with socket.socket() as sk:
                sk.bind(("127.0.0.1", 0))
                port = sk.getsockname()[1]
            os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0", WORLD_SIZE="1")
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    from hierarchical_sparse_attention_avg_b200 import cp, lh
    from hierarchical_sparse_attention_avg_b200.inputs import make_inputs

    P = lh.Params(**w)
    sp = cp.split(P, world)
    L = sp.local
    q, k, v, dout = make_inputs(L.B, L.H, L.N, L.d, seed=rank, device=dev)
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    st = cp.new_state(sp, rank, dev)
    ex = cp.TorchDistExchange()

    def step():
        cp.forward(st, q, k, v, ex, o=o)
        cp.backward(st, dout, ex, dq=dq, dk=dk, dv=dv)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize(dev)
    torch.distributed.barrier()
    clocks = make_clock_sampler(dev)
    clocks.start()
    lh.lh_profile_enable(True)
    lh.lh_profile_read()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    torch.distributed.barrier()
    lh.lh_profile_enable(False)
    prof = lh.lh_profile_read()
    clk = clocks.stop()
    t = torch.tensor([e0.elapsed_time(e1) / args.steps, float(lh.lh_get_status(dev))], dtype=torch.float64,
                     device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    ms, status = float(t[0]), int(t[1])
    if status != 0:
        raise RuntimeError(f"device status {status}: {lh.error_string(status)}")
    if rank == 0:
        tokens = w["B"] * w["N"]
        kernels = {n: {"launches": c, "ms": m / c} for n, (c, m) in sorted(prof.items(), key=lambda kv: -kv[1][1])}
        line = {"metric": METRIC, "value": tokens / (ms / 1e3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": args.workload, **w, "S": kernel_work(w)[1], "S_per_rank": sp.S_local,
                           "parallelism": f"cp{world}",
                           "exchange_bytes_per_rank": {"kv_all_gather": sp.kv_bytes * world,
                                                       "halo_all_gathers": 2 * sp.halo_bytes * world,
                                                       "dkv_reduce_scatter": sp.dkv_bytes * world}},
                "kernels": kernels, "gpu_launches": sum(c for c, _ in prof.values()), "clocks": clk, "e2e": None}
        print(json.dumps(line), flush=True)
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cp", action="store_true",
                    help="context parallelism: the ranks split ONE sequence of the workload (strong scaling), "
                         "exchanging through lh_cp_* and NCCL collectives; default: independent replicas")
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
        return
    if args.cp:
        run_cp(args, w)
        return

    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from hierarchical_sparse_attention_avg_b200 import lh
    from hierarchical_sparse_attention_avg_b200.inputs import make_inputs

    P = lh.Params(**w)
    q, k, v, dout = make_inputs(w["B"], w["H"], w["N"], w["d"], seed=rank, device=dev)
    o = torch.empty_like(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ctx = lh.new_ctx(P, dev)
    ws = lh.new_workspace(P, dev)

    def step():
        lh.lh_forward(P, q, k, v, o=o, ctx=ctx, ws=ws)
        lh.lh_backward(P, dout, ctx, dq=dq, dk=dk, dv=dv, ws=ws)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    clocks = make_clock_sampler(dev)
    clocks.start()
    lh.lh_profile_enable(True)
    lh.lh_profile_read()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    lh.lh_profile_enable(False)
    prof = lh.lh_profile_read()
    clk = clocks.stop()
    ms, status = max_over_ranks([e0.elapsed_time(e1) / args.steps, lh.lh_get_status(dev)], world, dev)
    if status != 0:
        raise RuntimeError(f"device status {int(status)}: {lh.error_string(int(status))}")
    tokens = whole_job_tokens(w, world)
    value = tokens / (ms / 1e3)

    # end to end through the C ABI with host buffers (lh_step_host): every step copies its inputs from page-locked
    # host memory and its outputs back, chunk by chunk of heads, the two copy directions and the compute overlapped
    e2e = None
    if not args.no_e2e:
        host_in = [t.cpu().pin_memory() for t in (q, k, v, dout)]
        host_out = [torch.empty(q.shape, dtype=q.dtype, pin_memory=True) for _ in range(4)]
        hc = lh.default_heads_per_chunk(P)
        dev_buf = torch.empty(lh.lh_step_host_bytes(P, hc), dtype=torch.uint8, device=dev)

        def e2e_step():
            lh.lh_step_host(P, *host_in, *host_out, heads_per_chunk=hc, dev_buf=dev_buf, device=dev)

        e2e_step()
        torch.cuda.synchronize(dev)
        n_e2e = max(1, min(args.steps, 3))
        if world > 1:
            torch.distributed.barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        ms_e2e = max_over_ranks([a0.elapsed_time(a1) / n_e2e], world, dev)[0]
        nbytes = sum(t.numel() * t.element_size() for t in host_in)
        obytes = sum(t.numel() * t.element_size() for t in host_out)
        e2e = {"value": tokens / (ms_e2e / 1e3), "unit": UNIT, "h2d_bytes_per_step": nbytes,
               "d2h_bytes_per_step": obytes, "ms_per_step": ms_e2e, "steps": n_e2e,
               "pipeline": f"lh_step_host, {w['B'] * (w['H'] // hc)} chunks of {hc} heads"}

    peaks = load_peaks()
    work, S = kernel_work(w)
    total_kernel_ms = sum(v_[1] for v_ in prof.values()) or 1.0
    kernels = {}
    for name, (launches, kms) in sorted(prof.items(), key=lambda kv: -kv[1][1]):
        bound, amount = work.get(name, ("hbm", 0))
        per_ms = kms / launches
        if bound == "tensor":
            # timed inside a step of milliseconds at full SM clock: the burst GEMM peak applies (the sustained
            # figure, a seconds-long GEMM loop at the power cap's lower clock, is reported beside it)
            ach = amount / (per_ms / 1e3) / 1e12
            kernels[name] = {"launches": launches, "ms": per_ms, "share": kms / total_kernel_ms, "bound": "tensor",
                             "achieved": ach, "unit": "TFLOP/s", "frac": ach / peaks["bf16"],
                             "frac_sustained": ach / peaks["bf16_sust"]}
        else:
            ach = amount / (per_ms / 1e3) / 1e9
            kernels[name] = {"launches": launches, "ms": per_ms, "share": kms / total_kernel_ms, "bound": "hbm",
                             "achieved": ach, "unit": "GB/s", "frac": ach / peaks["hbm"]}
    top = max(kernels.items(), key=lambda kv: kv[1]["share"])
    tname, tk = top
    traffic, traffic_src = measured_traffic(tname, w)
    roofline = {"kernel": tname, "bound": tk["bound"], "achieved": tk["achieved"],
                "peak": peaks["bf16"] if tk["bound"] == "tensor" else peaks["hbm"], "unit": tk["unit"],
                "frac": tk["frac"], "traffic": traffic,
                "peak_source": f"{peaks['src']} ({'bf16 burst' if tk['bound'] == 'tensor' else 'HBM copy'})"}
    if tk["bound"] == "tensor":
        roofline["frac_sustained"] = tk["frac_sustained"]
    if traffic_src is not None:
        roofline["traffic_source"] = (f"ncu one-kernel capture on {traffic_src}" +
                                      ("" if traffic_src == args.workload else
                                       f", scaled by the kernel's algorithmic bytes to {args.workload}"))
    gpu_launches = sum(v_[0] for v_ in prof.values())

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": arm_config(args, w, world),
                "roofline": roofline, "kernels": kernels, "gpu_launches": gpu_launches,
                "clocks": clk, "e2e": e2e}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = {k_: v_ for k_, v_ in cpu_baseline(w).items() if k_ != "seconds"}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
