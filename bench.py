#!/usr/bin/env python
"""Throughput benchmark of the GSPN 4-direction propagation on B200.

One step = one full pass of the propagation (all four directions, sigmoid +
normalisation, local/global recurrence, merge into y) over one batch of the
workload, through the library's C ABI.  Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one process per GPU): every rank runs its own
independent copy of the workload (planes are independent; no collective on
the data path) and the time is the max over ranks ("scaling": "weak").
``--impl reference`` times the fp64 CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import pathlib
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = pathlib.Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

from linear_spatial_propagation_line_b200 import gspn  # noqa: E402
from linear_spatial_propagation_line_b200.inputs import HEADLINE, WORKLOADS, make_inputs  # noqa: E402

METRIC = "GSPN 4-dir propagation Gpix·ch/s and achieved HBM GB/s (% of B200 peak)"
UNIT = "Gpix·ch/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024

# Kernel -> (source files whose hash identifies it, algorithmic elements moved
# per pix*ch by one launch of it).  Inputs: 1 x + 12 logits + 4 lambda + 4 u;
# output: 1 y.  The chain kernel's fp32 workspace traffic is not algorithmic.
KERNELS = {
    "small_plane_kernel": (["gspn_small.cu", "gspn_common.cuh"], 22),
    "chain_kernel": (["gspn_chain.cu", "gspn_common.cuh"], 21),
    "fused_kernel": (["gspn_fused.cu", "gspn_ptx.cuh", "gspn_common.cuh"], 22),
    "sweep_kernel": (["gspn_sweep.cu", "gspn_ptx.cuh", "gspn_common.cuh"], 22),
}
CSRC = ROOT / "linear_spatial_propagation_line_b200" / "csrc"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--C", type=int, default=None,
                    help="override the channel count (small cases for profiler captures)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pass", dest="pass_", choices=["forward", "backward"], default="forward",
                    help="backward: time gspn_backward (gradients of sum(gy * y)) instead")
    ap.add_argument("--path", choices=["auto", "fused", "sweep"], default="auto",
                    help="large-plane kernel (auto: the fused kernel)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    return ap.parse_args()


# --------------------------------------------------------------------------
# distributed plumbing
# --------------------------------------------------------------------------
def dist_init(backend):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))
    return rank, local, world


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_close(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# --------------------------------------------------------------------------
# measurement helpers
# --------------------------------------------------------------------------
def measured_hbm_peak():
    p = ROOT / "MEASURED_PEAKS.json"
    try:
        v = float(json.loads(p.read_text())["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_hash(files):
    h = hashlib.sha256()
    for f in files:
        h.update((CSRC / f).read_bytes())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, or None if the
    kernel's sources changed since the counters were taken."""
    try:
        data = json.loads((ROOT / "profiles" / "traffic.json").read_text())
        ent = data[kernel]
        if ent.get("workload") != workload:
            return None
        if ent.get("source_sha") != source_hash(KERNELS[kernel][0]):
            return None
        return float(ent["traffic_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        try:
            props = torch.cuda.get_device_properties(device_index)
            self.bus = f"{props.pci_bus_id:02X}:{props.pci_device_id:02X}."
        except Exception:
            self.bus = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="gspn_clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in pathlib.Path(self.path).read_text().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            if self.bus and self.bus not in parts[0].upper():
                continue
            rows.append(parts)
        try:
            os.unlink(self.path)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}

        def num(s):
            try:
                return float(s)
            except ValueError:
                return None

        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for r in rows for j in range(4) if r[5 + j] == "Active"})
        loaded = [v for v in sm if v is not None]
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------
# CPU baseline (the fp64 oracle on the host cores, bounded sample)
# --------------------------------------------------------------------------
def oracle_sample_rate(wl, target_seconds: float, max_planes: int = 16):
    import oracle

    cores = oracle.default_threads()
    planes = max(1, min(max_planes, cores, wl.B * wl.C))
    sample_wl = wl.with_(B=1, C=planes)
    inp = make_inputs(sample_wl, seed=99)
    import numpy as np  # noqa: F401  (conversion below happens outside timing)
    x = oracle.as_f64(inp["x"])
    z = [oracle.as_f64(t) for t in inp["wlogit"]]
    la = [oracle.as_f64(t) for t in inp["lam"]]
    uu = [oracle.as_f64(t) for t in inp["u"]]
    reps, elapsed = 0, 0.0
    t0 = time.perf_counter()
    while True:
        oracle.forward(x, z, la, uu, wl.group_len, nthreads=planes)
        reps += 1
        elapsed = time.perf_counter() - t0
        if elapsed >= target_seconds or reps >= 1000:
            break
    pixch = sample_wl.pixch * reps
    return {"value": pixch / elapsed / 1e9, "unit": UNIT, "cores": planes, "kind": "oracle",
            "sample": f"{planes} planes of {wl.H}x{wl.W} x {reps} repeats "
                      f"({elapsed:.1f} s, fp64 C++ loop, one thread per plane)"}


def run_reference(args, wl):
    rank, _local, world = dist_init("gloo")
    if rank != 0:
        dist_close(world)
        return
    import oracle

    cores = oracle.default_threads()
    planes = max(1, min(16, cores, wl.B * wl.C))
    sample_wl = wl.with_(B=1, C=planes)
    inp = make_inputs(sample_wl, seed=99)
    x = oracle.as_f64(inp["x"])
    z = [oracle.as_f64(t) for t in inp["wlogit"]]
    la = [oracle.as_f64(t) for t in inp["lam"]]
    uu = [oracle.as_f64(t) for t in inp["u"]]
    for _ in range(args.warmup):
        oracle.forward(x, z, la, uu, wl.group_len, nthreads=planes)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward(x, z, la, uu, wl.group_len, nthreads=planes)
    dt = (time.perf_counter() - t0) / args.steps
    value = sample_wl.pixch / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_dict(wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": planes, "kind": "oracle",
                         "sample": f"{planes} planes of {wl.H}x{wl.W} per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    dist_close(world)


def config_dict(wl, n):
    return {"workload": wl.name, "B": wl.B, "C": wl.C, "H": wl.H, "W": wl.W,
            "group_len": wl.group_len, "storage_dtype": wl.dtype,
            "global_batch": wl.B * n, "planes_per_gpu": wl.B * wl.C,
            "l2": f"inputs {wl.algorithmic_bytes() / 1e9:.2f} GB per step > 126 MB L2; no flush",
            "parallelism": f"replicas x{n} (independent planes, no collective)"}


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
def run_ours(args, wl):
    rank, local, world = dist_init("nccl")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    gspn.load_library()
    gspn.debug_select_path({"auto": gspn.PATH_AUTO, "fused": gspn.PATH_FUSED,
                            "sweep": gspn.PATH_SWEEP}[args.path])

    inp = make_inputs(wl, seed=rank, device=str(device), gen_device=str(device))
    y = torch.empty_like(inp["x"])
    step = lambda: gspn.forward(inp["x"], inp["wlogit"], inp["lam"], inp["u"], wl.group_len,
                                out=y)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    launches_per_step = gspn.last_launch_count()
    kernel = gspn.last_kernel_name()

    K = args.steps
    kb = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ke = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    for ev in kb + ke:  # torch creates the CUDA event on first record
        ev.record()
    clocks = ClockSampler(local)

    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.25)
    t_start.record()
    for i in range(K):
        gspn.set_timing_events(kb[i], ke[i])
        step()
    t_end.record()
    gspn.set_timing_events(None, None)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)

    ms_local = t_start.elapsed_time(t_end) / K
    kern_ms_local = statistics.mean(kb[i].elapsed_time(ke[i]) for i in range(K))
    ms = max_over_ranks(ms_local, world, device)
    kern_ms = max_over_ranks(kern_ms_local, world, device)

    pixch_total = wl.pixch * world
    value = pixch_total / (ms * 1e-3) / 1e9
    peak, peak_kind = measured_hbm_peak()
    files, elems = KERNELS.get(kernel, ([], 22))
    alg_bytes = elems * wl.pixch * wl.esize
    achieved = alg_bytes / (kern_ms * 1e-3) / 1e9
    step_gbs = wl.algorithmic_bytes() / (ms * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(args, wl, inp, device, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample_rate(wl, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": config_dict(wl, world),
            "achieved_hbm_gbs": step_gbs,
            "hbm_frac_of_nominal_8tbs": step_gbs / NOMINAL_HBM_GBS,
            "hbm_frac_of_measured": step_gbs / peak,
            "roofline": {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "algorithmic_bytes_per_launch": alg_bytes,
                         "kernel_ms": kern_ms,
                         "traffic": profiled_traffic(kernel, wl.name)},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * K,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    dist_close(world)


# Backward pass: inputs x, 12 logits, 4 lambda, 4 u and gy are read; dx, 12
# logit gradients, 4 lambda gradients and 4 u gradients are written.
BACKWARD_ELEMS = 22 + 21


def run_backward(args, wl):
    """Times gspn_backward on the same synthetic workload: one step is the
    whole backward call (its three kernels); the roofline is the call's
    algorithmic bytes over its time, with the reverse-scan kernel's own time
    beside it."""
    rank, local, world = dist_init("nccl")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    gspn.load_library()
    inp = make_inputs(wl, seed=rank, device=str(device), gen_device=str(device))
    g = torch.Generator(device=str(device)).manual_seed(1000 + rank)
    gy = torch.randn(inp["x"].shape, generator=g, device=device,
                     dtype=torch.float32).to(inp["x"].dtype)
    step = lambda: gspn.backward(inp["x"], inp["wlogit"], inp["lam"], inp["u"], gy,
                                 wl.group_len)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    launches_per_step = gspn.last_launch_count()
    K = args.steps
    kb = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ke = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    for ev in kb + ke:
        ev.record()
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.25)
    t_start.record()
    for i in range(K):
        gspn.set_timing_events(kb[i], ke[i])
        step()
    t_end.record()
    gspn.set_timing_events(None, None)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    ms = max_over_ranks(t_start.elapsed_time(t_end) / K, world, device)
    scan_ms = max_over_ranks(statistics.mean(kb[i].elapsed_time(ke[i]) for i in range(K)),
                             world, device)
    peak, peak_kind = measured_hbm_peak()
    alg_bytes = BACKWARD_ELEMS * wl.pixch * wl.esize
    achieved = alg_bytes / (ms * 1e-3) / 1e9
    if rank == 0:
        line = {
            "metric": "GSPN 4-dir backward (dx, dwlogit, dlam, du) Gpix·ch/s",
            "pass": "backward", "value": wl.pixch * world / (ms * 1e-3) / 1e9, "unit": UNIT,
            "n_gpus": world, "steps": K, "warmup": max(3, args.warmup), "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": config_dict(wl, world),
            "roofline": {"bound": "hbm", "kernel": "hidden_kernel+backward_kernel+round_kernel",
                         "achieved": achieved, "peak": peak, "peak_kind": peak_kind,
                         "unit": "GB/s", "frac": achieved / peak,
                         "algorithmic_bytes_per_launch": alg_bytes,
                         "kernel_ms": ms, "backward_kernel_ms": scan_ms, "traffic": None},
            "gpu_launches": launches_per_step * K,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    dist_close(world)


def measure_e2e(args, wl, inp, device, world):
    """Same metric through gspn_forward_host: pinned host inputs copied in,
    y copied back, every step inside the timed region."""
    def pinned(t):
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        return h

    host = {"x": pinned(inp["x"]), "wlogit": [pinned(t) for t in inp["wlogit"]],
            "lam": [pinned(t) for t in inp["lam"]], "u": [pinned(t) for t in inp["u"]]}
    yh = torch.empty(inp["x"].shape, dtype=inp["x"].dtype, pin_memory=True)
    call = lambda: gspn.forward_host(host["x"], host["wlogit"], host["lam"], host["u"],
                                     wl.group_len, out=yh, device=device)
    call()
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.e2e_steps):
        call()
    t1.record()
    torch.cuda.synchronize()
    dt = t0.elapsed_time(t1) * 1e-3 / args.e2e_steps
    dt = max_over_ranks(dt, world, device)
    gspn.release()  # give the staging area back
    return {"value": wl.pixch * world / dt / 1e9, "unit": UNIT,
            "h2d_bytes_per_step": 21 * wl.pixch * wl.esize,
            "d2h_bytes_per_step": wl.pixch * wl.esize, "ms_per_step": dt * 1e3,
            "steps": args.e2e_steps}


def main():
    args = parse_args()
    wl = WORKLOADS[args.workload]
    if args.C is not None:
        wl = wl.with_(C=args.C)
    if args.impl == "reference":
        run_reference(args, wl)
    elif args.pass_ == "backward":
        run_backward(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
