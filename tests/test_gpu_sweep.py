"""GPU parity of the line-sweep large-plane kernel (sweep_kernel) against the
fp64 oracle, with the kernel selected explicitly.

The shapes reach every part of its plan: chains on 1, 2, 4 and 8 CTAs of a
cluster (DSMEM halo refreshes), two chains of one orientation per team item
and idle team halves (single directions), the largest owned share per CTA,
ragged owned ranges, partial last stages (H not a multiple of the stage),
local groups, channel-shared logits and many planes cycling through the L2
slots; planes outside its constraints fall back to another kernel.  Error metric and bars as in test_gpu_parity.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_spatial_propagation_line_b200 import gspn, inputs
from linear_spatial_propagation_line_b200.inputs import Workload

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}


@pytest.fixture
def sweep_path():
    gspn.debug_select_path(gspn.PATH_SWEEP)
    yield
    gspn.debug_select_path(gspn.PATH_AUTO)


def rel_err(y_gpu, ref):
    y = y_gpu.detach().double().cpu().numpy()
    assert np.isfinite(y).all()
    return float(np.abs(y - ref).max() / max(np.abs(ref).max(), 1e-300))


def to_dev(inp, device):
    return {"x": inp["x"].to(device),
            "wlogit": [t.to(device) for t in inp["wlogit"]],
            "lam": [t.to(device) for t in inp["lam"]],
            "u": [t.to(device) for t in inp["u"]]}


def run_check(wl, device, seed):
    inp = inputs.make_inputs(wl, seed)
    dev = to_dev(inp, device)
    y = gspn.forward(dev["x"], dev["wlogit"], dev["lam"], dev["u"], wl.group_len)
    torch.cuda.synchronize()
    assert gspn.last_kernel_name() == "sweep_kernel"
    ref = oracle.forward(inp["x"], inp["wlogit"], inp["lam"], inp["u"], wl.group_len)
    err = rel_err(y, ref)
    assert err <= TOL[wl.dtype], f"{wl.name} {wl.H}x{wl.W}: rel err {err:.3e}"


SWEEP_SHAPES = [
    # (H, W, g)
    (72, 96, 0),        # one CTA per chain in both orientations
    (700, 96, 0),       # horizontal chains on 2 CTAs, both vertical chains in one item
    (96, 704, 0),       # vertical chains on 2 CTAs
    (1500, 200, 0),     # horizontal on 4 CTAs, vertical on 2
    (200, 1504, 0),
    (2100, 64, 0),      # horizontal on 8 CTAs, vertical on 4 (16 columns each)
    (3000, 256, 0),
    (1100, 1000, 0),
    (513, 520, 0),      # just over one CTA's share
    (4100, 72, 0),      # 520-position shares on 8 CTAs (near the largest window)
    (1201, 160, 100),   # local groups, ragged last group
    (160, 1208, 33),
    (257, 136, 5),
]


@pytest.mark.parametrize("H,W,g", SWEEP_SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_sweep_shapes(H, W, g, dtype, cuda_device, sweep_path):
    run_check(Workload("sweep", 1, 2, H, W, g, dtype), cuda_device, seed=3 * H + W + g)


@pytest.mark.parametrize("H,W", [(8000, 16), (8000, 256)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_planes_outside_the_plan_fall_back(H, W, dtype, cuda_device, sweep_path):
    """8000 rows need more than 8 CTAs of at most 544 owned rows, and 16
    columns over 4 CTAs would give a CTA fewer owned positions than the
    16-position halo it sends: the line-sweep plan refuses both planes and the
    line-chain kernel computes them (the fused kernel is switched off here)."""
    wl = Workload("outside", 1, 2, H, W, 0, dtype)
    inp = inputs.make_inputs(wl, 2)
    dev = to_dev(inp, cuda_device)
    y = gspn.forward(dev["x"], dev["wlogit"], dev["lam"], dev["u"], 0)
    torch.cuda.synchronize()
    assert gspn.last_kernel_name() == "chain_kernel"
    ref = oracle.forward(inp["x"], inp["wlogit"], inp["lam"], inp["u"], 0)
    assert rel_err(y, ref) <= TOL[dtype]


def test_sweep_many_planes_reuse_slots(cuda_device, sweep_path):
    """More planes than L2 slots: slots are handed from plane to plane."""
    run_check(Workload("slots", 3, 20, 1024, 1024, 0, "bf16"), cuda_device, seed=11)


@pytest.mark.parametrize("H,W", [(150, 96), (300, 520)])
@pytest.mark.parametrize("d", [0, 1, 2, 3])
def test_sweep_single_direction(H, W, d, cuda_device, sweep_path):
    wl = Workload("dir", 1, 2, H, W, 0, "f32")
    inp = inputs.make_inputs(wl, 5 + d)
    dev = to_dev(inp, cuda_device)
    y = gspn.forward_dir(dev["x"], dev["wlogit"][d], dev["lam"][d], dev["u"][d], d)
    torch.cuda.synchronize()
    assert gspn.last_kernel_name() == "sweep_kernel"
    ref = inp["u"][d].double().numpy() * oracle.hidden(inp["x"], inp["wlogit"][d], inp["lam"][d], d)
    assert rel_err(y, ref) <= TOL["f32"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_sweep_shared_logits(dtype, cuda_device, sweep_path):
    wl = Workload("shared", 2, 3, 520, 264, 0, dtype)
    inp = inputs.make_inputs(wl, 9)
    z1 = [t[:, :1].contiguous() for t in inp["wlogit"]]
    dev = to_dev(inp, cuda_device)
    y = gspn.forward_shared(dev["x"], [t.to(cuda_device) for t in z1], dev["lam"], dev["u"], 0)
    torch.cuda.synchronize()
    assert gspn.last_kernel_name() == "sweep_kernel"
    zfull = [t.expand(wl.B, wl.C, 3, wl.H, wl.W) for t in z1]
    ref = oracle.forward(inp["x"], zfull, inp["lam"], inp["u"], 0)
    assert rel_err(y, ref) <= TOL[dtype]


def test_sweep_matches_fused_kernel(cuda_device):
    """Both large-plane kernels agree with each other to fp32 rounding."""
    wl = Workload("both", 1, 2, 600, 392, 0, "f32")
    dev = to_dev(inputs.make_inputs(wl, 4), cuda_device)
    out = {}
    try:
        for path in (gspn.PATH_FUSED, gspn.PATH_SWEEP):
            gspn.debug_select_path(path)
            out[path] = gspn.forward(dev["x"], dev["wlogit"], dev["lam"], dev["u"], 0)
            torch.cuda.synchronize()
    finally:
        gspn.debug_select_path(gspn.PATH_AUTO)
    a, b = out[gspn.PATH_FUSED].double(), out[gspn.PATH_SWEEP].double()
    assert float((a - b).abs().max() / a.abs().max()) <= 1e-5
