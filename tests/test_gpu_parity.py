"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle.

Error metric: max|y_gpu - y_ref| / max|y_ref| over the compared outputs.
Bars: 1e-5 for fp32 storage, 2e-2 for bf16 storage with fp32 arithmetic.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_spatial_propagation_line_b200 import gspn, inputs
from linear_spatial_propagation_line_b200.inputs import WORKLOADS, Workload

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}


def rel_err(y_gpu, ref):
    y = y_gpu.detach().double().cpu().numpy()
    assert np.isfinite(y).all()
    return float(np.abs(y - ref).max() / max(np.abs(ref).max(), 1e-300))


def to_dev(inp, device):
    return {"x": inp["x"].to(device),
            "wlogit": [t.to(device) for t in inp["wlogit"]],
            "lam": [t.to(device) for t in inp["lam"]],
            "u": [t.to(device) for t in inp["u"]]}


def check(wl: Workload, device, seed=0, planes=None):
    inp = inputs.make_inputs(wl, seed)
    dev = to_dev(inp, device)
    y = gspn.forward(dev["x"], dev["wlogit"], dev["lam"], dev["u"], wl.group_len)
    torch.cuda.synchronize()
    if planes is None:
        ref = oracle.forward(inp["x"], inp["wlogit"], inp["lam"], inp["u"], wl.group_len)
        err = rel_err(y, ref)
    else:
        b_idx = [p // wl.C for p in planes]
        c_idx = [p % wl.C for p in planes]
        sel = lambda t: t[b_idx, c_idx].unsqueeze(0)
        ref = oracle.forward(sel(inp["x"]), [sel(t) for t in inp["wlogit"]],
                             [sel(t) for t in inp["lam"]], [sel(t) for t in inp["u"]],
                             wl.group_len)
        err = rel_err(y[b_idx, c_idx].unsqueeze(0), ref)
    assert err <= TOL[wl.dtype], f"{wl.name}: rel err {err:.3e}"
    return err


@pytest.mark.parametrize("name", ["tiny16_global_f32", "cls56_global_f32", "local28_g7_bf16",
                                  "gen32_global_bf16"])
def test_named_workload_full(name, cuda_device):
    check(WORKLOADS[name], cuda_device)


def test_headline_workload_full_size_sampled_planes(cuda_device):
    """2048x1024 bf16, all 64 planes on the GPU in the benchmark's launch
    configuration; the oracle recomputes three whole planes."""
    check(WORKLOADS[inputs.HEADLINE], cuda_device, planes=[0, 37, 63])


SHAPES = [
    # (H, W): small-plane kernel
    (1, 1), (1, 7), (7, 1), (2, 3), (16, 33), (33, 16), (31, 64), (64, 64), (17, 45),
    # generic line-chain path
    (65, 3), (3, 65), (65, 64), (130, 257), (257, 130), (1, 700), (700, 1), (96, 160),
]


@pytest.mark.parametrize("H,W", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_shapes_global(H, W, dtype, cuda_device):
    wl = Workload("shape", 1, 3, H, W, 0, dtype)
    check(wl, cuda_device, seed=H * 1000 + W)


# Large planes on the fused kernel with multi-CTA teams (halo exchange through
# DSMEM): 2-, 4- and 8-CTA teams, ragged owned ranges, local groups.
TEAM_SHAPES = [(700, 96, 0), (96, 704, 0), (1500, 200, 0), (200, 1504, 0), (2100, 64, 0),
               (3000, 256, 0), (1201, 160, 100), (160, 1208, 33), (1100, 1000, 0)]


@pytest.fixture
def fused_path():
    gspn.debug_select_path(gspn.PATH_FUSED)
    yield
    gspn.debug_select_path(gspn.PATH_AUTO)


@pytest.mark.parametrize("H,W,g", TEAM_SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_large_planes_multi_cta_teams(H, W, g, dtype, cuda_device, fused_path):
    wl = Workload("team", 1, 2, H, W, g, dtype)
    check(wl, cuda_device, seed=H + 7 * W + g)
    # the fused kernel takes planes whose rows are whole 32-byte segments
    es = 4 if dtype == "f32" else 2
    assert gspn.last_kernel_name() == ("fused_kernel" if (W * es) % 32 == 0 else "chain_kernel")


@pytest.mark.parametrize("H,W", [(300, 256), (256, 512)])
@pytest.mark.parametrize("d", [0, 1, 2, 3])
def test_fused_single_direction(H, W, d, cuda_device, fused_path):
    """One direction at a time on the fused kernel (its work queue then holds
    one chain per plane)."""
    wl = Workload("fdir", 1, 2, H, W, 0, "f32")
    inp = inputs.make_inputs(wl, seed=10 + d)
    dev = to_dev(inp, cuda_device)
    y = gspn.forward_dir(dev["x"], dev["wlogit"][d], dev["lam"][d], dev["u"][d], d)
    torch.cuda.synchronize()
    assert gspn.last_kernel_name() == "fused_kernel"
    ref = inp["u"][d].double().numpy() * oracle.hidden(inp["x"], inp["wlogit"][d], inp["lam"][d], d)
    assert rel_err(y, ref) <= TOL["f32"]


@pytest.mark.parametrize("path,kernel", [(1, "fused_kernel"), (2, "sweep_kernel")])
def test_forced_timeout_is_reported_and_recovers(path, kernel, cuda_device):
    """A slot hand-over that never comes makes the kernel give up after its
    bounded wait; the host sees GSPN_ERR_TIMEOUT and the next call is exact."""
    wl = Workload("timeout", 1, 3, 256, 512, 0, "f32")
    inp = inputs.make_inputs(wl, 6)
    dev = to_dev(inp, cuda_device)
    gspn.debug_select_path(path)
    try:
        assert gspn.check_device_status() == 0
        gspn.debug_force_timeout(50_000_000)  # 50 ms
        gspn.forward(dev["x"], dev["wlogit"], dev["lam"], dev["u"], 0)
        assert gspn.last_kernel_name() == kernel
        assert gspn.check_device_status() == -7
        assert gspn.check_device_status() == 0
        y = gspn.forward(dev["x"], dev["wlogit"], dev["lam"], dev["u"], 0)
        assert gspn.last_kernel_name() == kernel
        ref = oracle.forward(inp["x"], inp["wlogit"], inp["lam"], inp["u"], 0)
        assert rel_err(y, ref) <= TOL["f32"]
        assert gspn.check_device_status() == 0
    finally:
        gspn.debug_select_path(gspn.PATH_AUTO)


def test_large_plane_kernel_for_the_headline_shape(cuda_device):
    wl = WORKLOADS[inputs.HEADLINE].with_(C=2)
    dev = to_dev(inputs.make_inputs(wl, 0), cuda_device)
    gspn.forward(dev["x"], dev["wlogit"], dev["lam"], dev["u"], 0)
    assert gspn.last_kernel_name() == "fused_kernel"
    assert gspn.last_launch_count() == 1


@pytest.mark.parametrize("H,W,g", [(28, 28, 7), (30, 27, 7), (16, 16, 1), (16, 16, 16),
                                   (16, 16, 100), (64, 64, 5), (130, 96, 7), (97, 200, 64),
                                   (300, 70, 1), (70, 300, 301)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_shapes_local(H, W, g, dtype, cuda_device):
    wl = Workload("local", 2, 2, H, W, g, dtype, logit_std=2.0)
    check(wl, cuda_device, seed=g + H + W)


@pytest.mark.parametrize("H,W", [(12, 20), (150, 90)])
@pytest.mark.parametrize("d", [0, 1, 2, 3])
def test_single_direction(H, W, d, cuda_device):
    wl = Workload("dir", 1, 2, H, W, 0, "f32")
    inp = inputs.make_inputs(wl, seed=d)
    dev = to_dev(inp, cuda_device)
    y = gspn.forward_dir(dev["x"], dev["wlogit"][d], dev["lam"][d], dev["u"][d], d)
    ref = inp["u"][d].double().numpy() * oracle.hidden(inp["x"], inp["wlogit"][d], inp["lam"][d], d)
    assert rel_err(y, ref) <= TOL["f32"]


def test_extreme_logits_stay_finite(cuda_device):
    for H, W in [(20, 20), (100, 80)]:
        wl = Workload("extreme", 1, 2, H, W, 0, "f32", logit_std=15.0)
        check(wl, cuda_device, seed=3)


def test_small_plane_path_is_deterministic(cuda_device):
    wl = WORKLOADS["gen32_global_bf16"].with_(B=2)
    dev = to_dev(inputs.make_inputs(wl, 1), cuda_device)
    a = gspn.forward(dev["x"], dev["wlogit"], dev["lam"], dev["u"], 0)
    b = gspn.forward(dev["x"], dev["wlogit"], dev["lam"], dev["u"], 0)
    assert torch.equal(a, b)


def test_large_plane_repeat_within_tolerance(cuda_device):
    wl = Workload("rep", 1, 2, 300, 200, 0, "f32")
    dev = to_dev(inputs.make_inputs(wl, 2), cuda_device)
    a = gspn.forward(dev["x"], dev["wlogit"], dev["lam"], dev["u"], 0).double()
    b = gspn.forward(dev["x"], dev["wlogit"], dev["lam"], dev["u"], 0).double()
    assert float((a - b).abs().max() / a.abs().max()) <= 1e-6
    assert gspn.check_device_status() == 0


def test_host_entry_matches_device_entry(cuda_device):
    for wl in [WORKLOADS["tiny16_global_f32"], Workload("h", 1, 2, 100, 70, 3, "bf16")]:
        inp = inputs.make_inputs(wl, 4)
        pinned = {"x": inp["x"].pin_memory(),
                  "wlogit": [t.pin_memory() for t in inp["wlogit"]],
                  "lam": [t.pin_memory() for t in inp["lam"]],
                  "u": [t.pin_memory() for t in inp["u"]]}
        yh = gspn.forward_host(pinned["x"], pinned["wlogit"], pinned["lam"], pinned["u"],
                               wl.group_len, out=torch.empty_like(inp["x"]).pin_memory(),
                               device=cuda_device)
        ref = oracle.forward(inp["x"], inp["wlogit"], inp["lam"], inp["u"], wl.group_len)
        assert rel_err(yh, ref) <= TOL[wl.dtype]


def test_bad_arguments_launch_nothing(cuda_device):
    wl = WORKLOADS["tiny16_global_f32"]
    dev = to_dev(inputs.make_inputs(wl, 0), cuda_device)
    y = torch.full_like(dev["x"], 7.0)
    with pytest.raises(gspn.GSPNError) as e:
        gspn.forward(dev["x"], dev["wlogit"], dev["lam"], dev["u"], -1, out=y)
    assert e.value.status == -5
    misaligned = torch.empty(dev["x"].numel() + 1, device=cuda_device)[1:].view_as(dev["x"])
    misaligned.copy_(dev["x"])
    with pytest.raises(gspn.GSPNError) as e:
        gspn.forward(misaligned, dev["wlogit"], dev["lam"], dev["u"], 0, out=y)
    assert e.value.status == -4
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())


def test_runs_on_a_side_stream(cuda_device):
    wl = Workload("s", 1, 2, 80, 90, 0, "f32")
    inp = inputs.make_inputs(wl, 5)
    dev = to_dev(inp, cuda_device)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y = gspn.forward(dev["x"], dev["wlogit"], dev["lam"], dev["u"], 0)
    s.synchronize()
    ref = oracle.forward(inp["x"], inp["wlogit"], inp["lam"], inp["u"], 0)
    assert rel_err(y, ref) <= TOL["f32"]


def test_launch_count_is_reported(cuda_device):
    wl = WORKLOADS["tiny16_global_f32"]
    dev = to_dev(inputs.make_inputs(wl, 0), cuda_device)
    gspn.forward(dev["x"], dev["wlogit"], dev["lam"], dev["u"], 0)
    assert gspn.last_launch_count() >= 1
