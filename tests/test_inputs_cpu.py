"""The seeded synthetic-input recipe shared by the parity tests, smoke() and
bench.py (CPU only).

Every parity test compares the CUDA path and the oracle on the bytes
make_inputs() draws, and bench.py times the same recipe, so the recipe itself
is pinned here: the named workloads' shapes and distributions, the order of
the draws, seeded determinism and the cast to the storage dtype.
"""
import math

import pytest
import torch

from linear_spatial_propagation_line_b200 import inputs
from linear_spatial_propagation_line_b200.inputs import HEADLINE, WORKLOADS, Workload


def test_named_workloads():
    expect = {
        # name: (B, C, H, W, group_len, dtype)
        "tiny16_global_f32": (1, 4, 16, 16, 0, "f32"),
        "cls56_global_f32": (8, 96, 56, 56, 0, "f32"),
        "local28_g7_bf16": (32, 192, 28, 28, 7, "bf16"),
        "gen32_global_bf16": (32, 288, 32, 32, 0, "bf16"),
        "hires2048x1024_global_bf16": (1, 64, 2048, 1024, 0, "bf16"),
    }
    assert set(WORKLOADS) == set(expect)
    for name, (B, C, H, W, g, dt) in expect.items():
        wl = WORKLOADS[name]
        assert (wl.B, wl.C, wl.H, wl.W, wl.group_len, wl.dtype) == (B, C, H, W, g, dt), name
    assert WORKLOADS["local28_g7_bf16"].logit_std == 2.0
    assert (WORKLOADS["gen32_global_bf16"].lam_lo, WORKLOADS["gen32_global_bf16"].u_std) == (0.5, 0.5)


def test_headline_sizes():
    wl = WORKLOADS[HEADLINE]
    assert wl.pixch == 134_217_728
    # 1 x + 12 logits + 4 lambda + 4 u read, 1 y written, 2 bytes each
    assert wl.algorithmic_bytes() == 22 * 2 * 134_217_728 == 5_905_580_032


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_shapes_dtypes_and_layout(name):
    wl = WORKLOADS[name].with_(B=1, C=2, H=min(WORKLOADS[name].H, 40),
                               W=min(WORKLOADS[name].W, 48))
    inp = inputs.make_inputs(wl, seed=0)
    shape = (wl.B, wl.C, wl.H, wl.W)
    assert tuple(inp["x"].shape) == shape
    assert len(inp["wlogit"]) == len(inp["lam"]) == len(inp["u"]) == 4
    for d in range(4):
        assert tuple(inp["wlogit"][d].shape) == (wl.B, wl.C, 3, wl.H, wl.W)
        assert tuple(inp["lam"][d].shape) == shape
        assert tuple(inp["u"][d].shape) == shape
    for t in [inp["x"]] + inp["wlogit"] + inp["lam"] + inp["u"]:
        assert t.dtype == wl.torch_dtype and t.is_contiguous() and t.device.type == "cpu"


def test_seeded_determinism():
    wl = Workload("det", 2, 3, 17, 24, 0, "bf16")
    a = inputs.make_inputs(wl, seed=5)
    b = inputs.make_inputs(wl, seed=5)
    c = inputs.make_inputs(wl, seed=6)
    for k in ("x",):
        assert torch.equal(a[k], b[k]) and not torch.equal(a[k], c[k])
    for k in ("wlogit", "lam", "u"):
        for d in range(4):
            assert torch.equal(a[k][d], b[k][d])


def test_draw_order():
    """x first, then for each direction its logits, lambda and u, all in fp32
    from one generator, each then cast to the storage dtype."""
    wl = Workload("order", 1, 2, 9, 12, 0, "bf16", logit_std=1.5, lam_lo=0.25, lam_hi=0.75,
                  u_std=0.5)
    inp = inputs.make_inputs(wl, seed=11)
    g = torch.Generator().manual_seed(11)
    shape, zshape = (1, 2, 9, 12), (1, 2, 3, 9, 12)
    x = torch.empty(shape).normal_(0.0, 1.0, generator=g)
    assert torch.equal(inp["x"], x.to(torch.bfloat16))
    for d in range(4):
        z = torch.empty(zshape).normal_(0.0, 1.5, generator=g)
        lam = torch.empty(shape).uniform_(0.25, 0.75, generator=g)
        u = torch.empty(shape).normal_(0.0, 0.5, generator=g)
        assert torch.equal(inp["wlogit"][d], z.to(torch.bfloat16)), d
        assert torch.equal(inp["lam"][d], lam.to(torch.bfloat16)), d
        assert torch.equal(inp["u"][d], u.to(torch.bfloat16)), d


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_distributions(name):
    base = WORKLOADS[name]
    wl = base.with_(B=1, C=4, H=64, W=64)
    inp = inputs.make_inputs(wl, seed=0)
    n = wl.pixch

    def check_normal(t, std):
        t = t.double()
        tol = 6 * std / math.sqrt(t.numel())
        assert abs(float(t.mean())) < tol
        assert abs(float(t.std()) / std - 1.0) < 0.03

    check_normal(inp["x"], base.x_std)
    for d in range(4):
        check_normal(inp["wlogit"][d], base.logit_std)
        check_normal(inp["u"][d], base.u_std)
        lam = inp["lam"][d].double()
        # bf16 rounding may carry a value onto the interval's upper end
        assert float(lam.min()) >= base.lam_lo and float(lam.max()) <= base.lam_hi
        mid = (base.lam_lo + base.lam_hi) / 2
        assert abs(float(lam.mean()) - mid) < 6 * (base.lam_hi - base.lam_lo) / math.sqrt(12 * n)
