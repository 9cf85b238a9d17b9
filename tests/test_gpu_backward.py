"""GPU parity of the backward pass (gspn_backward through the C ABI) against
the fp64 oracle's backward, which is pinned by finite differences.

Error metric per output tensor: max|g_gpu - g_ref| / max|g_ref|.  Bars: 1e-5
for fp32 storage; 2e-2 for bf16 storage (each output rounded once)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from linear_spatial_propagation_line_b200 import gspn, inputs
from linear_spatial_propagation_line_b200 import build as gbuild
from linear_spatial_propagation_line_b200.inputs import Workload

TOL = {"f32": 1e-5, "bf16": 2e-2}


def _err(a, b):
    a = a.detach().double().cpu().numpy()
    assert np.isfinite(a).all()
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


CASES = [
    Workload("bw_tiny_f32", 1, 4, 16, 16, 0, "f32"),
    Workload("bw_rect_f32", 2, 3, 37, 70, 0, "f32"),
    Workload("bw_local_f32", 1, 3, 28, 28, 7, "f32", logit_std=2.0),
    Workload("bw_tall_bf16", 1, 2, 130, 33, 0, "bf16"),
    Workload("bw_local_bf16", 2, 4, 28, 28, 7, "bf16", logit_std=2.0),
    Workload("bw_line_f32", 1, 2, 1, 50, 0, "f32"),
    Workload("bw_wide_bf16", 1, 2, 64, 600, 0, "bf16"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("wl", CASES, ids=[c.name for c in CASES])
def test_backward_matches_oracle(wl, cuda_device):
    inp = inputs.make_inputs(wl, 31)
    g = torch.Generator().manual_seed(5)
    gy = torch.randn((wl.B, wl.C, wl.H, wl.W), generator=g).to(wl.torch_dtype)
    dev = lambda t: t.to(cuda_device)
    dx, dz, dl, du = gspn.backward(dev(inp["x"]), [dev(t) for t in inp["wlogit"]],
                                   [dev(t) for t in inp["lam"]], [dev(t) for t in inp["u"]],
                                   dev(gy), wl.group_len)
    torch.cuda.synchronize()
    assert gspn.last_kernel_name() == "backward_kernel"
    rx, rz, rl, ru = oracle.backward(inp["x"], inp["wlogit"], inp["lam"], inp["u"], gy,
                                     wl.group_len)
    tol = TOL[wl.dtype]
    assert _err(dx, rx) <= tol, "dx"
    for d in range(4):
        assert _err(dl[d], rl[d]) <= tol, f"dlam[{d}]"
        assert _err(du[d], ru[d]) <= tol, f"du[{d}]"
        if np.abs(rz[d]).max() > 0:
            assert _err(dz[d], rz[d]) <= tol, f"dwlogit[{d}]"
        else:
            assert float(dz[d].abs().max()) == 0.0


@pytest.mark.gpu
def test_autograd_wrapper_gives_the_same_gradients(cuda_device):
    wl = Workload("ag", 1, 2, 20, 24, 0, "f32")
    inp = inputs.make_inputs(wl, 3)
    leaves = [inp["x"]] + inp["wlogit"] + inp["lam"] + inp["u"]
    leaves = [t.to(cuda_device).requires_grad_(True) for t in leaves]
    x, z, l, u = leaves[0], leaves[1:5], leaves[5:9], leaves[9:13]
    y = gspn.gspn_autograd(x, z, l, u, 0)
    gy = torch.randn_like(y)
    y.backward(gy)
    dx, dz, dl, du = gspn.backward(x.detach(), [t.detach() for t in z], [t.detach() for t in l],
                                   [t.detach() for t in u], gy, 0)
    torch.cuda.synchronize()
    # dx sums four directions with atomic adds, so only its rounding order differs
    torch.testing.assert_close(x.grad, dx, rtol=1e-6, atol=1e-6)
    for d in range(4):
        assert torch.equal(z[d].grad, dz[d]) and torch.equal(l[d].grad, dl[d])
        assert torch.equal(u[d].grad, du[d])


def test_backward_rejects_bad_arguments_before_any_device_call():
    gbuild.build()
    lib = gspn.load_library()
    arr4 = ctypes.c_void_p * 4
    base = [(1 << 36) + i * (1 << 32) for i in range(30)]
    x, gy, dx = base[0], base[1], base[2]
    z, l, u = base[3:7], base[7:11], base[11:15]
    dz, dl, du = base[15:19], base[19:23], base[23:27]

    def call(**kw):
        a = dict(x=x, gy=gy, dx=dx, z=z, l=l, u=u, dz=dz, dl=dl, du=du, shape=(1, 2, 8, 8))
        a.update(kw)
        return lib.gspn_backward(a["x"], arr4(*a["z"]), arr4(*a["l"]), arr4(*a["u"]), a["gy"],
                                 *a["shape"], 0, 0, None, a["dx"], arr4(*a["dz"]),
                                 arr4(*a["dl"]), arr4(*a["du"]))

    assert call(gy=0) == -1
    assert call(dx=0) == -1
    assert call(dz=[dz[0], 0, dz[2], dz[3]]) == -1
    assert call(shape=(1, 0, 8, 8)) == -2
    assert call(gy=gy + 4) == -4
    assert call(du=[du[0], du[1], du[2], x + 64]) == -9   # output overlapping x
    assert call(dl=[dl[0], dl[0], dl[2], dl[3]]) == -9    # two outputs overlapping
