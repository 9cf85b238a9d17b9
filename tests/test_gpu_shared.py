"""gspn_forward_shared (channel-shared neighbour logits, [B,1,3,H,W]) against
the fp64 oracle run on the logits broadcast to every channel, on each of the
four kernels (whole-plane, line-chain, fused, line-sweep)."""
import numpy as np
import pytest
import torch

import oracle
from linear_spatial_propagation_line_b200 import gspn, inputs
from linear_spatial_propagation_line_b200.inputs import Workload

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}

CASES = [
    # (workload, kernel expected)
    (Workload("sh_small_f32", 2, 4, 16, 16, 0, "f32"), "small_plane_kernel"),
    (Workload("sh_local_bf16", 2, 6, 28, 28, 7, "bf16", logit_std=2.0), "small_plane_kernel"),
    (Workload("sh_chain_f32", 1, 3, 70, 131, 0, "f32"), "chain_kernel"),
    (Workload("sh_fused_bf16", 2, 4, 256, 512, 0, "bf16"), "fused_kernel"),
    (Workload("sh_fused_local_f32", 1, 3, 300, 256, 33, "f32"), "fused_kernel"),
    (Workload("sh_sweep_bf16", 2, 4, 256, 512, 0, "bf16"), "sweep_kernel"),
    (Workload("sh_sweep_local_f32", 1, 3, 300, 256, 33, "f32"), "sweep_kernel"),
]
PATHS = {"fused_kernel": gspn.PATH_FUSED, "sweep_kernel": gspn.PATH_SWEEP}


@pytest.mark.parametrize("wl,kernel", CASES, ids=[c[0].name for c in CASES])
def test_shared_logits_match_oracle(wl, kernel, cuda_device):
    gspn.debug_select_path(PATHS.get(kernel, gspn.PATH_AUTO))
    try:
        _check_shared(wl, kernel, cuda_device)
    finally:
        gspn.debug_select_path(gspn.PATH_AUTO)


def _check_shared(wl, kernel, cuda_device):
    inp = inputs.make_inputs(wl, 77)
    # one logit plane set per batch entry: take channel 0 of the drawn logits
    zs = [t[:, :1].contiguous() for t in inp["wlogit"]]
    dev = lambda t: t.to(cuda_device)
    y = gspn.forward_shared(dev(inp["x"]), [dev(t) for t in zs], [dev(t) for t in inp["lam"]],
                            [dev(t) for t in inp["u"]], wl.group_len)
    torch.cuda.synchronize()
    assert gspn.last_kernel_name() == kernel
    full = [t.expand(wl.B, wl.C, 3, wl.H, wl.W) for t in zs]
    ref = oracle.forward(inp["x"], full, inp["lam"], inp["u"], wl.group_len)
    yd = y.double().cpu().numpy()
    err = float(np.abs(yd - ref).max() / np.abs(ref).max())
    assert err <= TOL[wl.dtype], err
    # the same as gspn_forward on logits copied to every channel
    y2 = gspn.forward(dev(inp["x"]), [dev(t.contiguous()) for t in full],
                      [dev(t) for t in inp["lam"]], [dev(t) for t in inp["u"]], wl.group_len)
    torch.cuda.synchronize()
    err2 = float((y.double() - y2.double()).abs().max() / y2.double().abs().max())
    assert err2 <= (1e-6 if wl.dtype == "f32" else 8e-3), err2


def test_shared_rejects_per_channel_logits(cuda_device):
    wl = Workload("sh_bad", 1, 2, 8, 8, 0, "f32")
    inp = inputs.make_inputs(wl, 1)
    dev = lambda t: t.to(cuda_device)
    with pytest.raises(ValueError):
        gspn.forward_shared(dev(inp["x"]), [dev(t) for t in inp["wlogit"]],
                            [dev(t) for t in inp["lam"]], [dev(t) for t in inp["u"]], 0)
