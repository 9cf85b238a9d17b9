"""gspn_forward_noalloc: the allocation-free entry point.

It runs the line-chain kernel with its fp32 accumulator in a fixed device
array that is part of the library image.  The GPU tests compare it with
gspn_forward (and, on small cases, the fp64 oracle) on two calls in a row,
so a second call that saw the first call's accumulation would fail.  The
file is named to run last, after every other GPU test has used the library.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from linear_spatial_propagation_line_b200 import gspn, inputs
from linear_spatial_propagation_line_b200 import build as gbuild
from linear_spatial_propagation_line_b200.inputs import Workload

TOL = {"f32": 1e-5, "bf16": 2e-2}
# Both entry points compute in fp32; they differ only in the order of rounding.
# bf16 outputs may land one bf16 step apart (2^-8 relative to max|y|).
AGREE = {"f32": 2e-6, "bf16": 8e-3}


def _err(a, b):
    a = a.detach().double().cpu().numpy()
    b = b.detach().double().cpu().numpy() if torch.is_tensor(b) else b
    assert np.isfinite(a).all()
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def _dev(inp, device):
    return {"x": inp["x"].to(device),
            "wlogit": [t.to(device) for t in inp["wlogit"]],
            "lam": [t.to(device) for t in inp["lam"]],
            "u": [t.to(device) for t in inp["u"]]}


# ---------------------------------------------------------------- host checks
def test_noalloc_rejects_oversize_before_any_device_call():
    gbuild.build()
    lib = gspn.load_library()
    arr4 = ctypes.c_void_p * 4
    base = [(1 << 36) + i * (1 << 32) for i in range(13)]
    y = 1 << 44

    def call(shape, dtype=0, x=base[0]):
        return lib.gspn_forward_noalloc(x, arr4(*base[1:5]), arr4(*base[5:9]),
                                        arr4(*base[9:13]), *shape, 0, dtype, None, y)

    limit = gspn.NOALLOC_MAX_ELEMENTS
    assert call((1, 2, 2048, 2049)) == -10  # 2 * 2048 * 2049 > 2^23
    assert call((1, 1, limit + 1, 1), dtype=1) == -10
    assert call((1, 1, 4, 4), x=0) == -1
    assert call((1, 1, 0, 4)) == -2
    assert call((1, 1, 4, 4), dtype=7) == -3
    assert call((1, 1, 4, 4), x=base[0] + 4) == -4
    assert "scratch" in gspn.status_string(-10)


# ----------------------------------------------------------------- GPU parity
CASES = [
    # (name, workload)
    ("tiny16_global_f32", inputs.WORKLOADS["tiny16_global_f32"]),
    ("ragged_f32", Workload("ragged_f32", 2, 3, 70, 131, 0, "f32")),
    ("local_g7_bf16", Workload("local_g7_bf16", 2, 8, 28, 28, 7, "bf16", logit_std=2.0)),
    ("tall_local_bf16", Workload("tall_local_bf16", 1, 2, 300, 40, 33, "bf16")),
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,wl", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_forward_and_oracle_two_calls(name, wl, cuda_device):
    ins = [inputs.make_inputs(wl, seed) for seed in (11, 12)]
    devs = [_dev(i, cuda_device) for i in ins]
    outs = [torch.empty_like(d["x"]) for d in devs]
    # two calls in a row on the same stream, different inputs
    for d, y in zip(devs, outs):
        gspn.forward_noalloc(d["x"], d["wlogit"], d["lam"], d["u"], wl.group_len, out=y)
    assert gspn.last_kernel_name() == "chain_kernel"
    for inp, d, y in zip(ins, devs, outs):
        y_ref = gspn.forward(d["x"], d["wlogit"], d["lam"], d["u"], wl.group_len)
        torch.cuda.synchronize()
        assert _err(y, y_ref) <= AGREE[wl.dtype], name
        ref = oracle.forward(inp["x"], inp["wlogit"], inp["lam"], inp["u"], wl.group_len)
        assert _err(y, ref) <= TOL[wl.dtype], name


@pytest.mark.gpu
def test_noalloc_at_the_scratch_limit_repeated(cuda_device):
    """B*C*H*W exactly at the limit (1 x 2 x 2048 x 2048 bf16), twice; the
    second call reuses the whole scratch.  Compared with gspn_forward (the
    fused kernel at this size) and, on one plane, with the oracle."""
    wl = Workload("limit_bf16", 1, 2, 2048, 2048, 0, "bf16")
    assert wl.pixch == gspn.NOALLOC_MAX_ELEMENTS
    inp = inputs.make_inputs(wl, 5, device=cuda_device, gen_device=cuda_device)
    y_ref = gspn.forward(inp["x"], inp["wlogit"], inp["lam"], inp["u"], 0)
    y1 = torch.empty_like(y_ref)
    y2 = torch.empty_like(y_ref)
    gspn.forward_noalloc(inp["x"], inp["wlogit"], inp["lam"], inp["u"], 0, out=y1)
    gspn.forward_noalloc(inp["x"], inp["wlogit"], inp["lam"], inp["u"], 0, out=y2)
    torch.cuda.synchronize()
    assert _err(y1, y_ref) <= AGREE["bf16"]
    assert _err(y2, y_ref) <= AGREE["bf16"]
    sel = lambda t: t[:, 1:2].cpu()
    ref = oracle.forward(sel(inp["x"]), [sel(t) for t in inp["wlogit"]],
                         [sel(t) for t in inp["lam"]], [sel(t) for t in inp["u"]], 0)
    assert _err(y2[:, 1:2], ref) <= TOL["bf16"]


@pytest.mark.gpu
def test_noalloc_interleaved_with_forward_on_a_side_stream(cuda_device):
    wl = Workload("side", 1, 4, 96, 160, 0, "f32")
    inp = _dev(inputs.make_inputs(wl, 3), cuda_device)
    s = torch.cuda.Stream(cuda_device)
    s.wait_stream(torch.cuda.current_stream(cuda_device))
    with torch.cuda.stream(s):
        a = gspn.forward_noalloc(inp["x"], inp["wlogit"], inp["lam"], inp["u"], 0)
        b = gspn.forward(inp["x"], inp["wlogit"], inp["lam"], inp["u"], 0)
        c = gspn.forward_noalloc(inp["x"], inp["wlogit"], inp["lam"], inp["u"], 0)
    s.synchronize()
    assert _err(a, b) <= AGREE["f32"]
    assert _err(c, b) <= AGREE["f32"]
