"""Seeded synthetic inputs for GSPN propagation.

This module holds no propagation arithmetic: it only draws random tensors.
It is the one module shared by the CUDA path's tests/benchmark and the CPU
oracle's tests, so both see identical stored bytes.

Recipe: ``torch.Generator`` seeded with ``seed`` draws, in this order and in
fp32, ``x`` and then for d = 0..3 ``wlogit[d]``, ``lam[d]``, ``u[d]``; each
tensor is then cast to the storage dtype.  ``N(m, s)`` means standard
deviation ``s``.  Shapes: x, lam[d], u[d]: [B,C,H,W]; wlogit[d]: [B,C,3,H,W].

The five named workloads stand in for the workloads GSPN is used on (the
ImageNet classifier's 56x56 stage, a local early stage at 28x28, a 32x32
generation latent, and the 16K x 8K image at 8x latent downsampling); no
dataset is involved.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    C: int
    H: int
    W: int
    group_len: int
    dtype: str          # storage dtype of every tensor: "f32" or "bf16"
    x_std: float = 1.0
    logit_std: float = 1.0
    lam_lo: float = 0.0
    lam_hi: float = 1.0
    u_std: float = 1.0

    @property
    def pixch(self) -> int:
        return self.B * self.C * self.H * self.W

    @property
    def esize(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def algorithmic_bytes(self) -> int:
        """Minimum HBM bytes: 1 x + 12 logits + 4 lambda + 4 u read, 1 y written."""
        return 22 * self.pixch * self.esize

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny16_global_f32", 1, 4, 16, 16, 0, "f32"),
        Workload("cls56_global_f32", 8, 96, 56, 56, 0, "f32"),
        Workload("local28_g7_bf16", 32, 192, 28, 28, 7, "bf16", logit_std=2.0),
        Workload("gen32_global_bf16", 32, 288, 32, 32, 0, "bf16", lam_lo=0.5, u_std=0.5),
        Workload("hires2048x1024_global_bf16", 1, 64, 2048, 1024, 0, "bf16"),
    ]
}

# The workload the throughput headline is quoted on.
HEADLINE = "hires2048x1024_global_bf16"


def make_inputs(wl: Workload, seed: int = 0, device: str = "cpu", gen_device: str = "cpu"):
    """Draw one batch of inputs for ``wl``.

    Returns a dict with ``x`` and lists ``wlogit``, ``lam``, ``u`` (length 4),
    all contiguous tensors of ``wl.torch_dtype`` on ``device``.  With
    ``gen_device="cpu"`` (the default) the values are reproducible across
    machines; ``gen_device="cuda"`` draws on the GPU (same distributions,
    different values) for fast benchmark set-up.
    """
    g = torch.Generator(gen_device)
    g.manual_seed(seed)
    shape = (wl.B, wl.C, wl.H, wl.W)
    zshape = (wl.B, wl.C, 3, wl.H, wl.W)

    def normal(shp, std):
        t = torch.empty(shp, dtype=torch.float32, device=gen_device)
        t.normal_(0.0, std, generator=g)
        return t.to(device=device, dtype=wl.torch_dtype).contiguous()

    def uniform(shp, lo, hi):
        t = torch.empty(shp, dtype=torch.float32, device=gen_device)
        t.uniform_(lo, hi, generator=g)
        return t.to(device=device, dtype=wl.torch_dtype).contiguous()

    x = normal(shape, wl.x_std)
    wlogit, lam, u = [], [], []
    for _d in range(4):
        wlogit.append(normal(zshape, wl.logit_std))
        lam.append(uniform(shape, wl.lam_lo, wl.lam_hi))
        u.append(normal(shape, wl.u_std))
    return {"x": x, "wlogit": wlogit, "lam": lam, "u": u}
