"""fp64 CPU oracle for GSPN 4-direction line-scan propagation.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the CUDA library under ``linear_spatial_propagation_line_b200``) never calls
it, and the two share no code: this package holds a plain C++ loop
(``gspn_oracle.cpp``) and a brute-force unrolled-matrix form (``dense_g.py``).

Sources (GSPN, arXiv 2501.12381, as walked through on the CSDN page
"GSPN——在convolution基础上并行序列建模"):

* section "方法": the recurrence h_i = w_i h_{i-1} + lambda_i * x_i, output
  y_i = u_i * h_i, and the unrolled lower-triangular matrix G;
* section "如何设计一个高效的传播层": three-neighbour tridiagonal w_i and four
  scan directions;
* section "行随机矩阵": sigmoid then per-row normalisation over the row's
  non-zeros;
* section "全局与局部GSPN": local groups along the scan axis.

Every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` (unrolled form, row-stochastic invariant, bound,
linearity, textbook special cases, direction symmetries, a hand-computed
example in ``tests/golden/``).
"""
from __future__ import annotations

import ctypes
import os
import pathlib
import subprocess
import threading

import numpy as np

_HERE = pathlib.Path(__file__).resolve().parent
_SRC = _HERE / "gspn_oracle.cpp"
_BUILD_DIR = _HERE / "_build"
_LIB_PATH = _BUILD_DIR / "libgspn_oracle.so"
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> pathlib.Path:
    """Compile the C++ oracle into ``oracle/_build/libgspn_oracle.so``."""
    if not force and _LIB_PATH.exists() and _LIB_PATH.stat().st_mtime >= _SRC.stat().st_mtime:
        return _LIB_PATH
    _BUILD_DIR.mkdir(exist_ok=True)
    tmp = _LIB_PATH.with_suffix(f".{os.getpid()}.tmp.so")
    cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
           "-ffp-contract=off", str(_SRC), "-o", str(tmp)]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(str(build()))
            i64 = ctypes.c_int64
            lib.gspn_oracle_hidden.argtypes = [_dp, _dp, _dp, i64, i64, i64, i64, i64,
                                               ctypes.c_int, ctypes.c_int, _dp]
            lib.gspn_oracle_hidden.restype = ctypes.c_int
            lib.gspn_oracle_hidden_band.argtypes = [_dp, _dp, _dp, i64, i64, i64, i64, i64, i64,
                                                    ctypes.c_int, ctypes.c_int, _dp]
            lib.gspn_oracle_hidden_band.restype = ctypes.c_int
            lib.gspn_oracle_weights.argtypes = [_dp, i64, i64, i64, i64, ctypes.c_int, _dp]
            lib.gspn_oracle_weights.restype = ctypes.c_int
            arr4 = _dp * 4
            lib.gspn_oracle_forward.argtypes = [_dp, arr4, arr4, arr4, i64, i64, i64, i64, i64,
                                                ctypes.c_int, _dp]
            lib.gspn_oracle_forward.restype = ctypes.c_int
            lib.gspn_oracle_backward.argtypes = [_dp, arr4, arr4, arr4, _dp, i64, i64, i64, i64,
                                                 i64, ctypes.c_int, _dp, arr4, arr4, arr4]
            lib.gspn_oracle_backward.restype = ctypes.c_int
            lib.gspn_oracle_default_threads.argtypes = []
            lib.gspn_oracle_default_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def as_f64(a) -> np.ndarray:
    """Exact conversion of a stored tensor (numpy or torch, fp32/bf16/fp64) to a
    contiguous float64 numpy array."""
    if hasattr(a, "detach"):  # torch tensor: go through torch for bf16
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def default_threads() -> int:
    return int(_load().gspn_oracle_default_threads())


def hidden(x, wlogit_d, lam_d, d: int, group_len: int = 0, nthreads: int = 0) -> np.ndarray:
    """h_d for direction ``d``; x, lam_d: [B,C,H,W], wlogit_d: [B,C,3,H,W]."""
    x = as_f64(x)
    z = as_f64(wlogit_d)
    lam = as_f64(lam_d)
    B, C, H, W = x.shape
    assert z.shape == (B, C, 3, H, W) and lam.shape == x.shape
    h = np.empty_like(x)
    rc = _load().gspn_oracle_hidden(_ptr(x), _ptr(z), _ptr(lam), B, C, H, W, int(group_len),
                                    int(d), int(nthreads), _ptr(h))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments (rc={rc})")
    return h


def hidden_band(x, wlogit_d, lam_d, d: int, radius: int, group_len: int = 0,
                nthreads: int = 0) -> np.ndarray:
    """h_d with a (2 radius + 1)-neighbour band instead of three neighbours;
    wlogit_d: [B,C,2 radius + 1,H,W] (slot s = orthogonal offset s - radius).
    radius = 1 is hidden(); radius >= K - 1 links every pixel to the whole
    previous line."""
    x = as_f64(x)
    z = as_f64(wlogit_d)
    lam = as_f64(lam_d)
    B, C, H, W = x.shape
    assert z.shape == (B, C, 2 * radius + 1, H, W) and lam.shape == x.shape
    h = np.empty_like(x)
    rc = _load().gspn_oracle_hidden_band(_ptr(x), _ptr(z), _ptr(lam), B, C, H, W, int(radius),
                                         int(group_len), int(d), int(nthreads), _ptr(h))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments (rc={rc})")
    return h


def weights(wlogit_d, d: int) -> np.ndarray:
    """Normalised tridiagonal weights [B,C,3,H,W] of direction ``d``."""
    z = as_f64(wlogit_d)
    B, C, three, H, W = z.shape
    assert three == 3
    w = np.empty_like(z)
    rc = _load().gspn_oracle_weights(_ptr(z), B, C, H, W, int(d), _ptr(w))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments (rc={rc})")
    return w


def forward(x, wlogit, lam, u, group_len: int = 0, nthreads: int = 0) -> np.ndarray:
    """y = sum_d u_d * h_d in fp64; wlogit, lam, u are length-4 sequences."""
    x = as_f64(x)
    B, C, H, W = x.shape
    zs = [as_f64(t) for t in wlogit]
    ls = [as_f64(t) for t in lam]
    us = [as_f64(t) for t in u]
    for d in range(4):
        assert zs[d].shape == (B, C, 3, H, W), zs[d].shape
        assert ls[d].shape == x.shape and us[d].shape == x.shape
    arr4 = _dp * 4
    y = np.empty_like(x)
    rc = _load().gspn_oracle_forward(_ptr(x), arr4(*[_ptr(a) for a in zs]),
                                     arr4(*[_ptr(a) for a in ls]), arr4(*[_ptr(a) for a in us]),
                                     B, C, H, W, int(group_len), int(nthreads), _ptr(y))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments (rc={rc})")
    return y


def backward(x, wlogit, lam, u, gy, group_len: int = 0, nthreads: int = 0):
    """Gradients of L = sum(gy * y) in fp64 (chain rule on the forward
    definition; the walkthrough's section "反向传播" describes the adjoint
    flowing back from later lines).  Returns (dx, dwlogit[4], dlam[4], du[4])."""
    x = as_f64(x)
    gy = as_f64(gy)
    B, C, H, W = x.shape
    assert gy.shape == x.shape
    zs = [as_f64(t) for t in wlogit]
    ls = [as_f64(t) for t in lam]
    us = [as_f64(t) for t in u]
    dx = np.empty_like(x)
    dz = [np.empty_like(z) for z in zs]
    dl = [np.empty_like(x) for _ in range(4)]
    du = [np.empty_like(x) for _ in range(4)]
    arr4 = _dp * 4
    rc = _load().gspn_oracle_backward(_ptr(x), arr4(*[_ptr(a) for a in zs]),
                                      arr4(*[_ptr(a) for a in ls]), arr4(*[_ptr(a) for a in us]),
                                      _ptr(gy), B, C, H, W, int(group_len), int(nthreads),
                                      _ptr(dx), arr4(*[_ptr(a) for a in dz]),
                                      arr4(*[_ptr(a) for a in dl]), arr4(*[_ptr(a) for a in du]))
    if rc != 0:
        raise ValueError(f"oracle rejected arguments (rc={rc})")
    return dx, dz, dl, du
