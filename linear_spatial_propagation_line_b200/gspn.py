"""Python binding of the GSPN C ABI (``include/gspn.h``).

Argument marshalling only: tensors are checked and turned into raw pointers,
and every step of the propagation runs in the CUDA library
``_lib/libgspn_b200.so``.  There is no CPU or PyTorch fallback: if the
library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import threading

import torch

from . import build as _build

GSPN_F32 = 0
GSPN_BF16 = 1
_DTYPES = {torch.float32: GSPN_F32, torch.bfloat16: GSPN_BF16}

# Largest B*C*H*W of forward_noalloc (GSPN_NOALLOC_MAX_ELEMENTS).
NOALLOC_MAX_ELEMENTS = 1 << 23

_lock = threading.Lock()
_lib = None


class GSPNError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"gspn status {status}: {message}")
        self.status = status


def library_path():
    return _build.LIB_PATH


def load_library():
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = _build.LIB_PATH
        if not path.exists():
            raise RuntimeError(
                f"GSPN CUDA library not found at {path}; build it with "
                "`python -m linear_spatial_propagation_line_b200.build`")
        lib = ctypes.CDLL(str(path))
        vp, i64, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        arr4 = vp * 4
        lib.gspn_forward.argtypes = [vp, arr4, arr4, arr4, i64, i64, i64, i64, i64, ci, vp, vp]
        lib.gspn_forward.restype = ci
        lib.gspn_forward_dir.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, ci, ci, vp, vp]
        lib.gspn_forward_dir.restype = ci
        lib.gspn_forward_host.argtypes = [vp, arr4, arr4, arr4, i64, i64, i64, i64, i64, ci, vp,
                                          vp]
        lib.gspn_forward_host.restype = ci
        lib.gspn_forward_shared.argtypes = [vp, arr4, arr4, arr4, i64, i64, i64, i64, i64, ci,
                                            vp, vp]
        lib.gspn_forward_shared.restype = ci
        lib.gspn_backward.argtypes = [vp, arr4, arr4, arr4, vp, i64, i64, i64, i64, i64, ci, vp,
                                      vp, arr4, arr4, arr4]
        lib.gspn_backward.restype = ci
        lib.gspn_forward_noalloc.argtypes = [vp, arr4, arr4, arr4, i64, i64, i64, i64, i64, ci,
                                             vp, vp]
        lib.gspn_forward_noalloc.restype = ci
        for name in ("gspn_last_launch_count", "gspn_release", "gspn_version"):
            getattr(lib, name).argtypes = []
            getattr(lib, name).restype = ci
        lib.gspn_status_string.argtypes = [ci]
        lib.gspn_status_string.restype = ctypes.c_char_p
        lib.gspn_last_cuda_error.argtypes = []
        lib.gspn_last_cuda_error.restype = ctypes.c_char_p
        lib.gspn_set_timing_events.argtypes = [vp, vp]
        lib.gspn_set_timing_events.restype = ci
        lib.gspn_last_kernel_name.argtypes = []
        lib.gspn_last_kernel_name.restype = ctypes.c_char_p
        lib.gspn_check_device_status.argtypes = [vp]
        lib.gspn_check_device_status.restype = ci
        lib.gspn_debug_force_timeout.argtypes = [i64]
        lib.gspn_debug_force_timeout.restype = ci
        lib.gspn_debug_select_path.argtypes = [ci]
        lib.gspn_debug_select_path.restype = ci
        _lib = lib
        return lib


def _check(status: int):
    if status != 0:
        lib = load_library()
        msg = lib.gspn_status_string(status).decode()
        if status == -6:
            msg += ": " + lib.gspn_last_cuda_error().decode()
        raise GSPNError(status, msg)


def status_string(status: int) -> str:
    return load_library().gspn_status_string(status).decode()


def version() -> int:
    return load_library().gspn_version()


def last_launch_count() -> int:
    """Kernels launched by this thread's most recent successful forward call."""
    return load_library().gspn_last_launch_count()


def set_timing_events(begin=None, end=None):
    """Record torch.cuda.Event ``begin``/``end`` around the dominant kernel of
    every later forward call on this thread (None, None stops)."""
    b = ctypes.c_void_p(begin.cuda_event) if begin is not None else None
    e = ctypes.c_void_p(end.cuda_event) if end is not None else None
    _check(load_library().gspn_set_timing_events(b, e))


def last_kernel_name() -> str:
    return load_library().gspn_last_kernel_name().decode()


def check_device_status(stream=None, device=None) -> int:
    """Synchronise and return GSPN_OK (0) or GSPN_ERR_TIMEOUT (-7) if a bounded
    device-side wait expired since the last check."""
    lib = load_library()
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(device):
        return lib.gspn_check_device_status(_stream_handle(device, stream))


def debug_force_timeout(timeout_ns: int):
    """Make the next large-plane launch on this thread expire a bounded wait."""
    _check(load_library().gspn_debug_force_timeout(int(timeout_ns)))


PATH_AUTO, PATH_FUSED, PATH_SWEEP = 0, 1, 2


def debug_select_path(path: int):
    """Choose the large-plane kernel for later calls on this thread:
    PATH_AUTO or PATH_FUSED (the fused kernel) or PATH_SWEEP (the line-sweep
    kernel); planes outside a kernel's constraints fall back to the line-chain
    kernel."""
    _check(load_library().gspn_debug_select_path(int(path)))


def release():
    """Free the current device's workspace and staging buffers."""
    _check(load_library().gspn_release())


def _shape_of(x):
    if x.dim() != 4:
        raise ValueError("x must be [B,C,H,W]")
    return tuple(int(s) for s in x.shape)


def _validate(x, wlogit, lam, u, dirs, device_kind):
    B, C, H, W = _shape_of(x)
    if x.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {x.dtype}")
    tensors = [x]
    for d in dirs:
        if tuple(wlogit[d].shape) != (B, C, 3, H, W):
            raise ValueError(f"wlogit[{d}] must be [B,C,3,H,W], got {tuple(wlogit[d].shape)}")
        for name, t in (("lam", lam[d]), ("u", u[d])):
            if tuple(t.shape) != (B, C, H, W):
                raise ValueError(f"{name}[{d}] must be [B,C,H,W], got {tuple(t.shape)}")
        tensors += [wlogit[d], lam[d], u[d]]
    for t in tensors:
        if t.dtype != x.dtype:
            raise TypeError("every tensor must have x's dtype")
        if not t.is_contiguous():
            raise ValueError("every tensor must be contiguous")
        if device_kind == "cuda" and (not t.is_cuda or t.device != x.device):
            raise ValueError("every tensor must be on x's CUDA device")
        if device_kind == "cpu" and t.is_cuda:
            raise ValueError("forward_host takes host tensors")
    return B, C, H, W


def _stream_handle(device, stream):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def forward(x, wlogit, lam, u, group_len: int = 0, out=None, stream=None):
    """y = sum_d u[d] * h_d on CUDA tensors (see include/gspn.h)."""
    lib = load_library()
    B, C, H, W = _validate(x, wlogit, lam, u, range(4), "cuda")
    y = torch.empty_like(x) if out is None else out
    _validate(y, wlogit, lam, u, [], "cuda")
    arr4 = ctypes.c_void_p * 4
    with torch.cuda.device(x.device):
        st = _stream_handle(x.device, stream)
        _check(lib.gspn_forward(x.data_ptr(), arr4(*[t.data_ptr() for t in wlogit]),
                                arr4(*[t.data_ptr() for t in lam]),
                                arr4(*[t.data_ptr() for t in u]), B, C, H, W, int(group_len),
                                _DTYPES[x.dtype], st, y.data_ptr()))
    return y


def forward_noalloc(x, wlogit, lam, u, group_len: int = 0, out=None, stream=None):
    """gspn_forward_noalloc: forward() without any device allocation inside
    the library.  The accumulator is a fixed per-device array of
    NOALLOC_MAX_ELEMENTS fp32 values, so B*C*H*W is limited to that, and calls
    on one device must not overlap on the GPU.  Pass ``out`` to keep the call
    itself free of allocations."""
    lib = load_library()
    B, C, H, W = _validate(x, wlogit, lam, u, range(4), "cuda")
    y = torch.empty_like(x) if out is None else out
    _validate(y, wlogit, lam, u, [], "cuda")
    arr4 = ctypes.c_void_p * 4
    with torch.cuda.device(x.device):
        st = _stream_handle(x.device, stream)
        _check(lib.gspn_forward_noalloc(x.data_ptr(), arr4(*[t.data_ptr() for t in wlogit]),
                                        arr4(*[t.data_ptr() for t in lam]),
                                        arr4(*[t.data_ptr() for t in u]), B, C, H, W,
                                        int(group_len), _DTYPES[x.dtype], st, y.data_ptr()))
    return y


def forward_shared(x, wlogit, lam, u, group_len: int = 0, out=None, stream=None):
    """forward() with channel-shared logits: wlogit[d] is [B,1,3,H,W]."""
    lib = load_library()
    B, C, H, W = _shape_of(x)
    for d in range(4):
        if tuple(wlogit[d].shape) != (B, 1, 3, H, W):
            raise ValueError(f"wlogit[{d}] must be [B,1,3,H,W], got {tuple(wlogit[d].shape)}")
    # the per-channel checks of _validate on a broadcast view of the logits
    _validate(x, [t.expand(B, C, 3, H, W) for t in wlogit], lam, u, [], "cuda")
    for t in list(wlogit) + list(lam) + list(u):
        if t.dtype != x.dtype or not t.is_contiguous() or not t.is_cuda or t.device != x.device:
            raise ValueError("every tensor must be contiguous, on x's device, with x's dtype")
    for d in range(4):
        if tuple(lam[d].shape) != (B, C, H, W) or tuple(u[d].shape) != (B, C, H, W):
            raise ValueError("lam[d], u[d] must be [B,C,H,W]")
    y = torch.empty_like(x) if out is None else out
    arr4 = ctypes.c_void_p * 4
    with torch.cuda.device(x.device):
        st = _stream_handle(x.device, stream)
        _check(lib.gspn_forward_shared(x.data_ptr(), arr4(*[t.data_ptr() for t in wlogit]),
                                       arr4(*[t.data_ptr() for t in lam]),
                                       arr4(*[t.data_ptr() for t in u]), B, C, H, W,
                                       int(group_len), _DTYPES[x.dtype], st, y.data_ptr()))
    return y


def backward(x, wlogit, lam, u, gy, group_len: int = 0, stream=None):
    """Gradients of sum(gy * forward(x, wlogit, lam, u)) with respect to every
    input, on CUDA tensors: returns (dx, [dwlogit_d], [dlam_d], [du_d])."""
    lib = load_library()
    B, C, H, W = _validate(x, wlogit, lam, u, range(4), "cuda")
    _validate(gy, wlogit, lam, u, [], "cuda")
    if gy.dtype != x.dtype or tuple(gy.shape) != tuple(x.shape) or not gy.is_contiguous():
        raise ValueError("gy must be a contiguous tensor like x")
    dx = torch.empty_like(x)
    dz = [torch.empty_like(t) for t in wlogit]
    dl = [torch.empty_like(t) for t in lam]
    du = [torch.empty_like(t) for t in u]
    arr4 = ctypes.c_void_p * 4
    with torch.cuda.device(x.device):
        st = _stream_handle(x.device, stream)
        _check(lib.gspn_backward(x.data_ptr(), arr4(*[t.data_ptr() for t in wlogit]),
                                 arr4(*[t.data_ptr() for t in lam]),
                                 arr4(*[t.data_ptr() for t in u]), gy.data_ptr(), B, C, H, W,
                                 int(group_len), _DTYPES[x.dtype], st, dx.data_ptr(),
                                 arr4(*[t.data_ptr() for t in dz]),
                                 arr4(*[t.data_ptr() for t in dl]),
                                 arr4(*[t.data_ptr() for t in du])))
    return dx, dz, dl, du


class GSPNFunction(torch.autograd.Function):
    """Autograd wrapper: forward() runs gspn_forward, backward() gspn_backward.
    Inputs: x, then the four logits, the four lambdas, the four u tensors."""

    @staticmethod
    def forward(ctx, group_len, x, *params):
        wlogit, lam, u = list(params[0:4]), list(params[4:8]), list(params[8:12])
        ctx.group_len = int(group_len)
        ctx.save_for_backward(x, *params)
        return forward(x.contiguous(), [t.contiguous() for t in wlogit],
                       [t.contiguous() for t in lam], [t.contiguous() for t in u], group_len)

    @staticmethod
    def backward(ctx, gy):
        x, *params = ctx.saved_tensors
        wlogit, lam, u = list(params[0:4]), list(params[4:8]), list(params[8:12])
        dx, dz, dl, du = backward(x, wlogit, lam, u, gy.contiguous(), ctx.group_len)
        return (None, dx, *dz, *dl, *du)


def gspn_autograd(x, wlogit, lam, u, group_len: int = 0):
    """y = sum_d u_d * h_d with gradients for every input (torch autograd)."""
    return GSPNFunction.apply(int(group_len), x, *wlogit, *lam, *u)


def forward_dir(x, wlogit_d, lam_d, u_d, d: int, group_len: int = 0, out=None, stream=None):
    """y = u_d * h_d for one direction d on CUDA tensors."""
    lib = load_library()
    z = [wlogit_d] * 4
    la = [lam_d] * 4
    uu = [u_d] * 4
    B, C, H, W = _validate(x, z, la, uu, [0], "cuda")
    y = torch.empty_like(x) if out is None else out
    with torch.cuda.device(x.device):
        st = _stream_handle(x.device, stream)
        _check(lib.gspn_forward_dir(x.data_ptr(), wlogit_d.data_ptr(), lam_d.data_ptr(),
                                    u_d.data_ptr(), B, C, H, W, int(group_len), int(d),
                                    _DTYPES[x.dtype], st, y.data_ptr()))
    return y


def forward_host(x, wlogit, lam, u, group_len: int = 0, out=None, device=None, stream=None):
    """gspn_forward_host on CPU tensors (pinned memory makes the copies
    asynchronous); returns y on the host, ready when the call returns."""
    lib = load_library()
    B, C, H, W = _validate(x, wlogit, lam, u, range(4), "cpu")
    y = torch.empty_like(x) if out is None else out
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    arr4 = ctypes.c_void_p * 4
    with torch.cuda.device(device):
        st = _stream_handle(device, stream)
        _check(lib.gspn_forward_host(x.data_ptr(), arr4(*[t.data_ptr() for t in wlogit]),
                                     arr4(*[t.data_ptr() for t in lam]),
                                     arr4(*[t.data_ptr() for t in u]), B, C, H, W,
                                     int(group_len), _DTYPES[x.dtype], st, y.data_ptr()))
    return y


def raw_forward(ptrs: dict, shape, group_len: int, dtype: int, stream_handle: int) -> int:
    """Direct C-ABI call on raw device pointers (for callers that manage their
    own buffers); returns the status code without raising."""
    lib = load_library()
    arr4 = ctypes.c_void_p * 4
    B, C, H, W = shape
    return lib.gspn_forward(ptrs["x"], arr4(*ptrs["wlogit"]), arr4(*ptrs["lam"]),
                            arr4(*ptrs["u"]), B, C, H, W, int(group_len), int(dtype),
                            ctypes.c_void_p(stream_handle), ptrs["y"])
