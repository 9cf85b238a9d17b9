"""C-ABI library checks that need no GPU: it builds, loads, exports every
symbol that include/gspn.h declares, and rejects bad arguments before any CUDA
call (validation runs on the host, so these calls never touch a device)."""
import ctypes
import os
import re

import pytest

from linear_spatial_propagation_line_b200 import build as gbuild
from linear_spatial_propagation_line_b200 import gspn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gspn.h")


@pytest.fixture(scope="module")
def lib():
    gbuild.build()
    return gspn.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(gspn_\w+)\s*\(", text, flags=re.M)))


def declared_macros():
    text = open(HEADER).read()
    return {m.group(1): int(m.group(2)) for m in
            re.finditer(r"#define\s+(GSPN_\w+)\s+\(?(-?\d+)\)?", text)}


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("gspn_forward", "gspn_forward_dir", "gspn_forward_host", "gspn_release",
                     "gspn_status_string", "gspn_last_cuda_error", "gspn_version",
                     "gspn_last_launch_count"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings_and_version(lib):
    macros = declared_macros()
    for name, code in macros.items():
        if name.startswith("GSPN_ERR_") or name == "GSPN_OK":
            s = gspn.status_string(code)
            assert s and s != "unknown status", name
    assert gspn.version() >= 100


def _fake_ptrs(base=0x10000000, n=13, stride=1 << 24):
    return [base + i * stride for i in range(n)]


def _call(x=None, z=None, l=None, u=None, shape=(1, 2, 8, 8), g=0, dtype=0, y=None):
    p = _fake_ptrs()
    x = p[0] if x is None else x
    z = p[1:5] if z is None else z
    l = p[5:9] if l is None else l
    u = p[9:13] if u is None else u
    y = 0x7f000000 if y is None else y
    lib = gspn.load_library()
    arr4 = ctypes.c_void_p * 4
    return lib.gspn_forward(x, arr4(*z), arr4(*l), arr4(*u), *shape, g, dtype, None, y)


def test_validation_rejects_before_launch(lib):
    assert _call(x=0) == -1
    assert _call(z=[0, 1 << 30, 1 << 31, 1 << 32]) == -1
    assert _call(y=0) == -1
    for bad in [(0, 1, 4, 4), (1, 0, 4, 4), (1, 1, 0, 4), (1, 1, 4, -3), (1, 1, 1 << 20, 1 << 20)]:
        assert _call(shape=bad) == -2, bad
    assert _call(dtype=2) == -3
    assert _call(x=0x10000008) == -4
    assert _call(y=0x7f000004) == -4
    assert _call(g=-1) == -5
    # y overlapping x
    assert _call(y=0x10000000 + 64) == -9


def test_forward_dir_rejects_bad_direction(lib):
    r = lib.gspn_forward_dir(0x1000, 0x2000, 0x3000, 0x4000, 1, 1, 4, 4, 0, 4, 0, None, 0x5000)
    assert r == -8
    r = lib.gspn_forward_dir(0x1000, 0x2000, 0x3000, 0x4000, 1, 1, 4, 4, 0, -1, 0, None, 0x5000)
    assert r == -8


def test_host_entry_validates_before_copying(lib):
    arr4 = ctypes.c_void_p * 4
    p = _fake_ptrs()
    r = lib.gspn_forward_host(p[0], arr4(*p[1:5]), arr4(*p[5:9]), arr4(*p[9:13]), 1, 1, 0, 4, 0,
                              0, None, 0x7f000000)
    assert r == -2
    r = lib.gspn_forward_host(0, arr4(*p[1:5]), arr4(*p[5:9]), arr4(*p[9:13]), 1, 1, 4, 4, 0, 0,
                              None, 0x7f000000)
    assert r == -1
