"""Host-side checks of the C ABI (no GPU needed).

The library must load, export every function declared in include/lapsum.h,
reject invalid arguments on the host before any CUDA call, and size its
workspace consistently.
"""
import ctypes
import os
import re

import pytest

import sparse_selection_primitive_b200 as L
from sparse_selection_primitive_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return L._lib()


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(lapsum_[a-z_0-9]+)\s*\(", text,
                            flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 10, names
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_abi_version_and_status_strings(lib):
    assert lib.lapsum_abi_version() == 1
    for code in range(6):
        assert lib.lapsum_status_string(code)
    assert lib.lapsum_status_string(99) == b"unknown status"


def test_invalid_arguments_rejected_on_host(lib):
    f = lib.lapsum_forward
    ws = ctypes.c_void_p(256)  # never dereferenced: every call below fails validation first
    d = ctypes.c_void_p(4096)
    # null pointers
    assert f(None, 8, d, d, None, 1, 8, 2.0, 0.1, 0, 0, ws, 1 << 20, None) == 1
    # B < 1, n < 1, ld < n
    assert f(d, 8, d, d, None, 0, 8, 2.0, 0.1, 0, 0, ws, 1 << 20, None) == 1
    assert f(d, 8, d, d, None, 1, 0, 0.5, 0.1, 0, 0, ws, 1 << 20, None) == 1
    assert f(d, 4, d, d, None, 1, 8, 2.0, 0.1, 0, 0, ws, 1 << 20, None) == 1
    # k outside (0, n), t <= 0, non-finite
    for k, t in [(0.0, 0.1), (8.0, 0.1), (-1.0, 0.1), (2.0, 0.0), (2.0, -1.0),
                 (float("nan"), 0.1), (2.0, float("inf"))]:
        assert f(d, 8, d, d, None, 1, 8, k, t, 0, 0, ws, 1 << 20, None) == 1
    # bad path code / unknown flag bits
    assert f(d, 8, d, d, None, 1, 8, 2.0, 0.1, 7, 0, ws, 1 << 20, None) == 1
    assert f(d, 8, d, d, None, 1, 8, 2.0, 0.1, 0x1000, 0, ws, 1 << 20, None) == 1
    # workspace: null, misaligned, too small
    assert f(d, 8, d, d, None, 1, 8, 2.0, 0.1, 0, 0, None, 1 << 20, None) == 2
    assert f(d, 8, d, d, None, 1, 8, 2.0, 0.1, 0, 0, ctypes.c_void_p(257), 1 << 20, None) == 2
    assert f(d, 8, d, d, None, 1, 8, 2.0, 0.1, 0, 0, ws, 16, None) == 2
    b = lib.lapsum_backward
    assert b(None, 8, d, d, d, 1, 8, 0.1, ws, 1 << 20, None) == 1
    assert b(d, 8, d, d, d, 1, 8, 0.0, ws, 1 << 20, None) == 1
    assert b(d, 8, d, d, d, 1, 8000, 0.1, ws, 1 << 20, None) == 1  # ld < n
    assert b(d, 8000, d, d, d, 1, 8000, 0.1, None, 1 << 20, None) == 2


def test_workspace_sizes(lib):
    wb = L.workspace_bytes
    assert wb(0, 10, 1.0) == 0 and wb(1, 0, 1.0) == 0
    assert wb(1, 10, 1.0, path=9) == 0
    # sizes grow with the problem and are multiples of 256
    for B, n in [(1, 1024), (16384, 256), (256, 65536), (1, 3342336), (1, 10**8)]:
        s = wb(B, n, 1.0)
        assert s > 0 and s % 256 == 0
        assert int(lib.lapsum_backward_workspace_bytes(B, n)) <= s
    # the radix path holds two key buffers; the bracket path holds two band buffers
    assert wb(256, 65536, 1024.0) >= 2 * 256 * 65536 * 4
    assert wb(1, 10**8, 1e5) >= 2 * 10**8 * 4


def test_new_entry_points_reject_bad_arguments_on_host(lib):
    """Per-row budgets, the router form and the zero-temperature limit validate
    their arguments before any launch (no GPU needed)."""
    ws = ctypes.c_void_p(256)
    d = ctypes.c_void_p(4096)
    vp = ctypes.c_void_p
    rowk = lib.lapsum_forward_rowk
    rowk.argtypes = [vp, ctypes.c_int64, vp, vp, vp, ctypes.c_int64, ctypes.c_int64, vp,
                     ctypes.c_double, ctypes.c_int, vp, ctypes.c_size_t, vp, ctypes.c_size_t, vp]
    assert rowk(d, 8, d, d, None, 1, 8, None, 0.1, 0, ws, 1 << 20, None, 0, None) == 1  # k NULL
    assert rowk(d, 8, d, d, None, 1, 8, d, 0.0, 0, ws, 1 << 20, None, 0, None) == 1     # t <= 0
    assert rowk(d, 8, d, d, None, 1, 8, d, 0.1, 9, ws, 1 << 20, None, 0, None) == 1     # bad path
    assert rowk(d, 8, d, d, None, 1, 8, d, 0.1, 0, None, 1 << 20, None, 0, None) == 2   # no ws
    router = lib.lapsum_forward_router
    router.argtypes = [vp, ctypes.c_int, ctypes.c_int64, vp, vp, ctypes.c_int64, ctypes.c_int64,
                       ctypes.c_double, ctypes.c_double, ctypes.c_float, ctypes.c_int32, vp, vp,
                       vp, vp, ctypes.c_size_t, vp]
    ok = (d, 0, 8, d, d, 1, 8, 2.0, 0.1, 0.0, 0, None, None, None, ws, 1 << 20, None)
    assert router(*ok[:1], 3, *ok[2:]) == 1                                   # unknown dtype
    assert router(*ok[:6], 5000, *ok[7:]) == 1                                # n > 4096
    assert router(*ok[:11], d, None, None, *ok[14:]) == 1                     # partial list args
    assert router(*ok[:9], 1e-3, 0, d, d, d, *ok[14:]) == 1                   # cap < 1
    assert router(*ok[:9], -1.0, 4, d, d, d, *ok[14:]) == 1                   # eps < 0
    assert router(*ok[:14], None, 1 << 20, None) == 2                         # no ws
    hard = lib.lapsum_forward_hard
    hard.argtypes = [vp, ctypes.c_int64, vp, vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                     ctypes.c_int, vp, ctypes.c_size_t, vp]
    assert hard(d, 8, d, d, 1, 8, 8.0, 0, ws, 1 << 20, None) == 1   # k = n
    assert hard(d, 8, d, d, 1, 8, 0.0, 0, ws, 1 << 20, None) == 1   # k = 0
    assert hard(d, 8, d, d, 1, 1, 0.5, 0, ws, 1 << 20, None) == 1   # n < 2
    assert hard(d, 8, d, d, 1, 8, 2.0, 4, ws, 1 << 20, None) == 1   # one CTA per row: no
    assert hard(d, 8, d, d, 1, 8, 2.0, 0x202, ws, 1 << 20, None) == 1  # unknown flag
    assert hard(d, 8, d, d, 1, 8, 2.0, 0, None, 1 << 20, None) == 2  # no ws


def test_per_row_budget_workspace_sizes(lib):
    """lapsum_workspace_bytes_rowk follows the per-row solver choice: the on-chip
    sort, the one-CTA bracketing (band buffers), the radix sort (key buffers) and
    the whole-GPU bracketing (per-row ladders next to its buffers)."""
    f = lib.lapsum_workspace_bytes_rowk
    f.restype = ctypes.c_size_t
    f.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int]
    assert f(0, 100, 0) == 0 and f(4, 0, 0) == 0
    assert f(4, 5_000_000, 2) >= f(1, 5_000_000, 2) > 0   # whole-GPU bracketing
    assert f(4, 100, 9) == 0                      # unknown path
    assert f(4, 2_000_000, 4) == 0                # one-CTA bracketing is for n <= 2^20
    small = f(16, 256, 0)
    assert small > 0 and small % 256 == 0
    assert f(256, 65536, 0) >= 2 * 256 * 65536 * 4        # band buffers
    assert f(2, 1 << 19, 3) >= 2 * 2 * (1 << 19) * 4       # radix key buffers
    assert f(2, 1 << 19, 0) >= 2 * (1 << 19) * 4           # AUTO: whole-GPU bracketing bands
    assert f(256, 65536, 3) >= 2 * 256 * 65536 * 4         # radix forced


def test_low_precision_entry_points_on_host(lib):
    """lapsum_forward_lowp / lapsum_backward_lowp: argument checks before any
    launch, and workspace sizes that add the widened rows (B x ld fp32) to the
    fp32 solver's workspace."""
    vp = ctypes.c_void_p
    d = ctypes.c_void_p(4096)
    ws = ctypes.c_void_p(256)
    fw = lib.lapsum_forward_lowp
    fw.restype = ctypes.c_int
    fw.argtypes = [vp, ctypes.c_int, ctypes.c_int64, vp, vp, vp, ctypes.c_int64, ctypes.c_int64,
                   ctypes.c_double, ctypes.c_double, ctypes.c_int, ctypes.c_uint64, vp,
                   ctypes.c_size_t, vp, ctypes.c_size_t, vp]
    ok = [d, 1, 5000, d, d, None, 1, 5000, 10.0, 0.1, 0, 0, ws, 1 << 30, None, 0, None]
    bad = list(ok); bad[1] = 3
    assert fw(*bad) == 1                          # unknown dtype
    bad = list(ok); bad[8] = 5000.0
    assert fw(*bad) == 1                          # k = n
    bad = list(ok); bad[2] = 4000
    assert fw(*bad) == 1                          # ld < n
    bad = list(ok); bad[12] = None
    assert fw(*bad) == 2                          # no workspace
    bad = list(ok); bad[13] = 1024
    assert fw(*bad) == 2                          # workspace too small
    bw = lib.lapsum_backward_lowp
    bw.restype = ctypes.c_int
    bw.argtypes = [vp, ctypes.c_int, ctypes.c_int64, vp, vp, vp, ctypes.c_int64, ctypes.c_int64,
                   ctypes.c_double, vp, ctypes.c_size_t, vp, ctypes.c_size_t, vp]
    assert bw(d, 7, 5000, d, d, d, 1, 5000, 0.1, None, 0, ws, 1 << 30, None) == 1
    assert bw(d, 2, 5000, d, d, d, 1, 5000, -0.1, None, 0, ws, 1 << 30, None) == 1
    assert bw(d, 2, 5000, d, d, d, 1, 5000, 0.1, None, 0, ws, 64, None) == 2
    sz = lib.lapsum_workspace_bytes_lowp
    sz.restype = ctypes.c_size_t
    sz.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_double, ctypes.c_int]
    base = lib.lapsum_workspace_bytes
    base.restype = ctypes.c_size_t
    base.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_double, ctypes.c_int]
    assert sz(2, 70001, 70008, 300.0, 3) >= base(2, 70001, 300.0, 3) + 2 * 70008 * 4
    assert sz(2, 70001, 70000, 300.0, 3) == 0     # ld < n
    bsz = lib.lapsum_backward_workspace_bytes_lowp
    bsz.restype = ctypes.c_size_t
    bsz.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
    assert bsz(3, 9000, 9005) >= 3 * 9005 * 4 and bsz(0, 9000, 9000) == 0
