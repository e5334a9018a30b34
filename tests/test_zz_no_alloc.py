"""The allocation-free backward against the regular one (GPU).

lapsum_backward_noalloc serves callers that cannot allocate device memory
when they need the gradient (capture under a no-allocation rule, hosts that
reserve all device memory up front, plugin hosts that own every allocation).
It must give the same g as lapsum_backward, within the tests' VJP tolerance,
on two calls in a row (its scratch array keeps the previous call's contents),
and match the oracle's VJP on a row.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sparse_selection_primitive_b200 as L
from workloads import random_rows

pytestmark = pytest.mark.gpu

TOL_G = 1e-4


def _noalloc(lib, r, b, v, g, B, n, t, stream):
    fn = lib.lapsum_backward_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                   ctypes.c_void_p]
    return fn(r.data_ptr(), n, b.data_ptr(), v.data_ptr(), g.data_ptr(), B, n, t, stream)


@pytest.mark.parametrize("B,n,k,t,path", [(3, 70001, 500.0, 0.05, "radix"),
                                          (1, 3_000_000, 300.0, 0.01, "bracket"),
                                          (5, 1000, 20.0, 0.1, "fullsort")])
def test_noalloc_backward_matches_regular(cuda_device, B, n, k, t, path):
    r_h, v_h = random_rows(40 + B, B, n)
    r = torch.from_numpy(r_h).cuda()
    v = torch.from_numpy(v_h).cuda()
    _, b = L.forward(r, k, t, path=path)
    g_ref = L.backward(r, b, v, t)
    lib = L._lib()
    stream = torch.cuda.current_stream().cuda_stream
    scale = float(g_ref.abs().max())
    for call in range(2):  # the second call runs on the array the first one left behind
        g = torch.full_like(r, float("nan"))
        assert _noalloc(lib, r, b, v, g, B, n, t, stream) == 0
        torch.cuda.synchronize()
        err = float((g - g_ref).abs().max())
        assert err <= TOL_G * scale, (call, err, scale)
    # the Python wrapper reaches the same entry point
    g2 = L.backward_noalloc(r, b, v, t)
    assert float((g2 - g_ref).abs().max()) <= TOL_G * scale
    # and one row of it against the oracle (its own threshold and VJP)
    i = B - 1
    g_or, _, _ = oracle.vjp(r_h[i], v_h[i], oracle.solve_b(r_h[i], k, t), t)
    dg = float(np.max(np.abs(g2[i].cpu().numpy().astype(np.float64) - g_or)))
    assert dg <= TOL_G * float(np.max(np.abs(g_or))), dg


def test_noalloc_backward_rejects_too_many_rows(cuda_device):
    B, n = 1025, 5000
    r = torch.zeros((B, n), device="cuda")
    b = torch.zeros(B, dtype=torch.float64, device="cuda")
    g = torch.empty_like(r)
    lib = L._lib()
    assert _noalloc(lib, r, b, r, g, B, n, 0.1, torch.cuda.current_stream().cuda_stream) == 1
