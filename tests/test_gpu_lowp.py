"""GPU parity for 16-bit scores (bf16 and fp16) at every row length.

"Fast LapSum: Exact Differentiable Top-k at Million Scale" (gist.science
explainer pages), section 2.1 states the problem for real scores; here they
arrive as bf16 or fp16 values.  Both widen exactly to fp32, so b, p and g must
match the oracle solved on those values (converted to fp64), at the same
tolerances as fp32 scores:

* short rows (n <= 4096): the on-chip kernels read the 16-bit scores
  (lapsum_forward_router with fp16, and lapsum_forward_lowp);
* long rows: lapsum_forward_lowp / lapsum_backward_lowp widen the rows, then
  the radix, one-CTA-per-row and whole-GPU bracketing solvers run, with and
  without the gradient support;
* autograd on 16-bit scores returns the gradient in the scores' dtype.
"""
import numpy as np
import pytest
import torch

import sparse_selection_primitive_b200 as L
from tests.gpu_helpers import check_row
from workloads import random_rows

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "f16": torch.float16}


def _narrow(r: np.ndarray, dt: str):
    """16-bit tensor on the GPU and its exact values as fp64 (round to nearest even)."""
    rh = torch.from_numpy(r).to(DT[dt])
    return rh.cuda(), rh.to(torch.float64).numpy()


@pytest.mark.parametrize("B,n,k,t", [(64, 256, 8.0, 0.05), (7, 1000, 40.0, 0.02),
                                     (3, 4096, 64.0, 0.05), (5, 77, 3.5, 0.1)])
def test_router_fp16_matches_oracle(cuda_device, B, n, k, t):
    r, v = random_rows(700 + n, B, n)
    rt, r64 = _narrow(r, "f16")
    p, b = L.forward_router(rt, k, t)
    g = L.backward_router(rt, b, torch.from_numpy(v).cuda(), t)
    torch.cuda.synchronize()
    p, b, g = p.cpu().numpy().astype(np.float64), b.cpu().numpy(), g.cpu().numpy()
    for i in range(B):
        check_row(r64[i], v[i], k, t, b[i], p[i], g[i].astype(np.float64), label=f"row {i}")


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("B,n,k,t,path,support", [
    (4, 300, 9.0, 0.05, "auto", False),          # on-chip, 16-bit loads
    (2, 70001, 300.0, 0.02, "auto", True),       # one CTA per row
    (2, 70001, 300.0, 0.02, "radix", False),     # radix full sort
    (1, 400003, 500.0, 0.01, "bracket", True),   # whole-GPU bracketing
    (1, 300000, 250.0, 0.05, "bracket", False),
])
def test_lowp_rows_match_oracle(cuda_device, dt, B, n, k, t, path, support):
    r, v = random_rows(800 + n + B, B, n, "mix_nu" if n > 100000 else "normal")
    rt, r64 = _narrow(r, dt)
    sup = L.Support(B, n, rt.device) if support and n > 4096 else None
    p, b, sf = L.forward_lowp(rt, k, t, path=path, want_sum_f=True, support=sup)
    g = L.backward_lowp(rt, b, torch.from_numpy(v).cuda(), t, support=sup)
    torch.cuda.synchronize()
    p, b, g, sf = (p.cpu().numpy().astype(np.float64), b.cpu().numpy(),
                   g.cpu().numpy().astype(np.float64), sf.cpu().numpy())
    for i in range(B):
        b_ref = check_row(r64[i], v[i], k, t, b[i], p[i], g[i],
                          label=f"{dt} {path} n={n} row {i}")
        f = 0.5 * np.exp(-np.abs(r64[i] - b_ref) / t)
        assert abs(sf[i] - f.sum()) <= 1e-5 * max(1.0, f.sum())


def test_lowp_strided_rows(cuda_device):
    # rows with a leading dimension that rules out 16-byte accesses
    B, n, k, t = 3, 9000, 70.0, 0.03
    r, v = random_rows(901, B, n)
    big = torch.zeros((B, n + 5), dtype=torch.float16)
    big[:, :n] = torch.from_numpy(r).to(torch.float16)
    rt = big.cuda()[:, :n]
    r64 = big[:, :n].to(torch.float64).numpy()
    p, b = L.forward_lowp(rt, k, t)
    g = L.backward_lowp(rt, b, torch.from_numpy(v).cuda(), t)
    torch.cuda.synchronize()
    p, b, g = p.cpu().numpy().astype(np.float64), b.cpu().numpy(), g.cpu().numpy()
    for i in range(B):
        check_row(r64[i], v[i], k, t, b[i], p[i], g[i].astype(np.float64), label=f"row {i}")


@pytest.mark.parametrize("dt,n", [("f16", 512), ("bf16", 50000), ("f16", 50000)])
def test_autograd_16bit_scores(cuda_device, dt, n):
    B, k, t = 2, 20.0, 0.05
    r, v = random_rows(950 + n, B, n)
    rt, r64 = _narrow(r, dt)
    rt.requires_grad_(True)
    p = L.soft_topk(rt, k, t)
    p.backward(torch.from_numpy(v).cuda())
    torch.cuda.synchronize()
    assert rt.grad.dtype == DT[dt]
    # the fp32 gradient, rounded to the scores' dtype, is what comes back
    g32 = L.backward_lowp(rt.detach(), L.forward_lowp(rt.detach(), k, t)[1],
                          torch.from_numpy(v).cuda(), t)
    assert torch.equal(rt.grad, g32.to(DT[dt]))
    for i in range(B):
        check_row(r64[i], v[i], k, t, float(L.forward_lowp(rt.detach(), k, t)[1][i]),
                  p.detach()[i].cpu().numpy().astype(np.float64),
                  g32[i].cpu().numpy().astype(np.float64), label=f"{dt} row {i}")
