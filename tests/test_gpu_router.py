"""GPU parity of the router form (lapsum_forward_router / lapsum_backward_router).

"Fast LapSum: Exact Differentiable Top-k at Million Scale" (gist.science
explainer pages), sections 2.1 and 2.2: the same full-sort solver and VJP as
the on-chip rows, here with bf16 scores and a per-row list of the scores with
p > eps written next to p.

* bf16 scores are widened exactly to fp32, so b, p and g must match the
  oracle solved on the bf16 values (converted to fp64);
* the list is checked against the p the GPU wrote: the positions of p > eps in
  ascending order, their values, and the count (truncated at cap);
* sizes cover one warp per row, several warps per row, ragged rows and rows
  whose leading dimension rules out vector loads.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_selection_primitive_b200 as L
from tests.gpu_helpers import check_row
from workloads import random_rows

pytestmark = pytest.mark.gpu


def _bf16(r: np.ndarray):
    """bf16 tensor on the GPU and its exact values as fp64 (round to nearest even)."""
    rb = torch.from_numpy(r).to(torch.bfloat16)
    return rb.cuda(), rb.to(torch.float64).numpy()


@pytest.mark.parametrize("B,n,k,t", [(64, 256, 8.0, 0.05), (9, 100, 3.5, 0.1),
                                     (5, 1000, 40.0, 0.02), (3, 4096, 64.0, 0.05)])
def test_router_bf16_matches_oracle(cuda_device, B, n, k, t):
    r, v = random_rows(401 + n, B, n)
    rt, r64 = _bf16(r)
    p, b = L.forward_router(rt, k, t)
    vt = torch.from_numpy(v).cuda()
    g = L.backward_router(rt, b, vt, t)
    torch.cuda.synchronize()
    p, b, g = p.cpu().numpy().astype(np.float64), b.cpu().numpy(), g.cpu().numpy()
    for i in range(B):
        check_row(r64[i], v[i], k, t, b[i], p[i], g[i].astype(np.float64), label=f"row {i}")


def test_router_bf16_unaligned_rows(cuda_device):
    B, n, k, t = 6, 300, 12.0, 0.05
    r, v = random_rows(402, B, n)
    big = torch.zeros((B, n + 3), dtype=torch.bfloat16)
    big[:, :n] = torch.from_numpy(r).to(torch.bfloat16)
    rt = big.cuda()[:, :n]            # leading dimension n + 3: scalar loads
    r64 = big[:, :n].to(torch.float64).numpy()
    p, b = L.forward_router(rt, k, t)
    g = L.backward_router(rt, b, torch.from_numpy(v).cuda(), t)
    torch.cuda.synchronize()
    p, b, g = p.cpu().numpy().astype(np.float64), b.cpu().numpy(), g.cpu().numpy()
    for i in range(B):
        check_row(r64[i], v[i], k, t, b[i], p[i], g[i].astype(np.float64), label=f"row {i}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("n,eps,cap", [(256, 1e-3, 32), (256, 0.5, 4), (1000, 1e-4, 64),
                                       (77, 0.0, 80), (4096, 1e-3, 16)])
def test_router_selection_list(cuda_device, dtype, n, eps, cap):
    B, k, t = 40, 8.0, 0.05
    r, _ = random_rows(403 + n, B, n)
    rt = torch.from_numpy(r).to(dtype).cuda()
    out = (torch.empty((B, n), device="cuda"), torch.empty(B, dtype=torch.float64, device="cuda"),
           torch.full((B, cap), -1, dtype=torch.int32, device="cuda"),
           torch.zeros((B, cap), device="cuda"), torch.empty(B, dtype=torch.int32, device="cuda"))
    p, b, idx, vals, cnt = L.forward_router(rt, k, t, eps=eps, cap=cap, out=out)
    torch.cuda.synchronize()
    p, idx, vals, cnt = p.cpu().numpy(), idx.cpu().numpy(), vals.cpu().numpy(), cnt.cpu().numpy()
    for i in range(B):
        sel = np.nonzero(p[i] > np.float32(eps))[0]
        assert cnt[i] == sel.size, (i, cnt[i], sel.size)
        m = min(cap, sel.size)
        assert np.array_equal(idx[i, :m], sel[:m].astype(np.int32)), i
        assert np.array_equal(vals[i, :m], p[i, sel[:m]]), i
        assert (idx[i, m:] == -1).all()      # untouched past the list
    # the p the list was taken from is the solver's: spot-check against the oracle
    r64 = torch.from_numpy(r).to(dtype).to(torch.float64).numpy()
    b_ref = oracle.solve_b(r64[0], k, t)
    assert abs(b.cpu().numpy()[0] - b_ref) <= 1e-5 * max(t, abs(b_ref))


def test_router_refuses_long_rows_and_bad_selection(cuda_device):
    r = torch.zeros((2, 5000), device="cuda")
    with pytest.raises(L.LapSumError):
        L.forward_router(r, 5.0, 0.1)
    with pytest.raises(L.LapSumError):
        L.forward_router(torch.zeros((2, 100), device="cuda"), 5.0, 0.1, eps=-1.0, cap=4)


def test_router_bf16_autograd(cuda_device):
    """soft_topk on bf16 scores: p from the router form, the gradient with respect to
    r equal to lapsum_backward_router's rounded to bf16, and dL/dk and dL/dt from
    the widened scores as the oracle gives them."""
    B, n, t = 12, 256, 0.05
    r, v = random_rows(404, B, n)
    rb = torch.from_numpy(r).to(torch.bfloat16).cuda().requires_grad_(True)
    k = torch.tensor(8.0, dtype=torch.float64, device="cuda", requires_grad=True)
    p = L.soft_topk(rb, k, t)
    vt = torch.from_numpy(v).cuda()
    p.backward(vt)
    assert p.dtype == torch.float32 and rb.grad.dtype == torch.bfloat16
    p2, b2 = L.forward_router(rb.detach(), 8.0, t)
    g2 = L.backward_router(rb.detach(), b2, vt, t).to(torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(p.detach(), p2) and torch.equal(rb.grad, g2)
    r64 = rb.detach().to(torch.float64).cpu().numpy()
    gk_ref = 0.0
    for i in range(B):
        b_ref = oracle.solve_b(r64[i], 8.0, t)
        gk_ref += oracle.vjp_kt(r64[i], v[i], b_ref, t)[0]
    assert abs(k.grad.item() - gk_ref) <= 1e-4 * max(1.0, abs(gk_ref))
