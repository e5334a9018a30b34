"""GPU parity of the forward with one budget per row (lapsum_forward_rowk).

"Fast LapSum: Exact Differentiable Top-k at Million Scale" (gist.science
explainer pages), section 2.1, states the balance equation sum_i sigma((r_i -
b)/t) = k for one row; every row is solved on its own, so a budget per row is
the same equation with k_row in place of k.  Each row is compared with the
oracle solved at its own budget, at the tolerances of the other parity tests:

* on-chip rows (n <= 4096), one-CTA-per-row bracketing rows and radix rows, with
  fractional budgets, budgets near 0 and near n, and ragged lengths;
* a row whose budget lies outside (0, n) gets b = NaN and p = NaN, the status
  word reads LAPSUM_EINVAL, and the other rows are unaffected;
* equal budgets give the bits of the shared-budget call on the same solver;
* both bracketing arrangements (one CTA per row, and the whole GPU on each row)
  take their sample size and ranks per row on the device, equal to the
  oracle's; an out-of-range budget gives that row NaN there too;
* autograd: the gradient of a per-row k tensor is the oracle's dL/dk per row;
* the support hand-over of long rows with per-row budgets.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_selection_primitive_b200 as L
from tests.gpu_helpers import check_row, run_gpu
from workloads import random_rows

pytestmark = pytest.mark.gpu


def _budgets(rng, B, n):
    k = rng.uniform(0.5, n - 0.5, B)
    k[0] = 0.3            # below one score
    if B > 1:
        k[1] = n - 0.2    # above n - 1
    if B > 2:
        k[2] = float(max(1, n // 7))
    return k


@pytest.mark.parametrize("B,n,dist", [(7, 256, "normal"), (5, 1000, "normal_q64"),
                                      (3, 4096, "mix_nu"), (4, 5000, "normal"),
                                      (3, 70001, "abs_t3")])
def test_rowk_matches_oracle_per_row(cuda_device, B, n, dist):
    r, v = random_rows(301 + n, B, n, dist)
    rng = np.random.default_rng(n)
    k = _budgets(rng, B, n)
    t = 0.05
    kt = torch.tensor(k, dtype=torch.float64, device="cuda")
    res = run_gpu(r, kt, t, v=v)
    for i in range(B):
        check_row(r[i], v[i], float(k[i]), t, res["b"][i], res["p"][i], res["g"][i],
                  label=f"row {i} k={k[i]:.3f}")


def test_rowk_invalid_budgets_are_flagged_per_row(cuda_device):
    B, n, t = 6, 300, 0.1
    r, _ = random_rows(311, B, n)
    k = np.array([10.0, 0.0, 7.5, float(n), -3.0, math.nan])
    rt = torch.from_numpy(r).cuda()
    ws = L.Workspace(B, n, 1.0, "fullsort")
    p, b = L.forward(rt, torch.tensor(k, device="cuda"), t, ws=ws)
    torch.cuda.synchronize()
    bb, pp = b.cpu().numpy(), p.cpu().numpy()
    for i in (1, 3, 4, 5):
        assert math.isnan(bb[i]) and np.isnan(pp[i]).all(), i
    for i in (0, 2):
        check_row(r[i], None, float(k[i]), t, bb[i], pp[i].astype(np.float64))
    assert L.read_status(ws) == 1  # LAPSUM_EINVAL, then cleared
    assert L.read_status(ws) == 0


def test_rowk_invalid_budget_on_the_radix_path(cuda_device):
    B, n, t = 3, 6000, 0.05
    r, _ = random_rows(312, B, n)
    k = np.array([40.0, 6000.0, 2.5])
    rt = torch.from_numpy(r).cuda()
    ws = L.Workspace(B, n, 1.0, "fullsort")
    p, b = L.forward(rt, torch.tensor(k, device="cuda"), t, ws=ws, path="fullsort")
    torch.cuda.synchronize()
    bb, pp = b.cpu().numpy(), p.cpu().numpy()
    assert math.isnan(bb[1]) and np.isnan(pp[1]).all()
    for i in (0, 2):
        check_row(r[i], None, float(k[i]), t, bb[i], pp[i].astype(np.float64))
    assert L.read_status(ws) == 1


@pytest.mark.parametrize("n,path", [(512, "fullsort"), (9000, "radix")])
def test_rowk_equal_budgets_match_the_shared_budget(cuda_device, n, path):
    B, t, k = 4, 0.02, 17.0
    r, _ = random_rows(313, B, n)
    rt = torch.from_numpy(r).cuda()
    p1, b1 = L.forward(rt, k, t, path=path)
    p2, b2 = L.forward(rt, torch.full((B,), k, dtype=torch.float64, device="cuda"), t, path=path)
    torch.cuda.synchronize()
    assert torch.equal(b1, b2) and torch.equal(p1, p2)


@pytest.mark.parametrize("B,n,dist", [(2, 400000, "mix_nu"), (3, 300001, "abs_t3")])
def test_rowk_whole_gpu_bracketing(cuda_device, B, n, dist):
    """The whole-GPU bracketing with one budget per row: each row's sample size
    and ranks come from its own budget on the device (equal to the oracle's);
    b, p and g must match the oracle solved at that budget."""
    r, v = random_rows(319 + n, B, n, dist)
    rng = np.random.default_rng(n + 7)
    k = rng.uniform(2.0, n / 50.0, B)
    k[0] = 40.0
    kt = torch.tensor(k, dtype=torch.float64, device="cuda")
    rt = torch.from_numpy(r).cuda()
    ws = L.Workspace(B, n, 1.0, "auto", nbytes=L._lib().lapsum_workspace_bytes_rowk(B, n, 2))
    sup = L.Support(B, n)
    p, b = L.forward(rt, kt, 0.02, path="bracket", ws=ws, support=sup)
    g = L.backward(rt, b, torch.from_numpy(v).cuda(), 0.02, support=sup)
    torch.cuda.synchronize()
    assert L.read_status(ws) == 0
    p, bb, g = p.cpu().numpy().astype(np.float64), b.cpu().numpy(), g.cpu().numpy()
    for i in range(B):
        info = L.row_info(ws, i)
        assert info["path"] == 2, info
        m = info["sample_m"]
        q = float(k[i]) / n
        want_m = 4096
        while want_m < 32768 and want_m < 64.0 / q:
            want_m *= 2
        assert m == want_m
        l, h = oracle.binom_ranks(m, q, 1e-6)
        assert (info["rank_l"], info["rank_h"]) == (l, h), (i, info, l, h)
        check_row(r[i], v[i], float(k[i]), 0.02, bb[i], p[i], g[i].astype(np.float64),
                  label=f"row {i}")


def test_rowk_bad_budget_on_the_whole_gpu_bracketing(cuda_device):
    B, n = 3, 300000
    r, _ = random_rows(321, B, n, "mix_nu")
    k = np.array([150.0, float(n), 400.0])  # the middle budget is out of range
    rt = torch.from_numpy(r).cuda()
    ws = L.Workspace(B, n, 1.0, "auto", nbytes=L._lib().lapsum_workspace_bytes_rowk(B, n, 2))
    p, b = L.forward(rt, torch.tensor(k, device="cuda"), 0.05, path="bracket", ws=ws)
    torch.cuda.synchronize()
    bb, pp = b.cpu().numpy(), p.cpu().numpy()
    assert math.isnan(bb[1]) and np.isnan(pp[1]).all()
    for i in (0, 2):
        check_row(r[i], None, float(k[i]), 0.05, bb[i], pp[i].astype(np.float64))
    assert L.read_status(ws) == 1


@pytest.mark.parametrize("B,n,dist,path", [(5, 20000, "normal", "auto"),
                                           (3, 65536, "normal_q64", "auto"),
                                           (2, 300000, "mix_nu", "rowbracket")])
def test_rowk_one_cta_per_row_bracketing(cuda_device, B, n, dist, path):
    """Each row's sample size and binomial ranks come from its own budget, on the
    device; they must equal the oracle's for that budget, and b, p, g must match."""
    r, v = random_rows(317 + n, B, n, dist)
    rng = np.random.default_rng(n + 1)
    k = rng.uniform(1.0, n / 3.0, B)
    k[0] = 3.0
    kt = torch.tensor(k, dtype=torch.float64, device="cuda")
    rt = torch.from_numpy(r).cuda()
    ws = L.Workspace(B, n, 1.0, "auto",
                     nbytes=L._lib().lapsum_workspace_bytes_rowk(B, n, L.PATHS[path]))
    p, b = L.forward(rt, kt, 0.02, path=path, ws=ws)
    g = L.backward(rt, b, torch.from_numpy(v).cuda(), 0.02)
    torch.cuda.synchronize()
    p, bb, g = p.cpu().numpy().astype(np.float64), b.cpu().numpy(), g.cpu().numpy()
    for i in range(B):
        info = L.row_info(ws, i)
        assert info["path"] == 4, info
        m = info["sample_m"]
        q = float(k[i]) / n
        want_m = 4096
        while want_m < 32768 and want_m < 64.0 / q:
            want_m *= 2
        assert m == want_m
        l, h = oracle.binom_ranks(m, q, 1e-6)
        assert (info["rank_l"], info["rank_h"]) == (l, h), (i, info, l, h)
        check_row(r[i], v[i], float(k[i]), 0.02, bb[i], p[i], g[i].astype(np.float64),
                  label=f"row {i}")


def test_rowk_bad_budget_on_the_one_cta_bracketing(cuda_device):
    B, n = 3, 10000
    r, _ = random_rows(318, B, n)
    k = np.array([25.0, -1.0, 100.0])
    rt = torch.from_numpy(r).cuda()
    ws = L.Workspace(B, n, 1.0, "auto", nbytes=L._lib().lapsum_workspace_bytes_rowk(B, n, 0))
    p, b = L.forward(rt, torch.tensor(k, device="cuda"), 0.05, ws=ws)
    torch.cuda.synchronize()
    bb, pp = b.cpu().numpy(), p.cpu().numpy()
    assert math.isnan(bb[1]) and np.isnan(pp[1]).all()
    for i in (0, 2):
        check_row(r[i], None, float(k[i]), 0.05, bb[i], pp[i].astype(np.float64))
    assert L.read_status(ws) == 1


def test_rowk_autograd_gradient_per_row(cuda_device):
    B, n, t = 5, 777, 0.05
    r, v = random_rows(315, B, n)
    k = np.array([3.0, 10.5, 100.0, 400.25, 776.0])
    rt = torch.from_numpy(r).cuda().requires_grad_(True)
    kt = torch.tensor(k, dtype=torch.float64, device="cuda", requires_grad=True)
    p = L.soft_topk(rt, kt, t)
    p.backward(torch.from_numpy(v).cuda())
    gk = kt.grad.cpu().numpy()
    assert gk.shape == (B,)
    for i in range(B):
        b_ref = oracle.solve_b(r[i], float(k[i]), t)
        gk_ref, _ = oracle.vjp_kt(r[i], v[i], b_ref, t)
        assert abs(gk[i] - gk_ref) <= 1e-4 * max(1.0, abs(gk_ref)), (i, gk[i], gk_ref)
    assert rt.grad is not None and torch.isfinite(rt.grad).all()


def test_rowk_support_hand_over(cuda_device):
    B, n, t = 3, 50000, 0.01
    r, v = random_rows(316, B, n, "mix_nu")
    k = np.array([12.0, 250.5, 4000.0])
    res = run_gpu(r, torch.tensor(k, device="cuda"), t, v=v, support=True)
    for i in range(B):
        check_row(r[i], v[i], float(k[i]), t, res["b"][i], res["p"][i], res["g"][i],
                  label=f"row {i}")
