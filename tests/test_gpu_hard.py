"""GPU parity of the zero-temperature limit (lapsum_forward_hard).

"Fast LapSum: Exact Differentiable Top-k at Million Scale" (gist.science
explainer pages), section 2.3: DFTopK's midpoint threshold is LapSum at t -> 0.
The GPU's b and p must equal the oracle's limit exactly: b is the boundary
score or the fp64 midpoint of two fp32 scores on both sides, and p is 1, 0 or
the tie share (k - a)/m, rounded once to fp32.

Cases: on-chip rows (one and several warps per row, ragged) and radix rows,
integer and fractional budgets, ties at the boundary (scores on a 1/64 grid),
-0 and +0 in one group, non-finite rows, and budgets at both extremes.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_selection_primitive_b200 as L
from workloads import random_rows

pytestmark = pytest.mark.gpu


def _check(r, k, p, b, label=""):
    b_ref, p_ref = oracle.hard_topk(r.astype(np.float64), k)
    assert b == b_ref, f"{label}: b {b!r} vs {b_ref!r}"
    assert np.array_equal(p, p_ref.astype(np.float32)), f"{label}: p differs"


@pytest.mark.parametrize("B,n,dist", [(9, 256, "normal"), (6, 256, "normal_q64"),
                                      (5, 100, "normal_q64"), (4, 1000, "normal"),
                                      (3, 4096, "normal_q64"), (3, 5000, "normal_q64"),
                                      (2, 70001, "normal")])
def test_hard_matches_oracle(cuda_device, B, n, dist):
    r, _ = random_rows(501 + n, B, n, dist)
    rng = np.random.default_rng(n)
    for k in (1.0, float(n // 5), n / 3.0 + 0.37, float(n - 1), 0.25, n - 0.5,
              float(rng.integers(1, n))):
        p, b = L.hard_topk(torch.from_numpy(r).cuda(), k)
        torch.cuda.synchronize()
        p, b = p.cpu().numpy(), b.cpu().numpy()
        for i in range(B):
            _check(r[i], k, p[i], b[i], label=f"k={k} row {i}")


@pytest.mark.parametrize("n,path", [(300, "auto"), (6000, "auto"), (300, "radix")])
def test_hard_signed_zero_is_one_value(cuda_device, n, path):
    r = np.linspace(-1.0, 1.0, n).astype(np.float32)
    r[:10] = -0.0
    r[10:20] = 0.0
    r = np.random.default_rng(3).permutation(r)
    nonneg = int(np.sum(r >= 0))  # counts -0 and +0 together
    k = nonneg - 7.5              # the boundary group is the 20 zeros
    p, b = L.hard_topk(torch.from_numpy(r).cuda(), k, path=path)
    torch.cuda.synchronize()
    _check(r, k, p.cpu().numpy(), b.item(), label="signed zeros")
    assert b.item() == 0.0


@pytest.mark.parametrize("n", [500, 9000])
def test_hard_nonfinite_rows(cuda_device, n):
    r, _ = random_rows(502, 3, n)
    r[1, 7] = np.inf
    p, b = L.hard_topk(torch.from_numpy(r).cuda(), 10.0)
    torch.cuda.synchronize()
    p, b = p.cpu().numpy(), b.cpu().numpy()
    assert math.isnan(b[1]) and np.isnan(p[1]).all()
    for i in (0, 2):
        _check(r[i], 10.0, p[i], b[i])


def test_hard_refuses_bracketing_and_bad_budgets(cuda_device):
    rt = torch.zeros((1, 5000), device="cuda")
    with pytest.raises(L.LapSumError):
        L.hard_topk(rt, 5.0, path="bracket")
    with pytest.raises(L.LapSumError):
        L.hard_topk(rt, 5000.0)
    with pytest.raises(L.LapSumError):
        L.hard_topk(rt, 0.0)
