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
from workloads import WORKLOADS, make_inputs, random_rows

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


def test_hard_refuses_one_cta_bracketing_and_bad_budgets(cuda_device):
    rt = torch.zeros((1, 5000), device="cuda")
    with pytest.raises(L.LapSumError):
        L.hard_topk(rt, 5.0, path="rowbracket")
    with pytest.raises(L.LapSumError):
        L.hard_topk(rt, 5000.0)
    with pytest.raises(L.LapSumError):
        L.hard_topk(rt, 0.0)


@pytest.mark.parametrize("B,n,dist", [(3, 70001, "normal"), (2, 65536, "normal_q64"),
                                      (1, 400003, "mix_nu"), (2, 300000, "abs_t3")])
def test_hard_bracketing_matches_oracle(cuda_device, B, n, dist):
    """Long rows through the bracketed selection (no full sort): b and p bit for
    bit equal to the oracle's limit, for integer budgets (the midpoint case on
    distinct scores), fractional ones and ties at the boundary; the radix
    full sort gives the same bits."""
    r, _ = random_rows(601 + n, B, n, dist)
    rt = torch.from_numpy(r).cuda()
    rng = np.random.default_rng(n + 3)
    for k in (1.0, 37.0, float(n // 100) + 0.5, float(rng.integers(2, n // 20)), n / 40.0):
        ws = L.Workspace(B, n, k, "fullsort")
        p, b = L.hard_topk(rt, k, ws=ws)
        p2, b2 = L.hard_topk(rt, k, path="radix")
        torch.cuda.synchronize()
        for i in range(B):
            info = L.row_info(ws, i)
            assert info["path"] == 2 and info["attempts"] == 1, info
        assert torch.equal(b, b2) and torch.equal(p, p2)
        p, b = p.cpu().numpy(), b.cpu().numpy()
        for i in range(B):
            _check(r[i], k, p[i], b[i], label=f"{dist} k={k} row {i}")


def test_hard_bracketing_forced_miss_selects_exactly(cuda_device):
    """A bracket that excludes the boundary score: the exact selection over the
    row takes over and the result is still the oracle's, bit for bit."""
    B, n = 2, 50000
    r, _ = random_rows(611, B, n, "normal_q64")
    rt = torch.from_numpy(r).cuda()
    for k in (5.0, 123.5, 700.0):
        ws = L.Workspace(B, n, k, "radix")
        p, b = L.hard_topk(rt, k, path=L.PATHS["bracket"] | L.FLAG_FORCE_MISS, ws=ws)
        torch.cuda.synchronize()
        for i in range(B):
            assert L.row_info(ws, i)["attempts"] == 2
        p, b = p.cpu().numpy(), b.cpu().numpy()
        for i in range(B):
            _check(r[i], k, p[i], b[i], label=f"forced miss k={k} row {i}")


def test_hard_bracketing_signed_zeros_and_nonfinite(cuda_device):
    n = 20000
    r = np.linspace(-1.0, 1.0, n).astype(np.float32)
    r[:300] = -0.0
    r[300:600] = 0.0
    r = np.random.default_rng(5).permutation(r)
    k = int(np.sum(r >= 0)) - 100.5  # the boundary group is the 600 zeros
    rr = np.stack([r, r.copy()])
    rr[1, 17] = np.inf
    p, b = L.hard_topk(torch.from_numpy(rr).cuda(), k, path="bracket")
    torch.cuda.synchronize()
    _check(r, k, p[0].cpu().numpy(), b[0].item(), label="signed zeros")
    assert b[0].item() == 0.0
    assert math.isnan(b[1].item()) and torch.isnan(p[1]).all()


@pytest.mark.parametrize("name,rows", [("memory_select_256x65536", [0, 1, 77, 200, 255]),
                                       ("extreme_1e8", [0])])
def test_hard_bracketing_full_size_workloads(cuda_device, name, rows):
    """The memory-selection batch and the 10^8-score row at full size, through
    the bracketed selection: b and p bit for bit equal to the oracle's limit on
    sampled rows, and sum p = k on every row."""
    w = WORKLOADS[name]
    r, _ = make_inputs(w)
    rt = torch.from_numpy(r).cuda()
    ws = L.Workspace(w.B, w.n, w.k, "fullsort")
    p, b = L.hard_topk(rt, w.k, ws=ws)
    torch.cuda.synchronize()
    assert L.row_info(ws, 0)["path"] == 2
    sums = p.double().sum(dim=1).cpu().numpy()
    assert np.max(np.abs(sums - w.k)) <= 1e-3
    for i in rows:
        _check(r[i], w.k, p[i].cpu().numpy(), b[i].item(), label=f"{name} row {i}")
