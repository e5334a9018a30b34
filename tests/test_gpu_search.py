"""GPU parity of the segment search for rows of at most 256 scores (AUTO).

"Fast LapSum: Exact Differentiable Top-k at Million Scale" (gist.science
explainer pages), section 2.2: between two neighbouring scores the budget
equation has a closed-form root.  The on-chip search evaluates that root for
the segment around a point and moves the point until the root falls inside
its own segment, with no sort; a row it does not settle is sorted in the same
kernel.  Both must give the oracle's b, p and VJP at the parity tolerances:
ragged lengths across 1, 2, 4 and 8 scores per lane, ties, heavy tails,
temperatures from far below the gaps (a staircase F) to far above the spread,
budgets at both extremes, per-row budgets, and every row pushed to the sort
(FLAG_FORCE_MISS).
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_selection_primitive_b200 as L
from tests.gpu_helpers import check_row, run_gpu
from workloads import random_rows

pytestmark = pytest.mark.gpu

DISTS = ["normal", "normal_q64", "abs_t3", "mix_nu"]
FORCE_SORT = L.PATHS["auto"] | L.FLAG_FORCE_MISS


def _case(seed):
    rng = np.random.default_rng(7000 + seed)
    n = int(rng.choice([2, 3, 5, 17, 31, 32, 33, 63, 64, 65, 100, 127, 128, 129, 200, 255, 256]))
    B = int(rng.integers(1, 20))
    dist = DISTS[int(rng.integers(0, len(DISTS)))]
    scale = float(10.0 ** rng.uniform(-2, 2))
    t = float(10.0 ** rng.uniform(-4, 1)) * scale
    u = rng.uniform()
    k = float(max(0.2, min(n - 0.2, (u ** 2) * n)))
    if rng.uniform() < 0.3:
        k = float(max(1, min(n - 1, round(k))))
    return B, n, dist, scale, t, k


@pytest.mark.parametrize("seed", range(48))
def test_search_matches_oracle(cuda_device, seed):
    B, n, dist, scale, t, k = _case(seed)
    r, v = random_rows(8000 + seed, B, n, dist, scale=scale)
    res = run_gpu(r, k, t, path="auto", v=v)
    for i in range(B):
        check_row(r[i], v[i], k, t, res["b"][i], res["p"][i], res["g"][i],
                  label=f"seed {seed} B={B} n={n} {dist} t={t:.3g} k={k:.4g} row {i}",
                  sum_ref="auto")


@pytest.mark.parametrize("seed", range(0, 48, 4))
def test_forced_sort_matches_oracle(cuda_device, seed):
    """The same draws with every row sent on to the in-kernel sort."""
    B, n, dist, scale, t, k = _case(seed)
    r, v = random_rows(8000 + seed, B, n, dist, scale=scale)
    res = run_gpu(r, k, t, path=FORCE_SORT, v=v)
    for i in range(B):
        check_row(r[i], v[i], k, t, res["b"][i], res["p"][i], res["g"][i],
                  label=f"forced sort seed {seed} row {i}", sum_ref="auto")


@pytest.mark.parametrize("t", [1e-6, 1e-3, 0.05, 1.0, 1e3])
@pytest.mark.parametrize("k", [0.5, 1.0, 7.5, 8.0, 128.0, 255.0, 255.7])
def test_temperature_and_budget_extremes(cuda_device, t, k):
    """n = 256 N(0,1) rows from a staircase F (t far below the gaps: b between
    the two scores that bound the budget) to a nearly linear one (t far above
    the spread: b far outside the scores)."""
    r, v = random_rows(8100, 4, 256)
    res = run_gpu(r, k, t, path="auto", v=v)
    for i in range(4):
        check_row(r[i], v[i], k, t, res["b"][i], res["p"][i], res["g"][i],
                  label=f"t={t} k={k} row {i}", sum_ref="auto")


def test_degenerate_rows(cuda_device):
    rows, ks, ts = [], [], []
    n = 256
    rows.append(np.full(n, 0.75, np.float32)); ks.append(3.0); ts.append(0.1)       # all equal
    rows.append(np.full(n, -2.0, np.float32)); ks.append(200.0); ts.append(0.01)
    two = np.zeros(n, np.float32); two[::2] = 1.0
    rows.append(two); ks.append(64.0); ts.append(1e-4)                               # two values, b inside the top group
    rows.append(two.copy()); ks.append(128.0); ts.append(1e-4)                       # b between the groups
    rows.append(two.copy()); ks.append(128.0); ts.append(10.0)
    wide = np.linspace(-1e30, 1e30, n).astype(np.float32)
    rows.append(wide); ks.append(10.0); ts.append(1e27)                              # huge magnitudes
    tie = np.random.default_rng(5).permutation(np.repeat(np.arange(8, dtype=np.float32), 32))
    rows.append(tie); ks.append(40.0); ts.append(1e-3)                               # ties at the boundary
    signed = np.linspace(-1, 1, n).astype(np.float32); signed[:5] = -0.0; signed[5:10] = 0.0
    rows.append(signed); ks.append(128.0); ts.append(1e-3)                           # signed zeros near b
    for i, (row, k, t) in enumerate(zip(rows, ks, ts)):
        res = run_gpu(row[None, :], k, t, path="auto", v=np.ones((1, n), np.float32))
        check_row(row.astype(np.float32), np.ones(n, np.float32), k, t, res["b"][0],
                  res["p"][0], res["g"][0], label=f"degenerate {i}", sum_ref="auto")


def test_nonfinite_and_ragged_batch(cuda_device):
    B, n = 19, 150
    r, v = random_rows(8200, B, n)
    r[3, 17] = np.inf
    r[11, 0] = np.nan
    p, b = L.forward(torch.from_numpy(r).cuda(), 12.0, 0.05)
    torch.cuda.synchronize()
    p, b = p.cpu().numpy(), b.cpu().numpy()
    for i in range(B):
        if i in (3, 11):
            assert np.isnan(b[i]) and np.isnan(p[i]).all()
        else:
            check_row(r[i], v[i], 12.0, 0.05, b[i], p[i].astype(np.float64), label=f"row {i}")


def test_per_row_budgets(cuda_device):
    B, n, t = 64, 256, 0.05
    r, v = random_rows(8300, B, n)
    k_rows = np.random.default_rng(8301).uniform(0.5, n - 0.5, size=B)
    k_rows[::5] = np.round(k_rows[::5])
    rt = torch.from_numpy(r).cuda()
    p, b = L.forward(rt, torch.from_numpy(k_rows).cuda(), t)
    torch.cuda.synchronize()
    p, b = p.cpu().numpy(), b.cpu().numpy()
    for i in range(B):
        check_row(r[i], v[i], float(k_rows[i]), t, b[i], p[i].astype(np.float64),
                  label=f"row {i} k={k_rows[i]:.3f}", sum_ref="auto")


def test_search_agrees_with_sort(cuda_device):
    """The moe-router shape: the search and the bitonic sort give the same b
    to well inside the tolerance on every row."""
    B, n, k, t = 4096, 256, 8.0, 0.05
    r, _ = random_rows(8400, B, n)
    rt = torch.from_numpy(r).cuda()
    _, b1 = L.forward(rt, k, t, path="auto")
    _, b2 = L.forward(rt, k, t, path="fullsort")
    torch.cuda.synchronize()
    d = (b1 - b2).abs().max().item()
    assert d <= 3e-6 * t, d
    for i in (0, 1, 2047, 4095):
        assert abs(b1[i].item() - oracle.solve_b(r[i], k, t)) <= 1e-5 * max(t, abs(b1[i].item()))
