"""Seeded random sweep of the whole surface against the oracle.

"Fast LapSum: Exact Differentiable Top-k at Million Scale" (gist.science
explainer pages), sections 2.1-2.2: every solver computes the same b, p and
VJP, so a random draw of shape, budget, temperature, score distribution and
solver must match the oracle at the parity tolerances.  The draw is seeded
(one case per seed), sizes stay small enough for the oracle to finish in a
fraction of a second per row, and lengths are ragged on purpose.
"""
import numpy as np
import pytest
import torch

import sparse_selection_primitive_b200 as L
from tests.gpu_helpers import check_row, run_gpu
from workloads import random_rows

pytestmark = pytest.mark.gpu

DISTS = ["normal", "normal_q64", "abs_t3", "mix_nu"]


def _case(seed):
    rng = np.random.default_rng(1000 + seed)
    path = ["auto", "fullsort", "radix", "rowbracket", "bracket"][seed % 5]
    if path == "fullsort":
        n = int(rng.integers(2, 4097))
    elif path in ("radix", "rowbracket"):
        n = int(rng.integers(4097, 70000))
    elif path == "bracket":
        n = int(rng.integers(20000, 400000))
    else:
        n = int(rng.choice([rng.integers(2, 4097), rng.integers(4097, 300000)]))
    B = int(rng.integers(1, 4)) if n > 4096 else int(rng.integers(1, 40))
    dist = DISTS[int(rng.integers(0, len(DISTS)))]
    scale = float(10.0 ** rng.uniform(-2, 2))
    t = float(10.0 ** rng.uniform(-3, 0)) * scale
    u = rng.uniform()
    k = float(max(0.3, min(n - 0.3, (u ** 3) * n)))  # small budgets more often
    if rng.uniform() < 0.3:
        k = float(max(1, round(k)))
    return path, B, n, dist, scale, t, k


@pytest.mark.parametrize("seed", range(30))
def test_random_case_matches_oracle(cuda_device, seed):
    path, B, n, dist, scale, t, k = _case(seed)
    r, v = random_rows(2000 + seed, B, n, dist, scale=scale)
    support = n > 4096 and seed % 2 == 0
    res = run_gpu(r, k, t, path=path, v=v, seed=seed, support=support)
    for i in range(B):
        check_row(r[i], v[i], k, t, res["b"][i], res["p"][i], res["g"][i],
                  label=f"seed {seed} {path} B={B} n={n} {dist} scale={scale:.3g} "
                        f"t={t:.3g} k={k:.4g} row {i}", sum_ref="auto")
