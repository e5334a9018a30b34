"""GPU parity of the bracketing steps themselves ("Fast LapSum: Exact
Differentiable Top-k at Million Scale", gist.science explainer pages,
section 2.2, probabilistic bracketing, steps 1-4).

* step 1: the GPU's sample equals the oracle's draw of the same counter-based
  SplitMix64 stream (indices exactly, values to fp32 rounding of the noise),
  and the bracket ends equal the oracle's order statistics of its own sample;
* step 2: the fold's tail counts and sums equal the oracle's fold over the
  oracle's bracket;
* steps 3-4: a bracket forced to miss is widened and still gives the exact b;
  with widening disabled the miss is reported, and b is NaN.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_selection_primitive_b200 as L
from tests.gpu_helpers import check_row
from workloads import random_rows

pytestmark = pytest.mark.gpu


def _forward(r, k, t, flags=0, seed=0):
    n = r.shape[-1]
    ws = L.Workspace(1, n, k, "bracket")
    rt = torch.from_numpy(r.reshape(1, -1)).cuda()
    p, b = L.forward(rt, k, t, path=2 | flags, seed=seed, ws=ws)
    torch.cuda.synchronize()
    return ws, p.cpu().numpy()[0].astype(np.float64), b.item()


# The order statistics come from one of three selections, by the number of
# sample keys in the wanted top-11-bit bins and above: one warp sorts them
# (a few, e.g. normal scores and a small budget), the whole block sorts them
# (up to 2048 of a 32768-key sample, e.g. the uniform half of mix_nu near its
# edge), or two radix levels narrow them (a dense top bin: uniform(3, 4)
# puts half the sample in [3.5, 4); or a short sample).
@pytest.mark.parametrize("n,k,t,seed,dist", [(200000, 150.0, 0.01, 0, "mix_nu"),
                                             (1 << 20, 1000.0, 0.005, 7, "mix_nu"),
                                             (50000, 25000.0, 0.3, 3, "mix_nu"),
                                             (1 << 20, 100.0, 0.01, 5, "normal"),
                                             (1 << 20, 2000.0, 0.002, 9, "uniform34")])
def test_sample_and_bracket_match_oracle(cuda_device, n, k, t, seed, dist):
    if dist == "uniform34":
        r = np.random.default_rng(seed).uniform(3.0, 4.0, (1, n)).astype(np.float32)
    else:
        r, _ = random_rows(seed, 1, n, dist)
    ws, _, _ = _forward(r[0], k, t, seed=seed)
    info = L.row_info(ws, 0)
    m = info["sample_m"]
    y_gpu = L.sample_values(ws, 0, m).astype(np.float64)
    y_ref, _ = oracle.sample(r[0], t, seed=seed, c0=0, m=m)
    assert np.max(np.abs(y_gpu - y_ref)) <= 1e-6 * max(1.0, np.max(np.abs(y_ref)))
    l, h = oracle.binom_ranks(m, k / n, 1e-6)
    assert (info["rank_l"], info["rank_h"]) == (l, h)
    aL, aR = oracle.bracket_from_sample(y_ref, l, h)
    if info["attempts"] == 1:
        assert abs(info["a_L"] - aL) <= 1e-6 * max(1.0, abs(aL)) or (aL == -math.inf and
                                                                     info["a_L"] == -math.inf)
        assert abs(info["a_R"] - aR) <= 1e-6 * max(1.0, abs(aR)) or (aR == math.inf and
                                                                    info["a_R"] == math.inf)


@pytest.mark.parametrize("n,k,t", [(300000, 200.0, 0.01), (1 << 21, 2000.0, 0.003)])
def test_fold_matches_oracle(cuda_device, n, k, t):
    r, _ = random_rows(11, 1, n, "normal")
    ws, _, _ = _forward(r[0], k, t)
    info = L.row_info(ws, 0)
    m = info["sample_m"]
    y_ref, _ = oracle.sample(r[0], t, seed=0, c0=0, m=m)
    l, h = oracle.binom_ranks(m, k / n, 1e-6)
    aL, aR = oracle.bracket_from_sample(y_ref, l, h)
    fo = oracle.fold(r[0], aL, aR, t)
    assert info["attempts"] == 1
    # the two brackets agree to fp32 rounding; scores falling between them may
    # change sides, so the counts may differ by exactly those scores
    lo_gap = np.sum((r[0] >= min(aL, info["a_L"])) & (r[0] < max(aL, info["a_L"])))
    hi_gap = np.sum((r[0] >= min(aR, info["a_R"])) & (r[0] < max(aR, info["a_R"])))
    assert abs(info["cnt_R"] - fo["cnt_R"]) <= hi_gap
    assert abs(info["n_band"] - fo["n_band"]) <= lo_gap + hi_gap
    if lo_gap == 0 and hi_gap == 0:
        assert info["cnt_R"] == fo["cnt_R"] and info["n_band"] == fo["n_band"]
        # The GPU's bracket ends are the oracle's up to the fp32 rounding of the
        # noise; with no score between them, moving an end rescales its tail
        # sum exactly:
        # S_R(a) = e^{a/t} sum e^{-r/t} and S_L(a) = e^{-a/t} sum e^{r/t}
        sr = info["S_R"] * math.exp((aR - info["a_R"]) / t) if math.isfinite(aR) else info["S_R"]
        sl = info["S_L"] * math.exp((info["a_L"] - aL) / t) if math.isfinite(aL) else info["S_L"]
        assert abs(sr - fo["S_R"]) <= 1e-5 * max(1.0, fo["S_R"])
        assert abs(sl - fo["S_L"]) <= 1e-5 * max(1.0, fo["S_L"])


@pytest.mark.parametrize("n", [20000, 400000])
def test_forced_miss_is_widened_and_exact(cuda_device, n):
    r, v = random_rows(5, 1, n)
    k, t = 60.0, 0.01
    ws, p, b = _forward(r[0], k, t, flags=L.FLAG_FORCE_MISS)
    info = L.row_info(ws, 0)
    assert info["attempts"] >= 2
    assert L.read_status(ws) == 0
    check_row(r[0], v[0], k, t, b, p, label=f"forced miss n={n}")


def test_forced_miss_without_retry_reports(cuda_device):
    r, _ = random_rows(6, 1, 30000)
    ws, _, b = _forward(r[0], 40.0, 0.01, flags=L.FLAG_FORCE_MISS | L.FLAG_NO_RETRY)
    assert L.read_status(ws) == 4
    assert math.isnan(b)
    assert L.row_info(ws, 0)["attempts"] == 1


def test_large_band_through_histogram(cuda_device):
    # q = 1/2 makes the binomial bracket hold ~n/10 scores: far more than the
    # on-chip sort, so the fold's band histogram picks the bin to solve on
    n = 1 << 20
    r, v = random_rows(8, 1, n, "normal_q64")
    k, t = n / 2.0, 0.05
    ws, p, b = _forward(r[0], k, t)
    info = L.row_info(ws, 0)
    assert info["n_band"] > 4096 and info["attempts"] == 1
    # k = n/2 on scores with heavy ties: the fp32 rounding of p alone moves
    # sum p by more than 1e-3, so the budget is checked against the sum of the
    # oracle's p rounded to fp32 (the best any fp32 output can do).
    check_row(r[0], v[0], k, t, b, p, label="large band", sum_ref="fp32")


def test_large_band_solved_in_one_cta(cuda_device):
    # The same large first band solved without the grid-wide extraction: the
    # single solve CTA walks the histogram and extracts the bin itself (the
    # path a band takes when it turns out far larger than the ranks predict).
    n = 1 << 20
    r, v = random_rows(8, 1, n, "normal_q64")
    k, t = n / 2.0, 0.05
    ws, p, b = _forward(r[0], k, t, flags=L.FLAG_ONE_CTA_SOLVE)
    info = L.row_info(ws, 0)
    assert info["n_band"] > 4096 and info["attempts"] == 1
    check_row(r[0], v[0], k, t, b, p, label="large band, one CTA", sum_ref="fp32")
    _, _, b2 = _forward(r[0], k, t)
    assert abs(b2 - b) <= 1e-12 * max(1.0, abs(b))


def test_large_band_exact_narrowing_after_a_miss(cuda_device):
    # After a failed first bracket the widened band is re-folded by one CTA
    # without a histogram, so it is narrowed by exact histogram levels.
    n = 1 << 19
    r, v = random_rows(12, 1, n, "normal")
    k, t = n / 4.0, 0.05
    ws, p, b = _forward(r[0], k, t, flags=L.FLAG_FORCE_MISS)
    info = L.row_info(ws, 0)
    assert info["attempts"] >= 2
    assert info["n_band"] > 4096
    assert info["refine_levels"] >= 1
    check_row(r[0], v[0], k, t, b, p, label="exact narrowing", sum_ref="fp32")
