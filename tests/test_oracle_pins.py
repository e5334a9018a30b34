"""Pins for the fp64 CPU oracle.

Each test ties an oracle function to something other than the oracle itself:
a closed form, a high-precision brute force that solves the budget equation by
a different method, an invariant of the definition, a limit the pages state,
finite differences, a published test vector or a library distribution.  The
definition pinned is the one in "Fast LapSum: Exact Differentiable Top-k at
Million Scale" (gist.science explainer pages), section 2.1 (operator, budget
constraint, analytic VJP), section 2.2 (bracketing) and section 2.3 (the zero
temperature limit is the midpoint threshold of DFTopK).
"""
import math
from decimal import Decimal, getcontext

import numpy as np
import pytest
from scipy import stats

import oracle
from workloads import random_rows


def sigma_inv(q: float) -> float:
    """Inverse of the Laplace(0,1) CDF."""
    return math.log(2 * q) if q < 0.5 else -math.log(2 * (1 - q))


def rel(b, ref, t):
    return abs(b - ref) / max(t, abs(ref))


# ---------------------------------------------------------------------------
# Brute force #2: every gap of the sorted order, solved in closed form with
# 60-digit decimals.  Independent of the oracle's bisection.
# ---------------------------------------------------------------------------
def brute_force_b(r, k, t, prec=60):
    getcontext().prec = prec
    s = sorted(Decimal(float(x)) for x in r)
    n = len(s)
    T = Decimal(float(t))
    K = Decimal(float(k))
    roots = []
    for j in range(n + 1):  # b in [s_{j-1}, s_j): s_0..s_{j-1} below, s_j.. at/above
        lo = s[j - 1] if j > 0 else None
        hi = s[j] if j < n else None
        if lo is not None and hi is not None and not lo < hi:
            continue
        A = sum(((-x / T).exp() for x in s[j:]), Decimal(0))   # sum e^{-s_i/t}, i >= j
        Bs = sum(((x / T).exp() for x in s[:j]), Decimal(0))   # sum e^{ s_i/t}, i <  j
        c = Decimal(n - j) - K
        if A > 0:
            S = (c * c + A * Bs).sqrt()
            # positive root of A z^2 - 2 c z - B = 0, in the form without cancellation
            z = (c + S) / A if c >= 0 else Bs / (S - c)
        else:
            if K - Decimal(n - j) <= 0:
                continue
            z = Bs / (2 * (K - Decimal(n - j)))
        if z <= 0:
            continue
        b = T * z.ln()
        if (lo is None or b >= lo) and (hi is None or b < hi):
            roots.append(b)
    assert len(roots) == 1, roots
    return float(roots[0])


@pytest.mark.parametrize("seed", range(40))
def test_bisection_matches_segment_brute_force(seed):
    rng = np.random.default_rng(1000 + seed)
    n = int(rng.integers(1, 13))
    t = float(10 ** rng.uniform(-3, math.log10(5)))
    r = rng.standard_normal(n).astype(np.float32)
    if seed % 4 == 0 and n >= 3:  # exact ties
        r[1] = r[0]
        r[2] = r[0]
    k = float(rng.uniform(0.05, n - 0.05)) if seed % 2 else float(rng.integers(1, n)) if n > 1 else 0.5
    b = oracle.solve_b(r, k, t)
    ref = brute_force_b(r, k, t)
    assert rel(b, ref, t) <= 1e-12, (b, ref, n, k, t)


def test_single_score_closed_form():
    for r0 in (-2.5, 0.0, 1.25):
        for k in (0.01, 0.3, 0.5, 0.8, 0.999):
            for t in (0.01, 1.0):
                b = oracle.solve_b([r0], k, t)
                assert rel(b, r0 - t * sigma_inv(k), t) <= 1e-13


def test_all_equal_row():
    n, c, t = 37, 1.75, 0.2
    for k in (1.0, 5.5, 18.5, 36.0):
        r = np.full(n, c, dtype=np.float32)
        b = oracle.solve_b(r, k, t)
        assert rel(b, c - t * sigma_inv(k / n), t) <= 1e-13
        p = oracle.emit_p(r, b, t)
        assert np.allclose(p, k / n, rtol=0, atol=1e-13)


def test_two_point_symmetry():
    for d in (0.001, 0.5, 3.0, 40.0):
        for t in (0.001, 0.1, 10.0):
            b = oracle.solve_b([0.0, d], 1.0, t)
            assert abs(b - d / 2) <= 1e-13 * max(t, d)


# ---------------------------------------------------------------------------
# Invariants of the definition.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("seed", range(6))
def test_invariants(seed):
    r, _ = random_rows(seed, 1, 200)
    r = r[0].astype(np.float64)
    k, t = 17.0, 0.07
    b = oracle.solve_b(r, k, t)
    # shift (3.0 + float32 value is exact in fp64)
    assert rel(oracle.solve_b(r + 3.0, k, t), b + 3.0, t) <= 1e-12
    # scale: b(a r, a t) = a b(r, t)
    assert rel(oracle.solve_b(3.0 * r, k, 3.0 * t), 3.0 * b, 3.0 * t) <= 1e-12
    # permutation
    perm = np.random.default_rng(seed).permutation(r.size)
    assert oracle.solve_b(r[perm], k, t) == b
    # mirror: b(-r, n-k) = -b(r, k), p(-r, n-k) = 1 - p(r, k)
    bm = oracle.solve_b(-r, r.size - k, t)
    assert rel(bm, -b, t) <= 1e-12
    p = oracle.emit_p(r, b, t)
    pm = oracle.emit_p(-r, bm, t)
    assert np.max(np.abs(pm - (1 - p))) <= 1e-12


@pytest.mark.parametrize("dist,k,t", [("normal", 10, 0.1), ("normal", 128, 0.01),
                                      ("normal_q64", 40, 0.02), ("abs_t3", 3, 0.01),
                                      ("mix_nu", 25, 0.005)])
def test_budget_and_probabilities(dist, k, t):
    r, _ = random_rows(7, 1, 4000, dist)
    r = r[0]
    b = oracle.solve_b(r, k, t)
    p = oracle.emit_p(r, b, t)
    assert abs(oracle.budget_sum(r, b, t) - k) <= 1e-9 * k
    assert abs(p.sum() - k) <= 1e-9 * k
    assert p.min() >= 0.0 and p.max() <= 1.0
    order = np.argsort(r, kind="stable")
    assert np.all(np.diff(p[order]) >= 0.0)  # monotone in r
    f = oracle.density(r, b, t)
    # 1 - p near p = 1 carries fp64 rounding of order 1e-16
    assert np.allclose(f, np.minimum(p, 1 - p), rtol=1e-12, atol=1e-15)


def test_sign_function_on_flat_plateau():
    # Gap 1, t = 1e-3: F is flat to ~e^-500 between neighbours; a plain sum of
    # sigma rounds to k on the whole plateau.  The sign function must still
    # put b at the midpoint (c = 0 branch, L vs U).
    r = np.arange(10, dtype=np.float64)
    t = 1e-3
    b = oracle.solve_b(r, 3.0, t)
    assert abs(b - 6.5) <= 1e-12
    assert oracle.budget_sign(r, 6.49, 3.0, t) > 0
    assert oracle.budget_sign(r, 6.51, 3.0, t) < 0


# ---------------------------------------------------------------------------
# Zero temperature limit (section 2.3): the threshold tends to the midpoint of
# the k-th and (k+1)-th largest scores, p to the hard top-k mask.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("k", [1, 5, 64, 250])
def test_zero_temperature_limit(k):
    n, t = 300, 0.01
    r = np.random.default_rng(k).permutation(n).astype(np.float64)  # gap 1
    b = oracle.solve_b(r, float(k), t)
    srt = np.sort(r)[::-1]
    mid = 0.5 * (srt[k - 1] + srt[k])
    assert abs(b - mid) <= 10 * t * math.exp(-1.0 / t)
    p = oracle.emit_p(r, b, t)
    mask = (r >= srt[k - 1]).astype(np.float64)
    assert np.max(np.abs(p - mask)) <= math.exp(-1.0 / (2 * t))


# ---------------------------------------------------------------------------
# VJP: algebraic identities, PSD, symmetry, and central finite differences.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("seed", range(4))
def test_vjp_identities(seed):
    r, v = random_rows(100 + seed, 1, 500)
    r, v = r[0], v[0]
    k, t = 20.0, 0.2
    b = oracle.solve_b(r, k, t)
    g, R, sf = oracle.vjp(r, v, b, t)
    scale = np.max(np.abs(g))
    assert abs(g.sum()) <= 1e-12 * scale * r.size
    g0, _, _ = oracle.vjp(r, np.full_like(v, 0.37), b, t)
    assert np.max(np.abs(g0)) <= 1e-15
    assert float(np.dot(v.astype(np.float64), g)) >= 0.0
    f = oracle.density(r, b, t)
    assert abs(sf - f.sum()) <= 1e-12 * f.sum()


def _loss(r, v, k, t):
    b = oracle.solve_b(r, k, t)
    return float(np.dot(v, oracle.emit_p(r, b, t)))


@pytest.mark.parametrize("seed,n,k,t", [(0, 12, 3.0, 0.5), (1, 40, 7.5, 0.2),
                                        (2, 64, 16.0, 0.05), (3, 9, 1.0, 2.0)])
def test_vjp_central_finite_differences(seed, n, k, t):
    rng = np.random.default_rng(200 + seed)
    r = rng.standard_normal(n)
    v = rng.standard_normal(n)
    b = oracle.solve_b(r, k, t)
    g, _, _ = oracle.vjp(r, v, b, t)
    h = 1e-5 * t
    checked = 0
    for j in range(n):
        if abs(r[j] - b) < 10 * h:
            continue
        rp, rm = r.copy(), r.copy()
        rp[j] += h
        rm[j] -= h
        fd = (_loss(rp, v, k, t) - _loss(rm, v, k, t)) / (2 * h)
        assert abs(fd - g[j]) <= 1e-6 * max(1.0, np.max(np.abs(g))), (j, fd, g[j])
        checked += 1
    assert checked >= n - 1


@pytest.mark.parametrize("seed,n,k,t", [(0, 12, 3.0, 0.5), (1, 40, 7.5, 0.05), (2, 64, 1.5, 2.0),
                                        (3, 30, 20.0, 0.01)])
def test_vjp_kt_central_finite_differences(seed, n, k, t):
    # dL/dk and dL/dt of L = sum v p against central differences of the full
    # solve (b to full fp64 resolution at each shifted k or t)
    rng = np.random.default_rng(300 + seed)
    r = rng.standard_normal(n)
    v = rng.standard_normal(n)
    b = oracle.solve_b(r, k, t)
    gk, gt = oracle.vjp_kt(r, v, b, t)
    hk, ht = 1e-6 * max(1.0, k), 1e-6 * t
    fdk = (_loss(r, v, k + hk, t) - _loss(r, v, k - hk, t)) / (2 * hk)
    fdt = (_loss(r, v, k, t + ht) - _loss(r, v, k, t - ht)) / (2 * ht)
    assert abs(fdk - gk) <= 1e-6 * max(1.0, abs(gk)), (fdk, gk)
    assert abs(fdt - gt) <= 1e-5 * max(1.0, abs(gt)), (fdt, gt)


def test_vjp_kt_identities():
    # sum p = k for every k and t: with v = 1, dL/dk = 1 and dL/dt = 0; both
    # gradients are linear in v, and a constant shift of the scores moves neither
    rng = np.random.default_rng(9)
    n, k, t = 25, 4.0, 0.3
    r = rng.standard_normal(n)
    b = oracle.solve_b(r, k, t)
    gk, gt = oracle.vjp_kt(r, np.ones(n), b, t)
    assert abs(gk - 1.0) <= 1e-12 and abs(gt) <= 1e-12
    v1, v2 = rng.standard_normal(n), rng.standard_normal(n)
    a1, a2 = oracle.vjp_kt(r, v1, b, t), oracle.vjp_kt(r, v2, b, t)
    a3 = oracle.vjp_kt(r, 2.0 * v1 - 3.0 * v2, b, t)
    assert abs(a3[0] - (2 * a1[0] - 3 * a2[0])) <= 1e-12
    assert abs(a3[1] - (2 * a1[1] - 3 * a2[1])) <= 1e-10
    c = 5.5
    bs = oracle.solve_b(r + c, k, t)
    s1 = oracle.vjp_kt(r + c, v1, bs, t)
    assert abs(s1[0] - a1[0]) <= 1e-10 and abs(s1[1] - a1[1]) <= 1e-8


def test_jacobian_symmetric_and_matches_fd():
    rng = np.random.default_rng(5)
    n, k, t = 8, 3.0, 0.3
    r = rng.standard_normal(n)
    b = oracle.solve_b(r, k, t)
    J = np.stack([oracle.vjp(r, np.eye(n)[i], b, t)[0] for i in range(n)])  # J[i, j] = dp_i/dr_j
    assert np.allclose(J, J.T, rtol=0, atol=1e-14)
    assert np.min(np.linalg.eigvalsh(0.5 * (J + J.T))) >= -1e-12
    h = 1e-6
    for j in range(n):
        rp, rm = r.copy(), r.copy()
        rp[j] += h
        rm[j] -= h
        pp = oracle.emit_p(rp, oracle.solve_b(rp, k, t), t)
        pm = oracle.emit_p(rm, oracle.solve_b(rm, k, t), t)
        assert np.allclose((pp - pm) / (2 * h), J[:, j], rtol=0, atol=1e-7)


# ---------------------------------------------------------------------------
# Bracketing (section 2.2): generator, sample law, binomial ranks, fold.
# ---------------------------------------------------------------------------
def test_splitmix64_published_vector():
    # First outputs of SplitMix64 seeded with 0 (the generator's reference test vector).
    want = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F, 0xF88BB8A8724C81EC]
    assert [oracle.splitmix64_at(0, c) for c in range(4)] == want


def test_sample_noise_is_laplace_and_indices_uniform():
    n, t, m = 1000, 0.3, 40000
    y, idx = oracle.sample(np.zeros(n), t, seed=12345, c0=0, m=m)
    assert stats.kstest(y, stats.laplace(scale=t).cdf).pvalue > 1e-3
    counts = np.bincount(idx, minlength=n)
    assert idx.min() >= 0 and idx.max() < n
    assert stats.chisquare(counts).pvalue > 1e-3


@pytest.mark.parametrize("m,q,alpha", [(32768, 1e-3, 1e-6), (32768, 1.8e-4, 1e-6),
                                       (4096, 0.25, 1e-3), (1000, 0.5, 0.05), (100, 0.02, 0.01)])
def test_binomial_ranks_match_scipy(m, q, alpha):
    l, h = oracle.binom_ranks(m, q, alpha)
    dist = stats.binom(m, q)
    # l: largest with P(C < l) <= alpha
    assert l == 0 or dist.cdf(l - 1) <= alpha * (1 + 1e-9)
    assert dist.cdf(l) > alpha * (1 - 1e-9)
    # h: smallest with P(C >= h) <= alpha
    assert h == m + 1 or dist.sf(h - 1) <= alpha * (1 + 1e-9)
    assert dist.sf(h - 2) > alpha * (1 - 1e-9)


def test_bracket_coverage_rate_matches_binomial_tail():
    r, _ = random_rows(3, 1, 2000)
    r = r[0]
    k, t, m, alpha = 50.0, 0.05, 400, 0.05
    b = oracle.solve_b(r, k, t)
    l, h = oracle.binom_ranks(m, k / r.size, alpha)
    misses, trials = 0, 400
    for s in range(trials):
        y, _ = oracle.sample(r, t, seed=777, c0=2 * m * s, m=m)
        aL, aR = oracle.bracket_from_sample(y, l, h)
        misses += not (aL <= b < aR)
    dist = stats.binom(m, k / r.size)
    p_miss = dist.cdf(l - 1) + dist.sf(h - 1)
    sd = math.sqrt(trials * p_miss * (1 - p_miss))
    assert abs(misses - trials * p_miss) <= 4 * sd + 2, (misses, trials * p_miss)


def test_fold_reconstructs_budget_inside_bracket():
    r, _ = random_rows(4, 1, 5000, "mix_nu")
    r = r[0]
    k, t = 40.0, 0.01
    b = oracle.solve_b(r, k, t)
    aL, aR = b - 0.05, b + 0.03
    fo = oracle.fold(r, aL, aR, t)
    assert fo["cnt_R"] + fo["cnt_L"] + fo["n_band"] == r.size
    band = r[(r >= aL) & (r < aR)].astype(np.float64)
    assert band.size == fo["n_band"]
    for bb in (aL, b, 0.5 * (aL + aR), aR):
        Fb = (fo["cnt_R"] - 0.5 * fo["S_R"] * math.exp((bb - aR) / t)
              + 0.5 * fo["S_L"] * math.exp((aL - bb) / t)
              + sum(oracle.laplace_cdf((x - bb) / t) for x in band))
        assert abs(Fb - oracle.budget_sum(r, bb, t)) <= 1e-9 * max(1.0, Fb)


def test_rejects_invalid_arguments():
    with pytest.raises(oracle.OracleError):
        oracle.solve_b([1.0, 2.0], 0.0, 1.0)
    with pytest.raises(oracle.OracleError):
        oracle.solve_b([1.0, 2.0], 2.0, 1.0)
    with pytest.raises(oracle.OracleError):
        oracle.solve_b([1.0, 2.0], 1.0, 0.0)
    with pytest.raises(oracle.OracleError):
        oracle.solve_b([1.0, float("nan")], 1.0, 1.0)


def test_bracket_order_statistics():
    # a_R is the l-th largest sample, a_L the h-th largest; l = 0 / h = m + 1 open the side.
    y = np.random.default_rng(9).standard_normal(101)
    desc = np.sort(y)[::-1]
    for l, h in [(1, 2), (3, 17), (50, 101), (0, 5), (4, 102)]:
        aL, aR = oracle.bracket_from_sample(y, l, h)
        assert aR == (desc[l - 1] if l >= 1 else math.inf)
        assert aL == (desc[h - 1] if h <= y.size else -math.inf)


# ---------------------------------------------------------------------------
# Zero-temperature limit (hard top-k): "Fast LapSum: Exact Differentiable Top-k
# at Million Scale" (gist.science explainer pages), section 2.3: DFTopK's
# midpoint threshold is the t -> 0 limit of LapSum.  Pinned by hand-worked
# cases, by the soft oracle itself at a temperature far below the gaps (a
# different code path: bisection on the smooth budget), and by invariants.
# ---------------------------------------------------------------------------

def test_hard_topk_worked_cases():
    # integer k at a gap: midpoint of the k-th and (k+1)-th largest, 0/1 mask
    b, p = oracle.hard_topk([5.0, 4.0, 3.0, 1.0], 2.0)
    assert b == 3.5 and list(p) == [1.0, 1.0, 0.0, 0.0]
    # a tie group straddles the budget: b is the tied value, the group shares
    # the remaining budget equally
    b, p = oracle.hard_topk([3.0, 2.0, 2.0, 2.0, 1.0], 2.0)
    assert b == 2.0 and np.allclose(p, [1.0, 1 / 3, 1 / 3, 1 / 3, 0.0], rtol=0, atol=1e-15)
    # a fractional budget lands on one score
    b, p = oracle.hard_topk([5.0, 4.0, 3.0], 1.5)
    assert b == 4.0 and list(p) == [1.0, 0.5, 0.0]
    # the whole tie group inside the budget: a gap below it
    b, p = oracle.hard_topk([7.0, 6.0, 6.0, 2.0, 0.0], 3.0)
    assert b == 4.0 and list(p) == [1.0, 1.0, 1.0, 0.0, 0.0]


@pytest.mark.parametrize("seed,n,k,grid", [(0, 40, 7.0, 0.0), (1, 25, 12.0, 0.25),
                                           (2, 60, 13.5, 0.0), (3, 33, 4.25, 0.5)])
def test_hard_topk_is_the_soft_solution_at_tiny_temperature(seed, n, k, grid):
    rng = np.random.default_rng(seed)
    r = rng.standard_normal(n)
    if grid > 0:
        r = np.round(r / grid) * grid  # ties, at the boundary for some k
    b_h, p_h = oracle.hard_topk(r, k)
    gaps = np.diff(np.unique(r))
    t = float(np.min(gaps)) / 80.0    # every neighbour weight below e^-80
    b_s = oracle.solve_b(r, k, t)
    p_s = oracle.emit_p(r, b_s, t)
    assert abs(b_s - b_h) <= 3 * t   # the soft b sits within a few t of the limit
    # p at a score equal to b moves by db/(2t): allow a few fp64 ulps of b over t
    tol_p = max(1e-12, 8 * np.finfo(float).eps * max(1.0, abs(b_s)) / t)
    assert np.max(np.abs(p_s - p_h)) <= tol_p
    assert abs(np.sum(p_h) - k) <= 1e-12


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_hard_topk_invariants(seed):
    rng = np.random.default_rng(seed)
    n = 50
    r = np.round(rng.standard_normal(n) * 4) / 4
    for k in (1.0, 9.0, 17.5, 48.75):
        b, p = oracle.hard_topk(r, k)
        assert abs(np.sum(p) - k) <= 1e-12
        assert np.all((p >= 0) & (p <= 1))
        order = np.argsort(r)
        assert np.all(np.diff(p[order]) >= 0)          # monotone in r
        perm = rng.permutation(n)
        b2, p2 = oracle.hard_topk(r[perm], k)          # permutation
        assert b2 == b and np.array_equal(p2, p[perm])
        b3, p3 = oracle.hard_topk(r + 2.5, k)          # shift
        assert b3 == b + 2.5 and np.array_equal(p3, p)
        b4, p4 = oracle.hard_topk(-r, n - k)           # mirror
        assert b4 == -b and np.allclose(p4, 1.0 - p, rtol=0, atol=1e-15)
