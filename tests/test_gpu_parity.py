"""GPU parity of every solver against the fp64 oracle on seeded inputs.

Sizes are chosen so the oracle finishes in seconds while the CUDA path still
crosses its tile boundaries (warp, CTA, 4096-key bitonic capacity, 4096-key
radix tiles) and ragged tails.  Solvers: the on-chip bitonic full sort, the
radix full sort, and probabilistic bracketing, each also forced onto sizes it
would not pick by itself.
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

SIZES_ONCHIP = [1, 2, 3, 7, 31, 32, 33, 64, 100, 255, 256, 257, 511, 1000, 1024, 2047, 2049, 4095,
                4096]
SIZES_LONG = [4097, 5000, 8192, 12345, 65536, 70001]


def k_values(n):
    ks = {min(n - 0.5, 0.5), max(0.25, n / 3.0)}
    if n > 2:
        ks |= {1.0, float(n - 1), float(max(1, n // 8))}
    return sorted(k for k in ks if 0 < k < n)


@pytest.mark.parametrize("n", SIZES_ONCHIP)
def test_onchip_bitonic_sizes(cuda_device, n):
    B = 3
    r, v = random_rows(10 + n, B, n)
    for k in k_values(n):
        for t in (0.05, 1.0):
            out = run_gpu(r, k, t, path="fullsort", v=v)
            for i in range(B):
                check_row(r[i], v[i], k, t, out["b"][i], out["p"][i], out["g"][i],
                          label=f"bitonic n={n} k={k} t={t} row={i}")


@pytest.mark.parametrize("n", [300, 4096, 5000, 12345, 70001])
def test_radix_sizes(cuda_device, n):
    B = 2
    r, v = random_rows(20 + n, B, n)
    for k in k_values(n):
        out = run_gpu(r, k, 0.05, path="radix", v=v)
        for i in range(B):
            check_row(r[i], v[i], k, 0.05, out["b"][i], out["p"][i], out["g"][i],
                      label=f"radix n={n} k={k} row={i}")


@pytest.mark.parametrize("n,dist", [(262145, "normal"), (300001, "normal_q64"),
                                    (1_000_003, "mix_nu"), (2_500_000, "abs_t3")])
def test_radix_long_rows(cuda_device, n, dist):
    """Rows past 4 x 65536 keys: the sorted row is solved over the whole GPU in
    chunks (closed-form chunk maps, then the crossing chunk solved with the rest
    folded into two anchors); ragged last chunks, ties, both temperatures.
    The budget bar |sum p - k| <= 1e-3 applies whenever the oracle's own p,
    rounded to fp32, meet it (sum_ref="auto"); b, p and g keep their own
    tolerances.  The soft case (t = 1, 10^5 to 10^6 probabilities away from 0
    and 1, ~600 scores per value on the quantised row) holds that bar because
    soft rows form p in fp64 and round it once."""
    B = 2
    r, v = random_rows(30 + n, B, n, dist)
    for k, t in ((1.0, 0.05), (n / 3.0 + 0.37, 1.0), (float(n // 100), 0.01), (n - 0.5, 0.05)):
        out = run_gpu(r, k, t, path="radix", v=v)
        for i in range(B):
            check_row(r[i], v[i], k, t, out["b"][i], out["p"][i], out["g"][i],
                      label=f"radix {dist} n={n} k={k} t={t} row={i}", sum_ref="auto")


@pytest.mark.parametrize("n,dist,path", [(262145, "normal", "rowbracket"),
                                         (1_000_003, "abs_t3", "bracket"),
                                         (600_001, "normal_q64", "bracket")])
def test_bracketing_soft_long_rows(cuda_device, n, dist, path):
    """Soft rows (t = 1, far above the gaps: every score carries weight) of
    2.6e5 to 1e6 scores through both bracketing arrangements: the fold's tail
    terms and p are formed in fp64 on such rows, so that the budget bar holds
    over 10^5 to 10^6 probabilities away from 0 and 1."""
    r, v = random_rows(50 + n, 1, n, dist)
    for k in (n / 3.0 + 0.37, float(n // 10)):
        out = run_gpu(r, k, 1.0, path=path, v=v)
        check_row(r[0], v[0], k, 1.0, out["b"][0], out["p"][0], out["g"][0],
                  label=f"{path} {dist} n={n} k={k} t=1", sum_ref="auto")


@pytest.mark.parametrize("n", [2, 100, 4097, 8191, 65536, 70001, 300000])
def test_rowbracket_sizes(cuda_device, n):
    B = 3
    r, v = random_rows(40 + n, B, n)
    for k in k_values(n):
        out = run_gpu(r, k, 0.02, path="rowbracket", v=v)
        for i in range(B):
            check_row(r[i], v[i], k, 0.02, out["b"][i], out["p"][i], out["g"][i],
                      label=f"rowbracket n={n} k={k} row={i}")


@pytest.mark.parametrize("n", [64, 5000, 65536, 300000])
def test_bracket_sizes(cuda_device, n):
    r, v = random_rows(30 + n, 1, n)
    for k in k_values(n):
        out = run_gpu(r, k, 0.02, path="bracket", v=v)
        check_row(r[0], v[0], k, 0.02, out["b"][0], out["p"][0], out["g"][0],
                  label=f"bracket n={n} k={k}")


@pytest.mark.parametrize("dist", ["normal", "normal_q64", "abs_t3", "mix_nu"])
@pytest.mark.parametrize("path", ["fullsort", "radix", "bracket", "rowbracket"])
def test_distributions_and_ties(cuda_device, dist, path):
    n = 3000 if path == "fullsort" else 20000
    r, v = random_rows(7, 2, n, dist)
    for k, t in [(10.0, 0.1), (123.5, 0.01), (n / 2, 0.3)]:
        out = run_gpu(r, k, t, path=path, v=v)
        for i in range(2):
            check_row(r[i], v[i], k, t, out["b"][i], out["p"][i], out["g"][i],
                      label=f"{path} {dist} k={k} t={t}")


@pytest.mark.parametrize("path", ["fullsort", "radix", "bracket", "rowbracket"])
def test_degenerate_rows(cuda_device, path):
    n = 1000 if path == "fullsort" else 9000
    # all equal: p = k/n everywhere
    r = np.full((1, n), 1.25, dtype=np.float32)
    v = np.random.default_rng(0).standard_normal((1, n)).astype(np.float32)
    out = run_gpu(r, 7.0, 0.1, path=path, v=v)
    check_row(r[0], v[0], 7.0, 0.1, out["b"][0], out["p"][0], out["g"][0], label="all equal")
    # two distinct values, huge gap relative to t (flat plateau of F)
    r2 = np.zeros((1, n), dtype=np.float32)
    r2[0, : n // 10] = 5.0
    out = run_gpu(r2, float(n // 10), 1e-3, path=path, v=v)
    check_row(r2[0], v[0], float(n // 10), 1e-3, out["b"][0], out["p"][0], out["g"][0],
              label="plateau")
    # wide score range
    r3, _ = random_rows(5, 1, n)
    r3 = (r3 * 1e4).astype(np.float32)
    out = run_gpu(r3, 50.0, 30.0, path=path, v=v)
    check_row(r3[0], v[0], 50.0, 30.0, out["b"][0], out["p"][0], out["g"][0], label="wide")
    # tiny temperature, well separated scores: close to the hard top-k mask
    r4 = np.random.default_rng(3).permutation(n).astype(np.float32)[None, :]
    out = run_gpu(r4, 17.0, 1e-3, path=path, v=v)
    check_row(r4[0], v[0], 17.0, 1e-3, out["b"][0], out["p"][0], out["g"][0], label="t->0")


def test_k_extremes(cuda_device):
    n = 777
    r, v = random_rows(9, 1, n)
    for k in (1e-6, 1e-3, n - 1e-3, n - 1e-6):
        for path in ("fullsort", "radix", "bracket", "rowbracket"):
            out = run_gpu(r, k, 0.2, path=path, v=v)
            check_row(r[0], v[0], k, 0.2, out["b"][0], out["p"][0], out["g"][0],
                      label=f"{path} k={k}")


def test_strided_rows_and_unaligned(cuda_device):
    # ld > n and a base pointer that is not 16-byte aligned take the scalar paths
    B, n, ld = 5, 300, 333
    r, v = random_rows(11, B, ld)
    full = torch.from_numpy(r).cuda()
    vv = torch.from_numpy(v).cuda()
    for path in ("fullsort", "radix", "rowbracket"):
        sub = full[:, 1:1 + n]
        p, b = L.forward(sub, 12.0, 0.1, path=path)
        g = L.backward(sub, b, vv[:, 1:1 + n], 0.1)
        for i in range(B):
            check_row(r[i, 1:1 + n], v[i, 1:1 + n], 12.0, 0.1, b[i].item(),
                      p[i].cpu().numpy().astype(np.float64), g[i].cpu().numpy().astype(np.float64),
                      label=f"strided {path} row={i}")


def test_nonfinite_scores_reported(cuda_device):
    for path, n in (("fullsort", 100), ("radix", 5000), ("bracket", 5000), ("rowbracket", 5000)):
        r, _ = random_rows(1, 2, n)
        r[1, n // 2] = np.nan
        ws = L.Workspace(2, n, 3.0, path)
        _, b = L.forward(torch.from_numpy(r).cuda(), 3.0, 0.1, path=path, ws=ws)
        assert L.read_status(ws) == 3, path
        bb = b.cpu().numpy()
        assert math.isnan(bb[1]), path
        if path != "bracket":  # the grid pipeline solves one row at a time
            assert not math.isnan(bb[0])
        assert L.read_status(ws) == 0  # cleared by the read


def test_sum_f_output(cuda_device):
    for path, n in (("fullsort", 1000), ("radix", 6000), ("bracket", 6000), ("rowbracket", 6000)):
        r, _ = random_rows(2, 2, n)
        out = run_gpu(r, 20.0, 0.05, path=path, want_sum_f=True)
        for i in range(2):
            f = oracle.density(r[i], oracle.solve_b(r[i], 20.0, 0.05), 0.05)
            assert abs(out["sum_f"][i] - f.sum()) <= 1e-4 * f.sum()


def test_autograd_matches_library_backward(cuda_device):
    r, v = random_rows(4, 3, 600)
    rt = torch.from_numpy(r).cuda().requires_grad_(True)
    p = L.soft_topk(rt, 9.0, 0.1)
    p.backward(torch.from_numpy(v).cuda())
    _, b = L.forward(rt.detach(), 9.0, 0.1)
    g = L.backward(rt.detach(), b, torch.from_numpy(v).cuda(), 0.1)
    assert torch.equal(rt.grad, g)


def test_repeat_calls_are_deterministic(cuda_device):
    for path, n in (("fullsort", 2000), ("radix", 20000), ("bracket", 20000),
                    ("rowbracket", 20000)):
        r, v = random_rows(6, 2, n)
        a = run_gpu(r, 50.0, 0.05, path=path, v=v)
        c = run_gpu(r, 50.0, 0.05, path=path, v=v)
        assert np.array_equal(a["b"], c["b"]), path
        assert np.array_equal(a["p"], c["p"]), path
        assert np.array_equal(a["g"], c["g"]), path


# ---------------------------------------------------------------------------
# Windowed backward of long rows: only |x| <= 90 carries gradient in fp32.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("n,k,t,dist", [
    (1 << 20, 1000.0, 0.001, "normal"),     # window ~4% of the row: served by the window pass
    (1 << 18, 2000.0, 0.05, "normal"),      # window holds the whole row: list overflow, dense
    (300001, 77.0, 0.0004, "mix_nu"),       # odd length, scalar tail of the window pass
])
def test_windowed_backward(cuda_device, n, k, t, dist):
    r, v = random_rows(51, 1, n, dist)
    out = run_gpu(r, k, t, path="radix" if n <= (1 << 20) else "bracket", v=v)
    check_row(r[0], v[0], k, t, out["b"][0], out["p"][0], out["g"][0], label=f"window n={n}")


def test_windowed_backward_far_threshold_falls_back(cuda_device):
    # gap 1 and t = 0.008: the nearest scores sit at |x| = 62.5, inside the
    # window but above 50, so the row is recomputed by the dense kernels
    n = 6000
    r = np.random.default_rng(4).permutation(n).astype(np.float32)[None, :]
    v = np.random.default_rng(5).standard_normal((1, n)).astype(np.float32)
    out = run_gpu(r, 17.0, 0.008, path="radix", v=v)
    check_row(r[0], v[0], 17.0, 0.008, out["b"][0], out["p"][0], out["g"][0], label="far")


# ---------------------------------------------------------------------------
# Gradient support handed from the forward to the backward (rows > 4096).
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("B,n,k,t,dist,path", [
    (1, 1 << 20, 1000.0, 0.001, "normal", "radix"),     # sparse support, full tiles
    (1, 1 << 18, 2000.0, 0.05, "normal", "radix"),      # support above half of every share: dense
    (1, 300001, 77.0, 0.0004, "mix_nu", "bracket"),     # ragged last tile
    (3, 70001, 500.0, 0.01, "normal_q64", "radix"),     # several rows, ties
    (2, 20000, 123.5, 0.01, "abs_t3", "bracket"),
])
def test_support_backward(cuda_device, B, n, k, t, dist, path):
    r, v = random_rows(61 + n, B, n, dist)
    out = run_gpu(r, k, t, path=path, v=v, support=True)
    for i in range(B):
        check_row(r[i], v[i], k, t, out["b"][i], out["p"][i], out["g"][i],
                  label=f"support n={n} row={i}")


def test_support_far_threshold_falls_back(cuda_device):
    # every |x| is at least 62.5 (> 50): the row is recomputed by the dense kernels
    n = 6000
    r = np.random.default_rng(4).permutation(n).astype(np.float32)[None, :]
    v = np.random.default_rng(5).standard_normal((1, n)).astype(np.float32)
    out = run_gpu(r, 17.0, 0.008, path="radix", v=v, support=True)
    check_row(r[0], v[0], 17.0, 0.008, out["b"][0], out["p"][0], out["g"][0], label="far")


def test_support_matches_plain_backward_and_is_deterministic(cuda_device):
    B, n = 2, 1 << 17
    r, v = random_rows(77, B, n)
    rt = torch.from_numpy(r).cuda()
    vt = torch.from_numpy(v).cuda()
    sup = L.Support(B, n)
    p1, b1 = L.forward(rt, 300.0, 0.002, support=sup)
    p0, b0 = L.forward(rt, 300.0, 0.002)
    assert torch.equal(p0, p1) and torch.equal(b0, b1)
    g_plain = L.backward(rt, b0, vt, 0.002)
    g1 = L.backward(rt, b1, vt, 0.002, support=sup)
    g2 = L.backward(rt, b1, vt, 0.002, support=sup)
    assert torch.equal(g1, g2)
    scale = g_plain.abs().max().item()
    assert (g1 - g_plain).abs().max().item() <= 1e-5 * scale
    for i in range(B):
        check_row(r[i], v[i], 300.0, 0.002, b1[i].item(), p1[i].cpu().numpy().astype(np.float64),
                  g1[i].cpu().numpy().astype(np.float64), label=f"row {i}")


def test_support_from_another_forward_is_not_trusted(cuda_device):
    # the list was written for other scores (another b): the backward notices
    # the mismatch and recomputes the rows densely, so g is still right
    B, n = 2, 50000
    r, v = random_rows(81, B, n)
    r_other, _ = random_rows(82, B, n)
    sup = L.Support(B, n)
    L.forward(torch.from_numpy(r_other).cuda(), 40.0, 0.01, support=sup)
    rt = torch.from_numpy(r).cuda()
    p, b = L.forward(rt, 40.0, 0.01)
    g = L.backward(rt, b, torch.from_numpy(v).cuda(), 0.01, support=sup)
    for i in range(B):
        check_row(r[i], v[i], 40.0, 0.01, b[i].item(), p[i].cpu().numpy().astype(np.float64),
                  g[i].cpu().numpy().astype(np.float64), label=f"stale list row {i}")


def test_support_strided_rows(cuda_device):
    # ld > n and an unaligned base: the scalar paths of the emit and write kernels
    B, n, ld = 3, 9000, 9011
    r, v = random_rows(12, B, ld)
    full = torch.from_numpy(r).cuda()
    vv = torch.from_numpy(v).cuda()
    sub = full[:, 1:1 + n]
    sup = L.Support(B, n)
    p, b = L.forward(sub, 30.0, 0.02, path="radix", support=sup)
    g = L.backward(sub, b, vv[:, 1:1 + n], 0.02, support=sup)
    for i in range(B):
        check_row(r[i, 1:1 + n], v[i, 1:1 + n], 30.0, 0.02, b[i].item(),
                  p[i].cpu().numpy().astype(np.float64), g[i].cpu().numpy().astype(np.float64),
                  label=f"strided support row={i}")


def test_autograd_long_rows_use_support(cuda_device):
    r, v = random_rows(14, 2, 30000)
    rt = torch.from_numpy(r).cuda().requires_grad_(True)
    p = L.soft_topk(rt, 25.0, 0.01)
    p.backward(torch.from_numpy(v).cuda())
    _, b = L.forward(rt.detach(), 25.0, 0.01)
    g = L.backward(rt.detach(), b, torch.from_numpy(v).cuda(), 0.01)
    scale = g.abs().max().item()
    assert (rt.grad - g).abs().max().item() <= 1e-5 * scale



def test_rowbracket_forced_miss_widens(cuda_device):
    # every row starts from a bracket above all its samples and is widened
    B, n = 4, 30000
    r, v = random_rows(93, B, n, "mix_nu")
    ws = L.Workspace(B, n, 50.0, "rowbracket")
    rt = torch.from_numpy(r).cuda()
    p, b = L.forward(rt, 50.0, 0.01, path=L.PATHS["rowbracket"] | L.FLAG_FORCE_MISS, ws=ws)
    for i in range(B):
        info = L.row_info(ws, i)
        assert info["attempts"] >= 2 and info["path"] == 4
        check_row(r[i], v[i], 50.0, 0.01, b[i].item(), p[i].cpu().numpy().astype(np.float64),
                  label=f"rowbracket forced miss row {i}")


def test_rowbracket_matches_radix(cuda_device):
    B, n = 8, 65536
    r, _ = random_rows(94, B, n, "normal_q64")
    a = run_gpu(r, 1024.0, 0.02, path="rowbracket")
    c = run_gpu(r, 1024.0, 0.02, path="radix")
    for i in range(B):
        assert abs(a["b"][i] - c["b"][i]) <= 1e-6 * max(0.02, abs(c["b"][i]))


# ---------------------------------------------------------------------------
# Gradients with respect to k and t.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("B,n,k,t,dist", [
    (3, 100, 7.0, 0.3, "normal"),
    (2, 5000, 40.0, 0.02, "normal_q64"),
    (1, 70001, 300.0, 0.005, "mix_nu"),
    (2, 1 << 18, 2000.0, 1.0, "normal"),
])
def test_backward_kt_matches_oracle(cuda_device, B, n, k, t, dist):
    r, v = random_rows(71 + n, B, n, dist)
    rt = torch.from_numpy(r).cuda()
    vt = torch.from_numpy(v).cuda()
    _, b = L.forward(rt, k, t)
    gk, gt = L.backward_kt(rt, b, vt, t)
    gk, gt, bb = gk.cpu().numpy(), gt.cpu().numpy(), b.cpu().numpy()
    for i in range(B):
        b_ref = oracle.solve_b(r[i], k, t)
        assert abs(bb[i] - b_ref) <= 1e-5 * max(t, abs(b_ref))
        rk, rt_ = oracle.vjp_kt(r[i], v[i], b_ref, t)
        assert abs(gk[i] - rk) <= 1e-4 * max(1.0, abs(rk)), (i, gk[i], rk)
        assert abs(gt[i] - rt_) <= 1e-4 * max(abs(rt_), 1e-3 * abs(rk) / t), (i, gt[i], rt_)


def test_autograd_learnable_k_and_t(cuda_device):
    B, n = 4, 3000
    r, v = random_rows(72, B, n)
    rt = torch.from_numpy(r).cuda().requires_grad_(True)
    k = torch.tensor(25.0, dtype=torch.float64, device="cuda", requires_grad=True)
    t = torch.tensor(0.05, dtype=torch.float64, device="cuda", requires_grad=True)
    p = L.soft_topk(rt, k, t)
    p.backward(torch.from_numpy(v).cuda())
    gk_ref = gt_ref = 0.0
    for i in range(B):
        b_ref = oracle.solve_b(r[i], 25.0, 0.05)
        a, c = oracle.vjp_kt(r[i], v[i], b_ref, 0.05)
        gk_ref += a
        gt_ref += c
    assert abs(k.grad.item() - gk_ref) <= 1e-4 * max(1.0, abs(gk_ref))
    assert abs(t.grad.item() - gt_ref) <= 1e-4 * max(1.0, abs(gt_ref))
    assert rt.grad is not None and torch.isfinite(rt.grad).all()
