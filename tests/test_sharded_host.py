"""Host logic of one row split over several devices, on CPU with two and three gloo ranks.

The split-row path ("Fast LapSum: Exact Differentiable Top-k at Million
Scale", gist.science explainer pages, section 2.2, with the row in shards)
exchanges the sample, the fold's tails and band, and the backward's shifted
sums between processes, then repeats the same decisions on every process.
Here the per-shard steps run on the CPU (the oracle's sample and fold, numpy
for the band solve and the VJP sums) so that the orchestration --
sample assembly by a sum, gathers in process order, padded band exchange,
certification and widening, the merged backward -- is tested without a GPU;
the result must match the oracle on the whole row.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class CpuShardOps:
    """CPU stand-ins of the per-shard GPU steps (fp64)."""

    def __init__(self, full_row, force_first_miss=False):
        self.full = full_row
        self.force = force_first_miss
        self.calls = 0

    def sample(self, r, offset, n, t, seed, m):
        import oracle
        y, idx = oracle.sample(self.full, t, seed, 0, m)
        own = (idx >= offset) & (idx < offset + r.numel())
        return torch.tensor(np.where(own, y, 0.0), dtype=torch.float64)

    def bracket(self, y, m, rank_l, rank_h):
        import oracle
        aL, aR = oracle.bracket_from_sample(y.numpy(), rank_l, rank_h if rank_h >= 1 else m + 1)
        self.calls += 1
        if self.force and self.calls == 1:
            aL, aR = float(y.max()) + abs(float(y.max())) + 1.0, float("inf")
        return torch.tensor([aL, aR], dtype=torch.float64)

    def fold(self, r, ends, t):
        import oracle
        x = r.numpy()
        aL, aR = float(ends[0]), float(ends[1])
        f = oracle.fold(x, aL, aR, t)
        band = x[(x >= aL) & (x < aR)]
        rec = torch.tensor([f["cnt_R"], f["S_L"], f["S_R"], 0.0, band.size], dtype=torch.float64)
        out = np.zeros(max(1, x.size))
        out[:band.size] = band
        return rec, torch.tensor(out)

    def band_solve(self, bands, stride, recs, world, ends, k, t):
        recs = recs.numpy()
        aL, aR = float(ends[0]), float(ends[1])
        cr, sl, sr = recs[:, 0].sum(), recs[:, 1].sum(), recs[:, 2].sum()
        band = np.concatenate([bands[w, :int(recs[w, 4])].numpy() for w in range(world)])

        def F(b):
            v = cr + np.sum(np.where(band >= b, 1 - 0.5 * np.exp(-(band - b) / t),
                                     0.5 * np.exp((band - b) / t)))
            if np.isfinite(aR):
                v -= 0.5 * sr * np.exp((b - aR) / t)
            if np.isfinite(aL):
                v += 0.5 * sl * np.exp((aL - b) / t)
            return v

        FL = F(aL) if np.isfinite(aL) else np.inf
        FR = F(aR) if np.isfinite(aR) else -np.inf
        if not (FL >= k >= FR):
            return torch.tensor([np.nan, FL, FR, 0.0])
        lo = aL if np.isfinite(aL) else band.min() - 200 * t
        hi = aR if np.isfinite(aR) else band.max() + 200 * t
        for _ in range(200):
            mid = 0.5 * (lo + hi)
            if mid in (lo, hi):
                break
            lo, hi = (mid, hi) if F(mid) >= k else (lo, mid)
        return torch.tensor([lo, FL, FR, 1.0])

    def emit(self, r, b, t):
        import oracle
        return torch.tensor(oracle.emit_p(r.numpy(), float(b[0]), t))

    def vjp_partial(self, r, v, b, t):
        x = np.abs(r.numpy() - float(b[0])) / t
        mu = x.min()
        w = np.exp(-(x - mu))
        return torch.tensor([mu, w.sum(), (w * v.numpy()).sum()])

    def vjp_apply(self, r, v, b, t, recs, world):
        recs = recs.numpy()
        mrow = recs[:, 0].min()
        f = np.exp(mrow - recs[:, 0])
        R = (recs[:, 2] * f).sum() / (recs[:, 1] * f).sum()
        fx = 0.5 * np.exp(-np.abs(r.numpy() - float(b[0])) / t)
        return torch.tensor(fx / t * (v.numpy() - R))


def _rank_main(rank, world, port, cuts, force, out):
    import torch.distributed as dist
    from sparse_selection_primitive_b200 import sharded
    from workloads import random_rows
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, v = random_rows(77, 1, cuts[-1], "mix_nu")
        full = r[0].astype(np.float64)
        lo, hi = cuts[rank], cuts[rank + 1]
        ops = CpuShardOps(full, force_first_miss=force)
        comm = sharded.DistComm()
        k, t = 40.0, 0.02
        rs = torch.tensor(full[lo:hi])
        p, b, attempts = sharded.forward(rs, k, t, cuts[-1], lo, comm, ops=ops, seed=3)
        g = sharded.backward(rs, torch.tensor(v[0, lo:hi].astype(np.float64)), b, t, comm,
                             ops=ops)
        out[rank] = (float(b[0]), attempts, p.numpy(), g.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,force", [(2, False), (2, True), (3, False)])
def test_gloo_ranks_split_one_row(world, force):
    import oracle
    from workloads import random_rows
    n = 30000
    cuts = {2: [0, 11111, n], 3: [0, 7001, 19999, n]}[world]  # unequal shards
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, cuts, force, out), nprocs=world, join=True,
                       start_method="spawn")
    res = [out[i] for i in range(world)]
    # every rank takes the same decisions and finds the same b
    assert all(x[0] == res[0][0] and x[1] == res[0][1] for x in res)
    b0, att0 = res[0][0], res[0][1]
    assert att0 >= (2 if force else 1)
    r, v = random_rows(77, 1, n, "mix_nu")
    row = r[0].astype(np.float64)
    b_ref = oracle.solve_b(row, 40.0, 0.02)
    assert abs(b0 - b_ref) <= 1e-10 * max(0.02, abs(b_ref))
    p = np.concatenate([x[2] for x in res])
    assert np.max(np.abs(p - oracle.emit_p(row, b_ref, 0.02))) <= 1e-8
    g = np.concatenate([x[3] for x in res])
    g_ref, _, _ = oracle.vjp(row, v[0], b_ref, 0.02)
    assert np.max(np.abs(g - g_ref)) <= 1e-7 * np.max(np.abs(g_ref))
