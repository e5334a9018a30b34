"""GPU parity of one row split over several devices (the lapsum_shard_* pieces).

"Fast LapSum: Exact Differentiable Top-k at Million Scale" (gist.science
explainer pages), section 2.2, with the row in contiguous shards: the shards'
sample draws, folds, band solve, emit and VJP pieces run in the library's
kernels, and the host moves the small results between them.  b, p and g must
match the oracle on the whole row at the parity tolerances.

* one process holding the whole row (no exchange);
* a first bracket forced to miss, so the band solve reports it uncertified and
  the host widens it;
* two processes on this GPU exchanging through gloo (their kernels never wait
  on one another; the exchange is on the host).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import sparse_selection_primitive_b200 as L
from sparse_selection_primitive_b200 import sharded
from tests.gpu_helpers import check_row
from workloads import random_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,k,t,dist", [(300000, 250.0, 0.01, "mix_nu"),
                                        (1_000_003, 600.0, 0.01, "abs_t3"),
                                        (200000, 20000.0, 0.05, "normal")])
def test_single_shard_matches_oracle(cuda_device, n, k, t, dist):
    r, v = random_rows(880 + n % 97, 1, n, dist)
    rt = torch.from_numpy(r[0]).cuda()
    p, b, attempts = sharded.forward(rt, k, t, n, 0, sharded.LocalComm(), seed=5)
    g = sharded.backward(rt, torch.from_numpy(v[0]).cuda(), b, t, sharded.LocalComm())
    torch.cuda.synchronize()
    check_row(r[0], v[0], k, t, b.item(), p.cpu().numpy().astype(np.float64),
              g.cpu().numpy().astype(np.float64), label=f"{dist} n={n}")
    # the same sample and bracket as the single-device bracketing
    _, b1 = L.forward(rt, k, t, path="bracket", seed=5)
    assert abs(b1.item() - b.item()) <= 1e-5 * max(t, abs(b.item()))


class _MissFirst(sharded.GpuShardOps):
    """Starts from a bracket above every sample value."""

    def __init__(self, *a, **kw):
        super().__init__(*a, **kw)
        self.calls = 0

    def bracket(self, y, m, rank_l, rank_h):
        ends = super().bracket(y, m, rank_l, rank_h)
        self.calls += 1
        if self.calls == 1:
            top = float(y.max())
            ends = torch.tensor([top + abs(top) + 1.0, float("inf")], dtype=torch.float32,
                                device=y.device)
        return ends


def test_single_shard_widens_a_missed_bracket(cuda_device):
    n, k, t = 250000, 300.0, 0.02
    r, v = random_rows(891, 1, n, "normal")
    rt = torch.from_numpy(r[0]).cuda()
    ops = _MissFirst(n, rt.device)
    p, b, attempts = sharded.forward(rt, k, t, n, 0, sharded.LocalComm(), ops=ops)
    torch.cuda.synchronize()
    assert attempts >= 2
    check_row(r[0], None, k, t, b.item(), p.cpu().numpy().astype(np.float64), label="widened")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, cuts, k, t, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        r, v = random_rows(893, 1, cuts[-1], "mix_nu")
        lo, hi = cuts[rank], cuts[rank + 1]
        rs = torch.from_numpy(r[0, lo:hi].copy()).cuda()
        vs = torch.from_numpy(v[0, lo:hi].copy()).cuda()
        comm = sharded.DistComm()
        p, b, attempts = sharded.forward(rs, k, t, cuts[-1], lo, comm, seed=7)
        g = sharded.backward(rs, vs, b, t, comm)
        torch.cuda.synchronize()
        out[rank] = (b.item(), attempts, p.cpu().numpy(), g.cpu().numpy())
    finally:
        dist.destroy_process_group()


def test_two_processes_split_one_row(cuda_device):
    n, k, t = 1_200_001, 900.0, 0.005
    cuts = [0, 700_003, n]
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(2, port, cuts, k, t, out), nprocs=2, join=True,
                       start_method="spawn")
    b0, a0, p0, g0 = out[0]
    b1, a1, p1, g1 = out[1]
    assert b0 == b1 and a0 == a1
    r, v = random_rows(893, 1, n, "mix_nu")
    check_row(r[0], v[0], k, t, b0, np.concatenate([p0, p1]).astype(np.float64),
              np.concatenate([g0, g1]).astype(np.float64), label="two shards")
