"""Host-side logic of bench.py, on CPU.

* The N-rank plumbing: every rank runs its own workload instance and the job
  value is the elements of all ranks over the slowest rank's time.  Two gloo
  ranks (world size 2, CPU) check the max-over-ranks reduction and the value.
* The reference arm (`--impl reference`), which times the fp64 oracle on the
  host: its JSON line, and that under two ranks only rank 0 runs and prints.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, lr = bench.rank_env()
        assert (w, r, lr) == (world, rank, rank)
        # rank-dependent step times: the job is as slow as its slowest rank
        ms_local = 2.0 + 3.0 * rank
        ms = bench.max_over_ranks(ms_local, w, torch.device("cpu"))
        out[rank] = (ms, bench.job_value(1000, w, ms))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    assert set(out.keys()) == {0, 1}
    for rank in range(world):
        ms, value = out[rank]
        assert ms == 5.0
        assert value == pytest.approx(2 * 1000 / 5e-3)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1, None) == 3.5
    assert bench.job_value(10, 1, 2.0) == pytest.approx(5000.0)


def _run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, env=env,
                          capture_output=True, text=True, timeout=600, cwd=ROOT)


def test_reference_arm_prints_one_line():
    res = _run_bench(["--impl", "reference", "--workload", "single_row_n1024", "--steps", "3",
                      "--warmup", "3"])
    assert res.returncode == 0, res.stderr
    lines = [ln for ln in res.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["steps"] == 3 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "single_row_n1024"


def test_reference_arm_other_ranks_exit_quietly():
    res = _run_bench(["--impl", "reference", "--workload", "single_row_n1024", "--steps", "3",
                      "--warmup", "3"], {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"})
    assert res.returncode == 0, res.stderr
    assert res.stdout.strip() == ""
