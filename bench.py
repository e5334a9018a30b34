#!/usr/bin/env python
"""Benchmark of the Fast LapSum soft top-k (forward + backward) on B200.

One step = one forward (exact threshold b and p) plus one backward (VJP g)
over one batch of synthetic scores, through the library's C ABI.  The default
workload is the 10^8-score row (k = 1e5, t = 0.005, 50/50 N(0,1)/U(-4,4)
scores) that the headline metric is quoted on.

Usage:
    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--no-table] [--no-cpu-baseline]
    torchrun --nproc-per-node N bench.py --gpus N ...   (one rank per GPU)

With N ranks every rank solves its own independent workload instance (seed =
rank): the path shards by problem, no collective touches the data path, and
the reported value is the elements of all ranks per max-over-ranks time
(weak scaling).  Rank 0 prints one JSON line.

`--impl reference` times the fp64 CPU oracle (the reference for this method)
on a bounded prefix of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import shutil
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import ORDER, WORKLOADS, make_inputs  # noqa: E402

METRIC = "soft top-k elements/s fwd+bwd"
UNIT = "elements/s"

# Algorithmic bytes per element of each kernel (what the kernel must move:
# reads of its inputs and writes of its outputs, once).
KERNEL_BYTES_PER_ELEMENT = {
    "onchip_fwd": 8,      # read r, write p
    "onchip_search": 8,   # read r, write p
    "onchip_bwd": 12,     # read r, v, write g
    "emit": 8,            # read r, write p
    "bwd_reduce": 8,      # read r, v
    "bwd_apply": 12,      # read r, v, write g
    "bracket_fold": 4,    # read r
    "sup_write": 4,       # write g (plus the support list, counted per entry elsewhere)
    "window_pass": 4,     # read r (v only inside the window)
    "window_write": 4,    # write g
    "radix_prep": 8,      # read r, write keys
    "radix_upsweep": 4,   # read keys (per pass)
    "radix_downsweep": 8,  # read keys, write keys (per pass)
    "rowsolve": 4,        # read sorted keys
}
# Algorithmic bytes per element of one fwd+bwd step, per solver: on-chip rows
# move r, p, r, v, g once (20 B); the long-row paths read r twice in the
# forward and r, v twice in the backward (32 B).
STEP_BYTES_PER_ELEMENT = {"onchip": 20, "radix": 20, "bracket": 32}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# Ranks: one process per GPU, each solving its own workload instance
# ---------------------------------------------------------------------------
def rank_env():
    """(world, rank, local_rank) from the launcher's environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest x over all ranks (every rank gets it); x itself when alone."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    tt = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def job_value(elements_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: the elements of every rank over the slowest rank's time."""
    return elements_per_rank * world / (ms_max / 1e3)


# ---------------------------------------------------------------------------
# nvidia-smi clock sampling during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.out = None

    def start(self):
        exe = shutil.which("nvidia-smi")
        if exe is None:
            return
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = subprocess.Popen(
            [exe, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
             "-i", str(self.gpu_index)], stdout=self.out, stderr=subprocess.DEVNULL)
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [ln.strip().split(",") for ln in self.out.read().splitlines() if ln.strip()]
        os.unlink(self.out.name)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for row in rows:
            try:
                sm.append(float(row[1]))
                mx = max(mx, float(row[2]))
                for nm, val in zip(names, row[5:9]):
                    if val.strip().lower() == "active":
                        reasons.add(nm)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle leg (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------
def oracle_sample_run(w, r_row, v_row, n_sample):
    """Oracle fwd+bwd on the first n_sample scores of one row (k scaled to keep k/n)."""
    import oracle
    n_s = min(n_sample, r_row.size)
    k_s = w.k * n_s / w.n if n_s < w.n else w.k
    k_s = min(max(k_s, 1e-3), n_s - 1e-3)
    t0 = time.perf_counter()
    b = oracle.solve_b(r_row[:n_s], k_s, w.t)
    oracle.emit_p(r_row[:n_s], b, w.t)
    oracle.vjp(r_row[:n_s], v_row[:n_s], b, w.t)
    return n_s, k_s, time.perf_counter() - t0


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_timings(w, r, v, budget=1 << 20):
    """The fp64 oracle, single-threaded, on a bounded sample of a workload: whole
    rows up to about `budget` scores for batched shapes, else a prefix of row 0
    (k scaled to keep k/n).  Forward (solve b, emit p), backward (VJP) and both,
    in elements per second, with the host's CPU model and core count."""
    import oracle
    if w.n <= budget:
        rows = max(1, min(w.B, budget // w.n))
        n_s, k_s = w.n, w.k
    else:
        rows, n_s = 1, budget
        k_s = min(max(w.k * n_s / w.n, 1e-3), n_s - 1e-3)
    tf = tb = 0.0
    for i in range(rows):
        rr, vv = r[i, :n_s], v[i, :n_s]
        t0 = time.perf_counter()
        b = oracle.solve_b(rr, k_s, w.t)
        oracle.emit_p(rr, b, w.t)
        t1 = time.perf_counter()
        oracle.vjp(rr, vv, b, w.t)
        t2 = time.perf_counter()
        tf += t1 - t0
        tb += t2 - t1
    el = rows * n_s
    return {"fwd_elements_per_s": el / tf, "bwd_elements_per_s": el / tb,
            "fwdbwd_elements_per_s": el / (tf + tb), "cores": 1, "cpu": cpu_model(),
            "host_cpu_count": os.cpu_count(),
            "sample": (f"{rows} whole rows" if n_s == w.n else
                       f"first {n_s} scores of row 0, k={k_s:g} (same k/n)")}


def cpu_sample_size(w):
    # about 10 s of single-thread oracle work on this machine's cores
    return min(w.elements, 1 << 23)


def cpu_baseline(w, r, v):
    n_s, k_s, sec = oracle_sample_run(w, r[0], v[0], cpu_sample_size(w))
    return {"value": n_s / sec, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"first {n_s} scores of row 0 of {w.name}, k={k_s:g} (same k/n), "
                      f"t={w.t}; fp64 full sort + bisection, p, VJP; {sec:.1f} s single thread",
            "cpu": cpu_model(), "host_cpu_count": os.cpu_count()}


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    r, v = make_inputs(w, seed=0)
    n_s = min(cpu_sample_size(w), w.n)
    # warm-up steps on a tiny prefix, then K timed steps on the bounded sample
    for _ in range(args.warmup):
        oracle_sample_run(w, r[0], v[0], min(4096, w.n))
    n_step = max(1 << 16, n_s // max(1, args.steps))
    times = []
    for _ in range(args.steps):
        n_done, k_s, sec = oracle_sample_run(w, r[0], v[0], n_step)
        times.append(sec)
    ms = 1e3 * statistics.mean(times)
    value = n_done / (ms / 1e3)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "n": w.n, "k": w.k, "t": w.t,
                   "step_sample": f"first {n_done} scores of row 0 (k scaled to {k_s:g})"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"{args.steps} steps, each the first {n_done} scores of row 0"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU leg
# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="extreme_1e8", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-table", action="store_true", help="skip the per-workload table")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--n-override", type=int, default=0,
                    help="profiling runs: shrink the workload's row length (k scaled to keep k/n)")
    ap.add_argument("--path", default="auto", choices=["auto", "fullsort", "radix", "bracket", "rowbracket"],
                    help="solver of the timed workload (default: the library's choice)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world, rank, local = rank_env()

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    import sparse_selection_primitive_b200 as L

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    L._build.build()
    w = WORKLOADS[args.workload]
    if args.n_override:
        from dataclasses import replace
        w = replace(w, n=args.n_override, k=max(1.0, round(w.k * args.n_override / w.n)),
                    name=f"{w.name}@n={args.n_override}")
    r_h, v_h = make_inputs(w, seed=rank)
    stream = torch.cuda.current_stream(dev)

    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.empty(2 * l2_bytes // 4 + 1024, dtype=torch.float32, device=dev)

    def run_workload(w, r_h, v_h, steps, warmup, table=False, k_rows=None, path="auto"):
        rd = torch.from_numpy(r_h).to(dev)
        vd = torch.from_numpy(v_h).to(dev)
        pd = torch.empty_like(rd)
        gd = torch.empty_like(rd)
        bd = torch.empty(w.B, dtype=torch.float64, device=dev)
        # one budget per row (lapsum_forward_rowk) when k_rows is given
        kk = w.k if k_rows is None else torch.from_numpy(k_rows).to(dev)
        ws = (L.Workspace(w.B, w.n, w.k, path, dev) if k_rows is None else
              L.Workspace(w.B, w.n, 1.0, path, dev,
                          nbytes=L._lib().lapsum_workspace_bytes_rowk(w.B, w.n, 0)))
        # rows longer than 4096 hand the gradient support from forward to
        # backward, as the autograd wrapper does
        sup = L.Support(w.B, w.n, dev) if L.support_bytes(w.B, w.n) > 0 else None
        working = 4 * rd.numel() * 4
        flush = working < 2 * l2_bytes

        def fwd():
            L.forward(rd, kk, w.t, path=path, ws=ws, p=pd, b=bd, support=sup)

        def bwd():
            L.backward(rd, bd, vd, w.t, ws=ws, g=gd, support=sup)

        def bwd_plain():
            L.backward(rd, bd, vd, w.t, ws=ws, g=gd)

        def timed(fn, k_steps, profile=False):
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(k_steps)]
            torch.cuda.synchronize(dev)
            if profile:
                L.profile_enable(True)
            for s, e in evs:
                if flush:
                    flush_buf.zero_()
                s.record(stream)
                fn()
                e.record(stream)
            torch.cuda.synchronize(dev)
            prof = L.profile_read() if profile else None
            if profile:
                L.profile_enable(False)
            return [s.elapsed_time(e) for s, e in evs], prof

        for _ in range(warmup):
            fwd()
            bwd()
        torch.cuda.synchronize(dev)
        # the same step captured once into a CUDA graph (the library's calls are
        # stream-ordered and allocate nothing, so they capture as they are)
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fwd()
            bwd()
        stream.wait_stream(side)
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(graph):
            fwd()
            bwd()
        torch.cuda.synchronize(dev)
        res = {"flush": flush, "ws": ws, "rd": rd, "vd": vd, "pd": pd, "gd": gd, "bd": bd,
               "fwd": fwd, "bwd": bwd, "timed": timed, "graph": graph, "sup": sup}
        res["near"] = support_count(r_h, bd.cpu().numpy(), w.t) if sup is not None else 0
        if w.path == "bracket" and path == "auto":
            info = L.row_info(ws, 0)
            res["bracket"] = {key: info[key] for key in ("attempts", "n_band", "refine_levels",
                                                       "sample_m", "rank_l", "rank_h")}
        if table:
            tf, _ = timed(fwd, steps)
            tb, _ = timed(bwd, steps)
            tfb, _ = timed(lambda: (fwd(), bwd()), steps)
            tg, _ = timed(graph.replay, steps)
            res["table"] = {"fwd_ms": statistics.median(tf), "bwd_ms": statistics.median(tb),
                            "fwdbwd_ms": statistics.median(tfb),
                            "fwdbwd_graph_ms": statistics.median(tg)}
            if sup is not None:
                tp, _ = timed(bwd_plain, steps)
                res["table"]["bwd_without_support_ms"] = statistics.median(tp)
        return res

    def hard_row(wk, peak_gbs):
        """The zero-temperature limit (lapsum_forward_hard) on a workload's scores:
        the on-chip sort for short rows, the bracketed selection for long ones
        (plain samples, one counting pass, the boundary group from the band)."""
        rr, _ = make_inputs(wk, seed=0)
        rd = torch.from_numpy(rr).to(dev)
        ws = L.Workspace(wk.B, wk.n, wk.k, "fullsort", dev)
        for _ in range(3):
            L.hard_topk(rd, wk.k, ws=ws)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            L.hard_topk(rd, wk.k, ws=ws)
        stream.wait_stream(side)
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(graph):
            L.hard_topk(rd, wk.k, ws=ws)
        torch.cuda.synchronize(dev)
        times = []
        for _ in range(10):
            flush_buf.zero_()
            s_ev = torch.cuda.Event(enable_timing=True)
            e_ev = torch.cuda.Event(enable_timing=True)
            s_ev.record(stream)
            graph.replay()
            e_ev.record(stream)
            torch.cuda.synchronize(dev)
            times.append(s_ev.elapsed_time(e_ev))
        ms = statistics.median(times)
        del graph
        return {"mode": "zero-temperature limit (forward only)",
                "solver": "on-chip sort" if wk.n <= 4096 else "bracketed selection",
                "fwd_graph_ms": round(ms, 5), "fwd_elements_per_s": wk.elements / (ms / 1e3),
                # r read by the counting pass, r read and p written by the emit
                "path_frac_of_peak": (8 if wk.n <= 4096 else 12) * wk.elements
                / (ms / 1e3) / 1e9 / peak_gbs}

    def router_bf16_row(peak_gbs):
        """The router shape through the router form: bf16 scores, p and the list of
        p > 1e-3 (at most 16 per row) in the forward, g from bf16 scores."""
        wk = WORKLOADS["moe_router_16384x256"]
        rr, vv = make_inputs(wk, seed=0)
        rd = torch.from_numpy(rr).to(dev).to(torch.bfloat16)
        vd = torch.from_numpy(vv).to(dev)
        ws = L.Workspace(wk.B, wk.n, wk.k, "fullsort", dev)
        outs = (torch.empty((wk.B, wk.n), device=dev),
                torch.empty(wk.B, dtype=torch.float64, device=dev),
                torch.empty((wk.B, 16), dtype=torch.int32, device=dev),
                torch.empty((wk.B, 16), device=dev), torch.empty(wk.B, dtype=torch.int32, device=dev))
        gd = torch.empty((wk.B, wk.n), device=dev)

        def fwd():
            L.forward_router(rd, wk.k, wk.t, eps=1e-3, cap=16, ws=ws, out=outs)

        def bwd():
            L.backward_router(rd, outs[1], vd, wk.t, g=gd)

        for _ in range(3):
            fwd()
            bwd()
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fwd()
            bwd()
        stream.wait_stream(side)
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(graph):
            fwd()
            bwd()
        torch.cuda.synchronize(dev)
        times = []
        for _ in range(10):
            flush_buf.zero_()
            s_ev = torch.cuda.Event(enable_timing=True)
            e_ev = torch.cuda.Event(enable_timing=True)
            s_ev.record(stream)
            graph.replay()
            e_ev.record(stream)
            torch.cuda.synchronize(dev)
            times.append(s_ev.elapsed_time(e_ev))
        ms = statistics.median(times)
        # bytes: r (2 B) and p (4 B) in the forward, r (2 B), v and g (4 B each) in the
        # backward, plus the list (16 x 8 B per row)
        nbytes = wk.elements * (2 + 4 + 2 + 4 + 4) + wk.B * 16 * 8
        del graph
        return {"scores": "bf16", "select": "p > 1e-3, at most 16 per row",
                "fwdbwd_graph_ms": round(ms, 5),
                "fwdbwd_graph_elements_per_s": wk.elements / (ms / 1e3),
                "path_frac_of_peak": nbytes / (ms / 1e3) / 1e9 / peak_gbs}

    peak_gbs, peak_kind = load_peaks()
    R = run_workload(w, r_h, v_h, args.steps, args.warmup, path=args.path)
    sampler = ClockSampler(local)
    sampler.start()
    barrier()
    torch.cuda.synchronize(dev)
    # per-kernel device times from an eager (profiled) pass over the same steps
    eager_ms, prof = R["timed"](lambda: (R["fwd"](), R["bwd"]()), args.steps, profile=True)
    barrier()
    torch.cuda.synchronize(dev)
    # the timed region proper: K replays of the captured step
    step_ms, _ = R["timed"](R["graph"].replay, args.steps)
    barrier()
    clocks = sampler.stop()
    ms_local = statistics.mean(step_ms)
    eager_ms_max = max_over_ranks(statistics.mean(eager_ms), world, dev)
    ms = max_over_ranks(ms_local, world, dev)
    elements = w.elements * world
    value = job_value(w.elements, world, ms)

    # dominant kernel of the timed region
    dom_name, (dom_launch, dom_ms) = max(prof.items(), key=lambda kv: kv[1][1])
    per_launch_ms = dom_ms / dom_launch
    bpe = KERNEL_BYTES_PER_ELEMENT.get(dom_name)
    per_launch_elems = w.elements if dom_name not in ("radix_upsweep", "radix_downsweep") else w.elements
    achieved = (bpe * per_launch_elems / (per_launch_ms / 1e3)) / 1e9 if bpe else None
    traffic = read_traffic(dom_name, w.name)
    roofline = {"bound": "hbm", "kernel": dom_name, "achieved": achieved, "peak": peak_gbs,
                "peak_kind": peak_kind, "unit": "GB/s",
                "frac": (achieved / peak_gbs) if achieved else None,
                "traffic": traffic, "algorithmic_bytes_per_launch": (bpe or 0) * per_launch_elems,
                "launch_ms": per_launch_ms}
    step_bytes = STEP_BYTES_PER_ELEMENT[w.path] * w.elements
    step_gbs = step_bytes / (ms_local / 1e3) / 1e9
    path_bytes = path_step_bytes(w, R["near"])
    path_gbs = path_bytes / (ms_local / 1e3) / 1e9
    kernels = {k: {"launches": v[0], "total_ms": round(v[1], 4),
                   "share": round(v[1] / sum(x[1] for x in prof.values()), 4)}
               for k, v in sorted(prof.items(), key=lambda kv: -kv[1][1])}
    gpu_launches = int(sum(v[0] for v in prof.values()))

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        import torch as _t
        r_pin = _t.from_numpy(r_h).pin_memory()
        v_pin = _t.from_numpy(v_h).pin_memory()
        p_pin = _t.empty_like(r_pin).pin_memory()
        g_pin = _t.empty_like(r_pin).pin_memory()

        def e2e_step():
            R["rd"].copy_(r_pin, non_blocking=True)
            R["vd"].copy_(v_pin, non_blocking=True)
            R["fwd"]()
            R["bwd"]()
            p_pin.copy_(R["pd"], non_blocking=True)
            g_pin.copy_(R["gd"], non_blocking=True)

        for _ in range(2):
            e2e_step()
        barrier()
        torch.cuda.synchronize(dev)
        e_s = torch.cuda.Event(enable_timing=True)
        e_e = torch.cuda.Event(enable_timing=True)
        k_e2e = max(3, min(args.steps, 10))
        e_s.record(stream)
        for _ in range(k_e2e):
            e2e_step()
        e_e.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_ms = max_over_ranks(e_s.elapsed_time(e_e) / k_e2e, world, dev)
        nb = r_pin.numel() * 4
        e2e = {"value": elements / (e2e_ms / 1e3), "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": 2 * nb, "d2h_bytes_per_step": 2 * nb}

    # per-workload table (fwd, bwd, fwd+bwd) on this GPU
    table = None
    if not args.no_table and rank == 0:
        table = {}
        for name in ORDER:
            wk = WORKLOADS[name]
            if name == w.name:
                rr, vv = r_h, v_h
            else:
                rr, vv = make_inputs(wk, seed=0)
            RW = run_workload(wk, rr, vv, 10, 3, table=True)
            T = RW["table"]
            table[name] = {
                "fwd_ms": round(T["fwd_ms"], 5), "bwd_ms": round(T["bwd_ms"], 5),
                "fwdbwd_ms": round(T["fwdbwd_ms"], 5),
                "fwdbwd_graph_ms": round(T["fwdbwd_graph_ms"], 5),
                "fwdbwd_graph_elements_per_s": wk.elements / (T["fwdbwd_graph_ms"] / 1e3),
                "fwd_elements_per_s": wk.elements / (T["fwd_ms"] / 1e3),
                "bwd_elements_per_s": wk.elements / (T["bwd_ms"] / 1e3),
                "fwdbwd_elements_per_s": wk.elements / (T["fwdbwd_ms"] / 1e3),
                # the fixed per-score byte count (STEP_BYTES_PER_ELEMENT) over the
                # step time: a reference figure, not bytes this path moves (it can
                # exceed the peak where the path skips passes the count assumes)
                "fwdbwd_fixed_bytes_gbs": STEP_BYTES_PER_ELEMENT[wk.path] * wk.elements
                / (T["fwdbwd_ms"] / 1e3) / 1e9,
            }
            table[name]["oracle"] = oracle_timings(wk, rr, vv)
            if "bwd_without_support_ms" in T:
                table[name]["bwd_without_support_ms"] = round(T["bwd_without_support_ms"], 5)
            table[name]["path_frac_of_peak"] = (path_step_bytes(wk, RW["near"])
                                                / (T["fwdbwd_graph_ms"] / 1e3) / 1e9 / peak_gbs)
            if "bracket" in RW:
                table[name]["bracket"] = RW["bracket"]
            del RW
            torch.cuda.empty_cache()
        # the full-sort solver (radix sort of every row) on the memory-selection
        # shape, as that configuration names it, and on the 10^8-score row, for
        # the bracketed-versus-full-sort comparison
        for name in ("memory_select_256x65536", "extreme_1e8"):
            wk = WORKLOADS[name]
            rr, vv = (r_h, v_h) if name == w.name else make_inputs(wk, seed=0)
            RW = run_workload(wk, rr, vv, 10, 3, table=True, path="fullsort")
            T = RW["table"]
            table[name + "_fullsort"] = {
                "solver": "radix full sort",
                "fwd_ms": round(T["fwd_ms"], 5), "bwd_ms": round(T["bwd_ms"], 5),
                "fwdbwd_ms": round(T["fwdbwd_ms"], 5),
                "fwdbwd_graph_ms": round(T["fwdbwd_graph_ms"], 5),
                "fwdbwd_graph_elements_per_s": wk.elements / (T["fwdbwd_graph_ms"] / 1e3),
                "fwd_elements_per_s": wk.elements / (T["fwd_ms"] / 1e3),
                "bwd_elements_per_s": wk.elements / (T["bwd_ms"] / 1e3),
                # r, p, v, g and the support list only: the sort's key passes
                # come on top of these bytes
                "endpoint_bytes_frac_of_peak": (path_step_bytes(wk, RW["near"])
                                                / (T["fwdbwd_graph_ms"] / 1e3) / 1e9 / peak_gbs),
            }
            del RW
            torch.cuda.empty_cache()
        # the router shape with one budget per row (integers 4..12, seeded)
        wk = WORKLOADS["moe_router_16384x256"]
        rr, vv = make_inputs(wk, seed=0)
        kr = np.random.default_rng(1).integers(4, 13, wk.B).astype(np.float64)
        RW = run_workload(wk, rr, vv, 10, 3, table=True, k_rows=kr)
        T = RW["table"]
        table["moe_router_16384x256_rowk"] = {
            "k_rows": "integers 4..12 (numpy default_rng(1))",
            "fwd_ms": round(T["fwd_ms"], 5), "bwd_ms": round(T["bwd_ms"], 5),
            "fwdbwd_graph_ms": round(T["fwdbwd_graph_ms"], 5),
            "fwdbwd_graph_elements_per_s": wk.elements / (T["fwdbwd_graph_ms"] / 1e3),
            "path_frac_of_peak": (path_step_bytes(wk, 0) / (T["fwdbwd_graph_ms"] / 1e3) / 1e9
                                  / peak_gbs),
        }
        del RW
        torch.cuda.empty_cache()
        # the memory-selection shape with one budget per row (768..1280, seeded):
        # the one-CTA-per-row bracketing with ranks computed per row on the device
        wk = WORKLOADS["memory_select_256x65536"]
        rr, vv = make_inputs(wk, seed=0)
        kr = np.random.default_rng(1).integers(768, 1281, wk.B).astype(np.float64)
        RW = run_workload(wk, rr, vv, 10, 3, table=True, k_rows=kr)
        T = RW["table"]
        table["memory_select_256x65536_rowk"] = {
            "k_rows": "integers 768..1280 (numpy default_rng(1))",
            "fwd_ms": round(T["fwd_ms"], 5), "bwd_ms": round(T["bwd_ms"], 5),
            "fwdbwd_graph_ms": round(T["fwdbwd_graph_ms"], 5),
            "fwdbwd_graph_elements_per_s": wk.elements / (T["fwdbwd_graph_ms"] / 1e3),
            "path_frac_of_peak": (path_step_bytes(wk, RW["near"]) / (T["fwdbwd_graph_ms"] / 1e3)
                                  / 1e9 / peak_gbs),
        }
        del RW
        torch.cuda.empty_cache()
        table["moe_router_16384x256_bf16_select"] = router_bf16_row(peak_gbs)
        torch.cuda.empty_cache()
        for name in ("moe_router_16384x256", "memory_select_256x65536", "extreme_1e8"):
            table[name + "_hard"] = hard_row(WORKLOADS[name], peak_gbs)
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, r_h, v_h)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "n": w.n, "k": w.k, "t": w.t,
                       "distribution": w.dist,
                       "solver": w.path if args.path == "auto" else args.path,
                       "l2": "flushed before each step" if R["flush"] else
                             "inputs larger than L2 (no flush)",
                       "parallelism": f"{world} independent instances (one per GPU)"},
            "bracket": R.get("bracket"),
            "timing": "CUDA-graph replay of one fwd+bwd step; eager calls in eager_ms_per_step",
            "eager_ms_per_step": eager_ms_max,
            "eager_value": elements / (eager_ms_max / 1e3),
            "fixed_bytes_gbs": step_gbs,
            "fixed_bytes_over_peak": step_gbs / peak_gbs,
            "step_bytes_note": "fixed_bytes_* divide a fixed per-score count (fwd 12, bwd 20 "
                               "B/score on long rows: r read twice in the forward, r and v "
                               "read twice and g written in the backward) by the step time: a reference "
                               "figure, not a fraction of bytes moved (this path skips re-reads "
                               "the count assumes, so it can exceed 1); path_* count what this "
                               "path must move: r read by the fold, r read + p written by the "
                               "emit, g written, plus 36 B per gradient-support entry",
            "path_step_bytes": path_bytes,
            "path_support_entries": R["near"],
            "path_frac_of_peak": path_gbs / peak_gbs,
            "roofline": roofline,
            "kernels": kernels,
            "gpu_launches": gpu_launches,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "workloads": table,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def support_count(r_h, b_h, t):
    """Scores with |r - b|/t <= 90 (the gradient support), summed over rows."""
    import numpy as np
    tot = 0
    for i in range(r_h.shape[0]):
        row = r_h[i]
        for s0 in range(0, row.size, 1 << 24):
            x = (row[s0:s0 + (1 << 24)].astype(np.float64) - float(b_h[i])) / t
            tot += int(np.count_nonzero(np.abs(x) <= 90.0))
    return tot


def path_step_bytes(w, near):
    """Bytes one fwd+bwd step of this library's path must move on workload w.

    On-chip rows: r, p, r, v, g once (20 B/score).  Longer rows: r read by the
    solve (radix prep or the bracketing fold; the radix passes are counted as
    measured, not here), r read and p written by the emit, g written by the
    backward, and per gradient-support entry 8 B listed + 8 B read back + 4 B
    v + 4 B kept + 8 + 4 B read by the write pass = 36 B."""
    if w.path == "onchip":
        return 20 * w.elements
    return 16 * w.elements + 36 * near


def read_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu summary."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        for ln in f:
            parts = ln.split()
            if len(parts) >= 3 and not ln.startswith("#") and parts[0] == kernel and \
                    parts[1] == workload:
                try:
                    return float(parts[2])
                except ValueError:
                    return None
    return None


if __name__ == "__main__":
    main()
