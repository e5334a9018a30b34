"""GPU parity at the five benchmark workloads' full sizes, in the launch
configuration the benchmark times (AUTO path, one call over all rows).

* single row n=1024 and the MoE batch: oracle on every row (C1) or on a
  seeded sample of rows plus the first and last (16384 x 256);
* memory-selection batch 256 x 65536: every row's b against the stored oracle
  thresholds, p and g on a sample of rows, with the AUTO solver and with the
  full-sort (radix) solver the configuration names;
* the two bracketing rows (n = 3,342,336 and 10^8): b against the stored
  oracle threshold and, independently, against the oracle's sign function at
  b +- tolerance; p and g on every element; the bracketing b also against
  the GPU full-sort (radix) b.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import sparse_selection_primitive_b200 as L
from tests.gpu_helpers import TOL_B, check_row, run_gpu
from workloads import WORKLOADS, input_digest, make_inputs

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "thresholds.json")


def stored(name):
    with open(GOLDEN) as f:
        return json.load(f)[name]


def test_single_row_n1024(cuda_device):
    w = WORKLOADS["single_row_n1024"]
    r, v = make_inputs(w)
    out = run_gpu(r, w.k, w.t, v=v)
    check_row(r[0], v[0], w.k, w.t, out["b"][0], out["p"][0], out["g"][0], label=w.name)


def test_moe_router_batch(cuda_device):
    w = WORKLOADS["moe_router_16384x256"]
    r, v = make_inputs(w)
    out = run_gpu(r, w.k, w.t, v=v)
    rows = sorted(set(np.random.default_rng(1).choice(w.B, 256, replace=False).tolist())
                  | {0, w.B - 1})
    for i in rows:
        check_row(r[i], v[i], w.k, w.t, out["b"][i], out["p"][i], out["g"][i],
                  label=f"{w.name} row {i}")
    # every row: budget and range (property valid at any size)
    sums = out["p"].sum(axis=1)
    assert np.max(np.abs(sums - w.k)) <= 1e-3
    assert out["p"].min() >= 0.0 and out["p"].max() <= 1.0
    assert np.all(np.abs(out["g"].sum(axis=1)) <= 1e-4 * np.abs(out["g"]).max(axis=1) * 16)


def test_memory_select_batch(cuda_device):
    w = WORKLOADS["memory_select_256x65536"]
    ref = stored(w.name)
    r, v = make_inputs(w)
    assert input_digest(r) == ref["digest_r"] and input_digest(v) == ref["digest_v"]
    out = run_gpu(r, w.k, w.t, v=v)
    b_ref = np.array(ref["b"])
    err = np.abs(out["b"] - b_ref) / np.maximum(w.t, np.abs(b_ref))
    assert err.max() <= TOL_B, err.max()
    for i in [0, 17, 128, 255]:
        check_row(r[i], v[i], w.k, w.t, out["b"][i], out["p"][i], out["g"][i], b_ref=b_ref[i],
                  label=f"{w.name} row {i}")
    assert np.max(np.abs(out["p"].sum(axis=1) - w.k)) <= 1e-3


def test_memory_select_batch_full_sort(cuda_device):
    # The configuration as it is written: the full-sort solver (radix sort of
    # every row) on the whole 256 x 65536 batch, forward and gradient-support
    # backward as the benchmark runs them; every row's b against the stored
    # oracle thresholds, p and g element by element on a sample of rows.
    w = WORKLOADS["memory_select_256x65536"]
    ref = stored(w.name)
    r, v = make_inputs(w)
    out = run_gpu(r, w.k, w.t, path="fullsort", v=v, support=True)
    b_ref = np.array(ref["b"])
    err = np.abs(out["b"] - b_ref) / np.maximum(w.t, np.abs(b_ref))
    assert err.max() <= TOL_B, err.max()
    for i in [0, 1, 100, 200, 255]:
        check_row(r[i], v[i], w.k, w.t, out["b"][i], out["p"][i], out["g"][i], b_ref=b_ref[i],
                  label=f"{w.name} full sort row {i}")
    assert np.max(np.abs(out["p"].sum(axis=1) - w.k)) <= 1e-3
    assert out["p"].min() >= 0.0 and out["p"].max() <= 1.0


def _bracket_row(name, cuda_device):
    w = WORKLOADS[name]
    ref = stored(name)
    r, v = make_inputs(w)
    assert input_digest(r) == ref["digest_r"] and input_digest(v) == ref["digest_v"]
    b_ref = ref["b"][0]
    ws = L.Workspace(1, w.n, w.k, "auto")
    out = run_gpu(r, w.k, w.t, v=v, ws=ws)
    info = L.row_info(ws, 0)
    assert info["path"] == 2 and info["attempts"] >= 1
    assert L.read_status(ws) == 0
    b = out["b"][0]
    tol = TOL_B * max(w.t, abs(b_ref))
    # independent of the stored value: the oracle's exact sign brackets the GPU b
    assert oracle.budget_sign(r[0], b - tol, w.k, w.t) >= 0
    assert oracle.budget_sign(r[0], b + tol, w.k, w.t) <= 0
    check_row(r[0], v[0], w.k, w.t, b, out["p"][0], out["g"][0], b_ref=b_ref, label=name)
    return r, w, b, info


def test_adv_mask_row(cuda_device):
    _bracket_row("adv_mask_3342336", cuda_device)


def test_extreme_row_and_full_sort_cross_check(cuda_device):
    r, w, b, info = _bracket_row("extreme_1e8", cuda_device)
    out = run_gpu(r, w.k, w.t, path="radix")
    b_sort = out["b"][0]
    assert abs(b_sort - b) <= TOL_B * max(w.t, abs(b)), (b_sort, b)
