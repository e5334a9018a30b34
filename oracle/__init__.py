"""Fast LapSum soft top-k: plain fp64 CPU oracle (ctypes wrapper).

TEST INFRASTRUCTURE ONLY.  The test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The CUDA product path
never imports this package, and this package never imports the product.

The arithmetic lives in ``lapsum_oracle.c`` (plain C, fp64, single thread);
this module compiles it with gcc on first use and converts numpy arrays.
Every function cites, in the C file, the passage of "Fast LapSum: Exact
Differentiable Top-k at Million Scale" (gist.science explainer pages) that it
follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lapsum_oracle.c")
_SO = os.path.join(_HERE, "liblapsum_oracle.so")
_LOCK = threading.Lock()
_LIB = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile the oracle into ``liblapsum_oracle.so`` (plain -O2, no fast-math)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _SO)
    return _SO


def configure(lib):
    """Declare the C signatures on a loaded oracle library and return it."""
    lib.lso_abi_version.restype = ctypes.c_int
    lib.lso_laplace_cdf.restype = ctypes.c_double
    lib.lso_laplace_cdf.argtypes = [ctypes.c_double]
    lib.lso_budget_sum.restype = ctypes.c_double
    lib.lso_budget_sum.argtypes = [_dp, ctypes.c_int64, ctypes.c_double, ctypes.c_double]
    lib.lso_budget_sign.restype = ctypes.c_int
    lib.lso_budget_sign.argtypes = [_dp, ctypes.c_int64, ctypes.c_double, ctypes.c_double,
                                    ctypes.c_double]
    lib.lso_solve_b.restype = ctypes.c_int
    lib.lso_solve_b.argtypes = [_dp, ctypes.c_int64, ctypes.c_double, ctypes.c_double, _dp,
                                ctypes.POINTER(ctypes.c_int)]
    lib.lso_emit_p.restype = None
    lib.lso_emit_p.argtypes = [_dp, ctypes.c_int64, ctypes.c_double, ctypes.c_double, _dp]
    lib.lso_density.restype = None
    lib.lso_density.argtypes = [_dp, ctypes.c_int64, ctypes.c_double, ctypes.c_double, _dp]
    lib.lso_vjp.restype = None
    lib.lso_vjp.argtypes = [_dp, _dp, ctypes.c_int64, ctypes.c_double, ctypes.c_double, _dp,
                            _dp, _dp]
    lib.lso_vjp_kt.restype = None
    lib.lso_vjp_kt.argtypes = [_dp, _dp, ctypes.c_int64, ctypes.c_double, ctypes.c_double, _dp,
                               _dp]
    lib.lso_fold.restype = None
    lib.lso_fold.argtypes = [_dp, ctypes.c_int64, ctypes.c_double, ctypes.c_double,
                             ctypes.c_double, _i64p, _i64p, _i64p, _dp, _dp]
    lib.lso_splitmix64_at.restype = ctypes.c_uint64
    lib.lso_splitmix64_at.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
    lib.lso_sample.restype = None
    lib.lso_sample.argtypes = [_dp, ctypes.c_int64, ctypes.c_double, ctypes.c_uint64,
                               ctypes.c_uint64, ctypes.c_int64, _dp, _i64p]
    lib.lso_binom_ranks.restype = None
    lib.lso_binom_ranks.argtypes = [ctypes.c_int64, ctypes.c_double, ctypes.c_double, _i64p,
                                    _i64p]
    lib.lso_hard_topk.restype = ctypes.c_int
    lib.lso_hard_topk.argtypes = [_dp, ctypes.c_int64, ctypes.c_double, _dp, _dp]
    lib.lso_bracket_from_sample.restype = None
    lib.lso_bracket_from_sample.argtypes = [_dp, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.c_int64, _dp, _dp]
    return lib


def _lib():
    global _LIB
    with _LOCK:
        if _LIB is None:
            build()
            _LIB = configure(ctypes.CDLL(_SO))
    return _LIB


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64).reshape(-1))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_dp)


class OracleError(ValueError):
    pass


STATUS = {0: "ok", 1: "invalid argument", 3: "non-finite score"}


def laplace_cdf(x: float) -> float:
    return _lib().lso_laplace_cdf(float(x))


def budget_sum(r, b: float, t: float) -> float:
    """F(b) = sum_i sigma((r_i - b)/t), pairwise-summed in fp64."""
    a = _f64(r)
    return _lib().lso_budget_sum(_ptr(a), a.size, float(b), float(t))


def budget_sign(r, b: float, k: float, t: float) -> int:
    """Sign of F(b) - k, computed without cancellation."""
    a = _f64(r)
    return _lib().lso_budget_sign(_ptr(a), a.size, float(b), float(k), float(t))


def solve_b(r, k: float, t: float) -> float:
    """Exact threshold b of one row (full sort + cancellation-free bisection)."""
    a = _f64(r)
    out = ctypes.c_double(0.0)
    it = ctypes.c_int(0)
    st = _lib().lso_solve_b(_ptr(a), a.size, float(k), float(t), ctypes.byref(out),
                            ctypes.byref(it))
    if st != 0:
        raise OracleError(STATUS.get(st, str(st)))
    return out.value


def solve_rows(r2d, k: float, t: float) -> np.ndarray:
    """b for every row of a 2-D array."""
    r2d = np.asarray(r2d)
    return np.array([solve_b(row, k, t) for row in r2d.reshape(r2d.shape[0], -1)])


def emit_p(r, b: float, t: float) -> np.ndarray:
    a = _f64(r)
    p = np.empty_like(a)
    _lib().lso_emit_p(_ptr(a), a.size, float(b), float(t), _ptr(p))
    return p


def density(r, b: float, t: float) -> np.ndarray:
    a = _f64(r)
    f = np.empty_like(a)
    _lib().lso_density(_ptr(a), a.size, float(b), float(t), _ptr(f))
    return f


def vjp(r, v, b: float, t: float):
    """Returns (g, R, sum_f) with g_i = (f_i/t)(v_i - R)."""
    a = _f64(r)
    w = _f64(v)
    if a.size != w.size:
        raise OracleError("r and v differ in length")
    g = np.empty_like(a)
    R = ctypes.c_double(0.0)
    sf = ctypes.c_double(0.0)
    _lib().lso_vjp(_ptr(a), _ptr(w), a.size, float(b), float(t), _ptr(g), ctypes.byref(R),
                   ctypes.byref(sf))
    return g, R.value, sf.value


def vjp_kt(r, v, b: float, t: float):
    """Returns (dL/dk, dL/dt) of L = sum_i v_i p_i."""
    a = _f64(r)
    w = _f64(v)
    if a.size != w.size:
        raise OracleError("r and v differ in length")
    gk = ctypes.c_double(0.0)
    gt = ctypes.c_double(0.0)
    _lib().lso_vjp_kt(_ptr(a), _ptr(w), a.size, float(b), float(t), ctypes.byref(gk),
                      ctypes.byref(gt))
    return gk.value, gt.value


def fold(r, aL: float, aR: float, t: float) -> dict:
    a = _f64(r)
    cr, cl, nb = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    sl, sr = ctypes.c_double(), ctypes.c_double()
    _lib().lso_fold(_ptr(a), a.size, float(aL), float(aR), float(t), ctypes.byref(cr),
                    ctypes.byref(cl), ctypes.byref(nb), ctypes.byref(sl), ctypes.byref(sr))
    return {"cnt_R": cr.value, "cnt_L": cl.value, "n_band": nb.value, "S_L": sl.value,
            "S_R": sr.value}


def splitmix64_at(seed: int, c: int) -> int:
    return int(_lib().lso_splitmix64_at(ctypes.c_uint64(seed & (2**64 - 1)),
                                        ctypes.c_uint64(c & (2**64 - 1))))


def sample(r, t: float, seed: int, c0: int, m: int):
    """Laplace-noised sample y (fp64) and the sampled indices."""
    a = _f64(r)
    y = np.empty(m, dtype=np.float64)
    idx = np.empty(m, dtype=np.int64)
    _lib().lso_sample(_ptr(a), a.size, float(t), ctypes.c_uint64(seed & (2**64 - 1)),
                      ctypes.c_uint64(c0 & (2**64 - 1)), int(m), _ptr(y),
                      idx.ctypes.data_as(_i64p))
    return y, idx


def binom_ranks(m: int, q: float, alpha: float):
    l, h = ctypes.c_int64(), ctypes.c_int64()
    _lib().lso_binom_ranks(int(m), float(q), float(alpha), ctypes.byref(l), ctypes.byref(h))
    return l.value, h.value


def bracket_from_sample(y, l: int, h: int):
    a = _f64(y)
    aL, aR = ctypes.c_double(), ctypes.c_double()
    _lib().lso_bracket_from_sample(_ptr(a), a.size, int(l), int(h), ctypes.byref(aL),
                                   ctypes.byref(aR))
    return aL.value, aR.value


def hard_topk(r, k: float):
    """Zero-temperature limit: (b, p) with p the hard top-k mask, tied scores at the
    boundary sharing the remaining budget (lso_hard_topk)."""
    a = _f64(r)
    b = ctypes.c_double(0.0)
    p = np.empty_like(a)
    st = _lib().lso_hard_topk(_ptr(a), a.size, float(k), ctypes.byref(b), _ptr(p))
    if st != 0:
        raise OracleError(f"lso_hard_topk failed with status {st}")
    return b.value, p
