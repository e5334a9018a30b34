"""Fast LapSum soft top-k on B200 (sm_100a): Python binding of ``liblapsum.so``.

The operator ("Fast LapSum: Exact Differentiable Top-k at Million Scale",
gist.science explainer pages, section 2.1): per row of scores ``r``,

    p_i = sigma((r_i - b)/t),  sigma = Laplace(0,1) CDF,  sum_i p_i = k,

with the exact threshold ``b`` and the analytic VJP
``g_i = (f_i/t)(v_i - sum_j v_j f_j / sum_j f_j)``, ``f_i = 0.5 exp(-|r_i - b|/t)``.

This module only marshals arguments: it takes torch CUDA tensors, passes their
device pointers and the current stream to the C ABI declared in
``include/lapsum.h``, and raises on a non-zero return code.  Every step of the
computation runs in the library's CUDA kernels; there is no CPU or PyTorch
fallback, and importing the package fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import _build

__all__ = [
    "LapSumError", "Workspace", "forward", "backward", "read_status", "row_info", "sample_values",
    "workspace_bytes", "soft_topk", "LapSumTopK", "PATHS", "FLAG_FORCE_MISS", "FLAG_NO_RETRY",
    "FLAG_ONE_CTA_SOLVE", "library_path", "profile_enable", "backward_kt", "profile_read", "backward_noalloc", "Support",
    "support_bytes", "forward_lowp", "backward_lowp",
]

PATHS = {"auto": 0, "fullsort": 1, "bracket": 2, "radix": 3, "rowbracket": 4}
FLAG_FORCE_MISS = 0x100
FLAG_NO_RETRY = 0x200
FLAG_ONE_CTA_SOLVE = 0x400

_c_i64 = ctypes.c_int64
_vp = ctypes.c_void_p


class LapSumError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {_lib().lapsum_status_string(code).decode()} (code {code})")


class RowInfo(ctypes.Structure):
    _fields_ = [("b", ctypes.c_double), ("sum_f", ctypes.c_double), ("S_L", ctypes.c_double),
                ("S_R", ctypes.c_double), ("a_L", ctypes.c_float), ("a_R", ctypes.c_float),
                ("cnt_R", ctypes.c_int64), ("n_band", ctypes.c_int64), ("path", ctypes.c_int32),
                ("attempts", ctypes.c_int32), ("sample_m", ctypes.c_int32),
                ("rank_l", ctypes.c_int32), ("rank_h", ctypes.c_int32),
                ("refine_levels", ctypes.c_int32), ("status", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int64),
                ("total_ms", ctypes.c_double)]


_LIB = None


def library_path() -> str:
    return _build.SO


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(_build.SO):
            raise ImportError(
                f"liblapsum.so is not built ({_build.SO}); run __graft_entry__.build() or "
                "python -m sparse_selection_primitive_b200._build")
        lib = ctypes.CDLL(_build.SO)
        lib.lapsum_abi_version.restype = ctypes.c_int
        lib.lapsum_status_string.restype = ctypes.c_char_p
        lib.lapsum_status_string.argtypes = [ctypes.c_int]
        lib.lapsum_workspace_bytes.restype = ctypes.c_size_t
        lib.lapsum_workspace_bytes.argtypes = [_c_i64, _c_i64, ctypes.c_double, ctypes.c_int]
        lib.lapsum_backward_workspace_bytes.restype = ctypes.c_size_t
        lib.lapsum_backward_workspace_bytes.argtypes = [_c_i64, _c_i64]
        lib.lapsum_workspace_init.restype = ctypes.c_int
        lib.lapsum_workspace_init.argtypes = [_vp, ctypes.c_size_t, _vp]
        lib.lapsum_forward.restype = ctypes.c_int
        lib.lapsum_forward.argtypes = [_vp, _c_i64, _vp, _vp, _vp, _c_i64, _c_i64, ctypes.c_double,
                                       ctypes.c_double, ctypes.c_int, ctypes.c_uint64, _vp,
                                       ctypes.c_size_t, _vp]
        lib.lapsum_backward.restype = ctypes.c_int
        lib.lapsum_backward.argtypes = [_vp, _c_i64, _vp, _vp, _vp, _c_i64, _c_i64,
                                        ctypes.c_double, _vp, ctypes.c_size_t, _vp]
        lib.lapsum_read_status.restype = ctypes.c_int
        lib.lapsum_read_status.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_int)]
        lib.lapsum_row_info_get.restype = ctypes.c_int
        lib.lapsum_row_info_get.argtypes = [_vp, _c_i64, ctypes.POINTER(RowInfo), _vp]
        lib.lapsum_profile_enable.restype = ctypes.c_int
        lib.lapsum_profile_enable.argtypes = [ctypes.c_int]
        lib.lapsum_profile_read.restype = ctypes.c_int
        lib.lapsum_profile_read.argtypes = [ctypes.POINTER(KernelTime), ctypes.c_int,
                                            ctypes.POINTER(ctypes.c_int)]
        lib.lapsum_support_bytes.restype = ctypes.c_size_t
        lib.lapsum_support_bytes.argtypes = [_c_i64, _c_i64]
        lib.lapsum_forward_support.restype = ctypes.c_int
        lib.lapsum_forward_support.argtypes = [_vp, _c_i64, _vp, _vp, _vp, _c_i64, _c_i64,
                                               ctypes.c_double, ctypes.c_double, ctypes.c_int,
                                               ctypes.c_uint64, _vp, ctypes.c_size_t, _vp,
                                               ctypes.c_size_t, _vp]
        lib.lapsum_backward_support.restype = ctypes.c_int
        lib.lapsum_backward_support.argtypes = [_vp, _c_i64, _vp, _vp, _vp, _c_i64, _c_i64,
                                                ctypes.c_double, _vp, ctypes.c_size_t, _vp,
                                                ctypes.c_size_t, _vp]
        lib.lapsum_backward_kt.restype = ctypes.c_int
        lib.lapsum_backward_kt.argtypes = [_vp, _c_i64, _vp, _vp, _c_i64, _c_i64, ctypes.c_double,
                                           _vp, _vp, _vp, ctypes.c_size_t, _vp]
        lib.lapsum_forward_hard.restype = ctypes.c_int
        lib.lapsum_forward_hard.argtypes = [_vp, _c_i64, _vp, _vp, _c_i64, _c_i64, ctypes.c_double,
                                            ctypes.c_int, _vp, ctypes.c_size_t, _vp]
        lib.lapsum_forward_router.restype = ctypes.c_int
        lib.lapsum_forward_router.argtypes = [_vp, ctypes.c_int, _c_i64, _vp, _vp, _c_i64, _c_i64,
                                              ctypes.c_double, ctypes.c_double, ctypes.c_float,
                                              ctypes.c_int32, _vp, _vp, _vp, _vp, ctypes.c_size_t,
                                              _vp]
        lib.lapsum_backward_router.restype = ctypes.c_int
        lib.lapsum_backward_router.argtypes = [_vp, ctypes.c_int, _c_i64, _vp, _vp, _vp, _c_i64,
                                               _c_i64, ctypes.c_double, _vp]
        lib.lapsum_workspace_bytes_rowk.restype = ctypes.c_size_t
        lib.lapsum_workspace_bytes_rowk.argtypes = [_c_i64, _c_i64, ctypes.c_int]
        lib.lapsum_forward_rowk.restype = ctypes.c_int
        lib.lapsum_forward_rowk.argtypes = [_vp, _c_i64, _vp, _vp, _vp, _c_i64, _c_i64, _vp,
                                            ctypes.c_double, ctypes.c_int, _vp, ctypes.c_size_t,
                                            _vp, ctypes.c_size_t, _vp]
        lib.lapsum_sample_get.restype = ctypes.c_int
        lib.lapsum_sample_get.argtypes = [_vp, _c_i64, _vp, _c_i64, _vp]
        lib.lapsum_workspace_bytes_lowp.restype = ctypes.c_size_t
        lib.lapsum_workspace_bytes_lowp.argtypes = [_c_i64, _c_i64, _c_i64, ctypes.c_double,
                                                    ctypes.c_int]
        lib.lapsum_backward_workspace_bytes_lowp.restype = ctypes.c_size_t
        lib.lapsum_backward_workspace_bytes_lowp.argtypes = [_c_i64, _c_i64, _c_i64]
        lib.lapsum_forward_lowp.restype = ctypes.c_int
        lib.lapsum_forward_lowp.argtypes = [_vp, ctypes.c_int, _c_i64, _vp, _vp, _vp, _c_i64,
                                            _c_i64, ctypes.c_double, ctypes.c_double, ctypes.c_int,
                                            ctypes.c_uint64, _vp, ctypes.c_size_t, _vp,
                                            ctypes.c_size_t, _vp]
        lib.lapsum_backward_lowp.restype = ctypes.c_int
        lib.lapsum_backward_lowp.argtypes = [_vp, ctypes.c_int, _c_i64, _vp, _vp, _vp, _c_i64,
                                             _c_i64, ctypes.c_double, _vp, ctypes.c_size_t, _vp,
                                             ctypes.c_size_t, _vp]
        _LIB = lib
    return _LIB


def _stream_ptr(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check(code: int, where: str):
    if code != 0:
        raise LapSumError(code, where)


def _path_code(path) -> int:
    if isinstance(path, str):
        return PATHS[path]
    return int(path)


def workspace_bytes(B: int, n: int, k: float, path="auto") -> int:
    return int(_lib().lapsum_workspace_bytes(B, n, float(k), _path_code(path)))


class Workspace:
    """Device workspace for forward/backward, allocated once with torch and reused.

    The library itself never allocates; this object owns the bytes (a torch
    uint8 tensor, 256-byte aligned) and clears them once with
    ``lapsum_workspace_init``.
    """

    def __init__(self, B: int, n: int, k: float, path="auto", device=None, nbytes: int = None):
        device = torch.device(device or "cuda")
        self.nbytes = workspace_bytes(B, n, k, path) if nbytes is None else int(nbytes)
        if self.nbytes == 0:
            raise LapSumError(1, "workspace_bytes")
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device)
        base = self.buf.data_ptr()
        self.ptr = (base + 255) // 256 * 256
        self.device = device
        _check(_lib().lapsum_workspace_init(self.ptr, self.nbytes, _stream_ptr(device)),
               "lapsum_workspace_init")

    def fits(self, B, n, k, path) -> bool:
        return workspace_bytes(B, n, k, path) <= self.nbytes

    def fits_backward(self, B, n) -> bool:
        return int(_lib().lapsum_backward_workspace_bytes(B, n)) <= self.nbytes


def support_bytes(B: int, n: int) -> int:
    return int(_lib().lapsum_support_bytes(B, n))


class Support:
    """Gradient-support buffer handed from forward to backward (rows with n > 4096).

    The forward lists the scores with |r - b|/t <= 90 (the only ones with a
    non-zero gradient in fp32); the backward then reads v only there and never
    reads r.  Owned by torch (uint8, 256-byte aligned); no initialisation.
    For n <= 4096 it holds no memory and the plain entry points run.
    """

    def __init__(self, B: int, n: int, device=None):
        device = torch.device(device or "cuda")
        self.B, self.n = B, n
        self.nbytes = support_bytes(B, n)
        self.buf = torch.empty(self.nbytes + 256 if self.nbytes else 0, dtype=torch.uint8,
                               device=device)
        base = self.buf.data_ptr()
        self.ptr = (base + 255) // 256 * 256 if self.nbytes else None
        self.device = device

    def fits(self, B, n) -> bool:
        return support_bytes(B, n) <= self.nbytes


def _as_rows(x: torch.Tensor) -> torch.Tensor:
    if x.dim() == 1:
        x = x.unsqueeze(0)
    if x.dim() != 2:
        raise ValueError("scores must be 1-D or 2-D (rows x n)")
    if x.dtype != torch.float32 or not x.is_cuda:
        raise TypeError("scores must be a float32 CUDA tensor")
    B, n = x.shape
    if x.stride(1) != 1 or (B > 1 and x.stride(0) < n):
        x = x.contiguous()
    return x


def _ld(x: torch.Tensor) -> int:
    """Leading dimension of a row-major (B, n) view; a single row has ld = n."""
    return x.stride(0) if x.shape[0] > 1 else x.shape[1]


def _like_rows(x: torch.Tensor, ld: int) -> torch.Tensor:
    """Uninitialised (B, n) float32 buffer with the same leading dimension as x."""
    B, n = x.shape
    if ld == n:
        return torch.empty((B, n), dtype=torch.float32, device=x.device)
    return torch.empty((B, ld), dtype=torch.float32, device=x.device)[:, :n]


def _check_out(out: torch.Tensor, ref: torch.Tensor, ld: int, what: str):
    if out.shape != ref.shape or out.dtype != torch.float32 or not out.is_cuda or \
            out.stride(1) != 1 or _ld(out) != ld:
        raise ValueError(f"{what} must be float32 CUDA with the shape and row stride of r")


def _row_budgets(k, B: int, device):
    """k as a per-row budget tensor (float64 on the scores' device), or None for
    a shared scalar budget.  A 1-D tensor with one entry per row is per-row."""
    if isinstance(k, torch.Tensor) and k.dim() == 1:
        if k.numel() != B:
            raise ValueError("a per-row k needs one entry per row")
        return k.detach().to(device=device, dtype=torch.float64).contiguous()
    return None


def forward(r: torch.Tensor, k, t: float, path="auto", seed: int = 0, ws: Workspace = None,
            want_sum_f: bool = False, p: torch.Tensor = None, b: torch.Tensor = None,
            support: Support = None):
    """Returns (p, b[, sum_f]) for each row of r (float32 CUDA, rows x n or n).

    k is a number shared by every row, or a 1-D tensor with one budget per row
    (lapsum_forward_rowk: every solver).  With ``support`` (a Support
    for the same B, n) the forward also lists the gradient support for
    backward(..., support=...)."""
    squeeze = r.dim() == 1
    r2 = _as_rows(r)
    B, n = r2.shape
    ld = _ld(r2)
    code = _path_code(path)
    k_rows = _row_budgets(k, B, r2.device)
    if k_rows is not None:
        need = int(_lib().lapsum_workspace_bytes_rowk(B, n, code))
        if need == 0:
            raise LapSumError(1, "lapsum_workspace_bytes_rowk")
        if ws is None or ws.nbytes < need:
            ws = Workspace(B, n, 1.0, code, r2.device, nbytes=need)
    elif ws is None or not ws.fits(B, n, k, code):
        ws = Workspace(B, n, k, code, r2.device)
    if p is None:
        p = _like_rows(r2, ld)
    else:
        p = p.view(B, n) if p.dim() == 1 else p
        _check_out(p, r2, ld, "p")
    if b is None:
        b = torch.empty(B, dtype=torch.float64, device=r2.device)
    elif b.dtype != torch.float64 or b.numel() != B or not b.is_contiguous():
        raise ValueError("b must be a contiguous float64 CUDA tensor with one entry per row")
    sf = torch.empty(B, dtype=torch.float64, device=r2.device) if want_sum_f else None
    if k_rows is not None:
        if support is not None and not support.fits(B, n):
            raise ValueError("support buffer too small for (B, n)")
        _check(_lib().lapsum_forward_rowk(
            r2.data_ptr(), ld, p.data_ptr(), b.data_ptr(),
            sf.data_ptr() if sf is not None else None, B, n, k_rows.data_ptr(), float(t), code,
            ws.ptr, ws.nbytes, support.ptr if support is not None else None,
            support.nbytes if support is not None else 0, _stream_ptr(r2.device)),
            "lapsum_forward_rowk")
    elif support is not None:
        if not support.fits(B, n):
            raise ValueError("support buffer too small for (B, n)")
        _check(_lib().lapsum_forward_support(
            r2.data_ptr(), ld, p.data_ptr(), b.data_ptr(),
            sf.data_ptr() if sf is not None else None, B, n, float(k), float(t), code,
            seed & (2**64 - 1), ws.ptr, ws.nbytes, support.ptr, support.nbytes,
            _stream_ptr(r2.device)), "lapsum_forward_support")
    else:
        _check(_lib().lapsum_forward(r2.data_ptr(), ld, p.data_ptr(), b.data_ptr(),
                                     sf.data_ptr() if sf is not None else None, B, n, float(k),
                                     float(t), code, seed & (2**64 - 1), ws.ptr, ws.nbytes,
                                     _stream_ptr(r2.device)), "lapsum_forward")
    if squeeze:
        p = p[0]
    return (p, b, sf) if want_sum_f else (p, b)


def backward(r: torch.Tensor, b: torch.Tensor, v: torch.Tensor, t: float, ws: Workspace = None,
             g: torch.Tensor = None, support: Support = None):
    """g = J^T v for each row (J the Jacobian of p with respect to r).

    With ``support`` (filled by forward(..., support=...) for this r and b)
    v is read only at the listed scores and r is not read."""
    squeeze = r.dim() == 1
    r2 = _as_rows(r)
    v2 = _as_rows(v)
    B, n = r2.shape
    if v2.shape != r2.shape:
        raise ValueError("v must have the shape of r")
    if _ld(v2) != _ld(r2):
        v2 = v2.contiguous()
        r2 = r2.contiguous()
    ld = _ld(r2)
    if ws is None or not ws.fits_backward(B, n):
        ws = Workspace(B, n, 0.5, "fullsort", r2.device)
    if g is None:
        g = _like_rows(r2, ld)
    else:
        g = g.view(B, n) if g.dim() == 1 else g
        _check_out(g, r2, ld, "g")
    if b.dtype != torch.float64 or not b.is_cuda or b.numel() != B:
        raise TypeError("b must be a float64 CUDA tensor with one entry per row")
    if support is not None:
        if not support.fits(B, n):
            raise ValueError("support buffer too small for (B, n)")
        _check(_lib().lapsum_backward_support(
            r2.data_ptr(), ld, b.data_ptr(), v2.data_ptr(), g.data_ptr(), B, n, float(t),
            support.ptr, support.nbytes, ws.ptr, ws.nbytes, _stream_ptr(r2.device)),
            "lapsum_backward_support")
    else:
        _check(_lib().lapsum_backward(r2.data_ptr(), ld, b.data_ptr(), v2.data_ptr(),
                                      g.data_ptr(), B, n, float(t), ws.ptr, ws.nbytes,
                                      _stream_ptr(r2.device)), "lapsum_backward")
    return g[0] if squeeze else g


def hard_topk(r: torch.Tensor, k: float, path="auto", ws: Workspace = None):
    """Zero-temperature limit (lapsum_forward_hard): (p, b) per row of r (float32
    CUDA): p = 1 above the boundary score c = the ceil(k)-th largest, 0 below,
    and the scores equal to c share the remaining budget (sum p = k)."""
    squeeze = r.dim() == 1
    r2 = _as_rows(r)
    B, n = r2.shape
    ld = _ld(r2)
    code = _path_code(path)
    # the full-sort workspace for AUTO and FULLSORT, the radix one otherwise
    wpath = "fullsort" if (code & 0xFF) in (PATHS["auto"], PATHS["fullsort"]) else "radix"
    if ws is None or not ws.fits(B, n, k, wpath):
        ws = Workspace(B, n, k, wpath, r2.device)
    p = _like_rows(r2, ld)
    b = torch.empty(B, dtype=torch.float64, device=r2.device)
    _check(_lib().lapsum_forward_hard(r2.data_ptr(), ld, p.data_ptr(), b.data_ptr(), B, n,
                                      float(k), code, ws.ptr, ws.nbytes, _stream_ptr(r2.device)),
           "lapsum_forward_hard")
    return (p[0] if squeeze else p), b


_DTYPES = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}


def _router_rows(x: torch.Tensor) -> torch.Tensor:
    if x.dim() == 1:
        x = x.unsqueeze(0)
    if x.dim() != 2 or x.dtype not in _DTYPES or not x.is_cuda:
        raise TypeError("router scores must be a float32, bfloat16 or float16 CUDA tensor, "
                        "rows x n")
    if x.stride(1) != 1 or (x.shape[0] > 1 and x.stride(0) < x.shape[1]):
        x = x.contiguous()
    return x


def forward_router(r: torch.Tensor, k: float, t: float, eps: float = None, cap: int = None,
                   ws: Workspace = None, out=None):
    """Router form for rows of n <= 4096 (lapsum_forward_router): r is float32 or
    bfloat16.  Returns (p, b), or with eps and cap also (idx, vals, cnt): per row
    the positions and values of p > eps (at most cap, ascending) and their count;
    list slots past the count are left as they were.  ``out`` may hold the
    output tensors to fill: (p, b) or (p, b, idx, vals, cnt), p with r's row
    stride."""
    r2 = _router_rows(r)
    B, n = r2.shape
    ld = r2.stride(0) if B > 1 else n
    if ws is None or not ws.fits(B, n, 0.5 * n, "fullsort"):
        ws = Workspace(B, n, 0.5 * n, "fullsort", r2.device)
    want = eps is not None
    if out is not None:
        p, b = out[0], out[1]
        _check_out(p, r2, ld, "p")
        if want:
            idx, vals, cnt = out[2], out[3], out[4]
            if idx.shape != (B, cap) or vals.shape != (B, cap) or cnt.numel() != B:
                raise ValueError("selection outputs must be (B, cap), (B, cap) and (B,)")
    else:
        p = torch.empty((B, ld), dtype=torch.float32, device=r2.device)[:, :n]
        b = torch.empty(B, dtype=torch.float64, device=r2.device)
        if want:
            idx = torch.empty((B, cap), dtype=torch.int32, device=r2.device)
            vals = torch.empty((B, cap), dtype=torch.float32, device=r2.device)
            cnt = torch.empty(B, dtype=torch.int32, device=r2.device)
    _check(_lib().lapsum_forward_router(
        r2.data_ptr(), _DTYPES[r2.dtype], ld, p.data_ptr(), b.data_ptr(), B, n, float(k),
        float(t), float(eps) if want else 0.0, int(cap) if want else 0,
        idx.data_ptr() if want else None, vals.data_ptr() if want else None,
        cnt.data_ptr() if want else None, ws.ptr, ws.nbytes, _stream_ptr(r2.device)),
        "lapsum_forward_router")
    if r.dim() == 1:
        p = p[0]
    return (p, b, idx, vals, cnt) if want else (p, b)


def backward_router(r: torch.Tensor, b: torch.Tensor, v: torch.Tensor, t: float,
                    g: torch.Tensor = None):
    """g (float32) for router scores r (float32 or bfloat16), n <= 4096."""
    r2 = _router_rows(r)
    B, n = r2.shape
    v2 = v.reshape(B, n).to(torch.float32).contiguous()
    if r2.stride(0) != n and B > 1:
        r2 = r2.contiguous()
    if g is None:
        g = torch.empty((B, n), dtype=torch.float32, device=r2.device)
    elif g.shape != (B, n) or g.dtype != torch.float32 or not g.is_contiguous():
        raise ValueError("g must be a contiguous float32 (B, n) tensor")
    _check(_lib().lapsum_backward_router(r2.data_ptr(), _DTYPES[r2.dtype], n, b.data_ptr(),
                                         v2.data_ptr(), g.data_ptr(), B, n, float(t),
                                         _stream_ptr(r2.device)), "lapsum_backward_router")
    return g[0] if r.dim() == 1 else g


def _lowp_rows(x: torch.Tensor) -> torch.Tensor:
    if x.dim() == 1:
        x = x.unsqueeze(0)
    if x.dim() != 2 or x.dtype not in _DTYPES or not x.is_cuda:
        raise TypeError("scores must be a float32, bfloat16 or float16 CUDA tensor, rows x n")
    if x.stride(1) != 1 or (x.shape[0] > 1 and x.stride(0) < x.shape[1]):
        x = x.contiguous()
    return x


def forward_lowp(r: torch.Tensor, k: float, t: float, path="auto", seed: int = 0,
                 want_sum_f: bool = False, support: Support = None, ws_bytes: int = None):
    """Forward on scores of any of float32, bfloat16, float16 and any row length
    (lapsum_forward_lowp: the on-chip kernels read 16-bit scores directly; longer
    rows are widened exactly into the workspace first).  Returns (p, b[, sum_f])
    with p float32 in r's row stride; ``support`` as in forward()."""
    r2 = _lowp_rows(r)
    B, n = r2.shape
    ld = r2.stride(0) if B > 1 else n
    code = _path_code(path)
    nbytes = int(_lib().lapsum_workspace_bytes_lowp(B, n, ld, float(k), code))
    if nbytes == 0:
        raise LapSumError(1, "lapsum_workspace_bytes_lowp")
    ws = Workspace(B, n, k, path, r2.device, nbytes=nbytes)
    p = torch.empty((B, ld), dtype=torch.float32, device=r2.device)[:, :n]
    b = torch.empty(B, dtype=torch.float64, device=r2.device)
    sf = torch.empty(B, dtype=torch.float64, device=r2.device) if want_sum_f else None
    sup_ptr, sup_n = (support.ptr, support.nbytes) if support is not None else (None, 0)
    _check(_lib().lapsum_forward_lowp(
        r2.data_ptr(), _DTYPES[r2.dtype], ld, p.data_ptr(), b.data_ptr(),
        sf.data_ptr() if want_sum_f else None, B, n, float(k), float(t), code, int(seed),
        ws.ptr, ws.nbytes, sup_ptr, sup_n, _stream_ptr(r2.device)), "lapsum_forward_lowp")
    if r.dim() == 1:
        p = p[0]
    return (p, b, sf) if want_sum_f else (p, b)


def backward_lowp(r: torch.Tensor, b: torch.Tensor, v: torch.Tensor, t: float,
                  support: Support = None):
    """g (float32) for scores r of float32, bfloat16 or float16 (lapsum_backward_lowp)."""
    r2 = _lowp_rows(r)
    B, n = r2.shape
    ld = r2.stride(0) if B > 1 else n
    v2 = v.reshape(B, n).to(torch.float32)
    v2 = torch.empty((B, ld), dtype=torch.float32, device=r2.device)[:, :n].copy_(v2) \
        if ld != n else v2.contiguous()
    g = torch.empty((B, ld), dtype=torch.float32, device=r2.device)[:, :n]
    nbytes = int(_lib().lapsum_backward_workspace_bytes_lowp(B, n, ld))
    ws = Workspace(B, n, 0.5 * n, "auto", r2.device, nbytes=nbytes)
    sup_ptr, sup_n = (support.ptr, support.nbytes) if support is not None else (None, 0)
    _check(_lib().lapsum_backward_lowp(r2.data_ptr(), _DTYPES[r2.dtype], ld, b.data_ptr(),
                                       v2.data_ptr(), g.data_ptr(), B, n, float(t), sup_ptr,
                                       sup_n, ws.ptr, ws.nbytes, _stream_ptr(r2.device)),
           "lapsum_backward_lowp")
    return g[0] if r.dim() == 1 else g


def backward_kt(r: torch.Tensor, b: torch.Tensor, v: torch.Tensor, t: float,
                ws: Workspace = None):
    """(dL/dk, dL/dt) per row of L = sum v p, as float64 tensors of B entries."""
    r2 = _as_rows(r)
    v2 = _as_rows(v)
    B, n = r2.shape
    if v2.shape != r2.shape:
        raise ValueError("v must have the shape of r")
    if _ld(v2) != _ld(r2):
        v2 = v2.contiguous()
        r2 = r2.contiguous()
    if b.dtype != torch.float64 or not b.is_cuda or b.numel() != B:
        raise TypeError("b must be a float64 CUDA tensor with one entry per row")
    if ws is None or not ws.fits_backward(B, n):
        ws = Workspace(B, n, 0.5, "fullsort", r2.device)
    gk = torch.empty(B, dtype=torch.float64, device=r2.device)
    gt = torch.empty(B, dtype=torch.float64, device=r2.device)
    _check(_lib().lapsum_backward_kt(r2.data_ptr(), _ld(r2), b.data_ptr(), v2.data_ptr(), B, n,
                                     float(t), gk.data_ptr(), gt.data_ptr(), ws.ptr, ws.nbytes,
                                     _stream_ptr(r2.device)), "lapsum_backward_kt")
    return gk, gt


def backward_noalloc(r: torch.Tensor, b: torch.Tensor, v: torch.Tensor, t: float,
                     g: torch.Tensor = None):
    """Backward without a workspace, for callers that cannot allocate device memory.

    Same result as backward(); the library keeps its scratch in a fixed array
    (limits: at most 1024 rows).  Calls on one device must not overlap on the
    GPU, and the first call on a device must come before any stream capture.
    """
    lib = _lib()
    fn = lib.lapsum_backward_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [_vp, _c_i64, _vp, _vp, _vp, _c_i64, _c_i64, ctypes.c_double, _vp]
    squeeze = r.dim() == 1
    r2 = _as_rows(r)
    v2 = _as_rows(v)
    B, n = r2.shape
    if v2.shape != r2.shape:
        raise ValueError("v must have the shape of r")
    if _ld(v2) != _ld(r2):
        v2 = v2.contiguous()
        r2 = r2.contiguous()
    ld = _ld(r2)
    if g is None:
        g = _like_rows(r2, ld)
    else:
        g = g.view(B, n) if g.dim() == 1 else g
        _check_out(g, r2, ld, "g")
    if b.dtype != torch.float64 or not b.is_cuda or b.numel() != B:
        raise TypeError("b must be a float64 CUDA tensor with one entry per row")
    _check(fn(r2.data_ptr(), ld, b.data_ptr(), v2.data_ptr(), g.data_ptr(), B, n, float(t),
              _stream_ptr(r2.device)), "lapsum_backward_noalloc")
    return g[0] if squeeze else g


def read_status(ws: Workspace) -> int:
    st = ctypes.c_int(0)
    _check(_lib().lapsum_read_status(ws.ptr, _stream_ptr(ws.device), ctypes.byref(st)),
           "lapsum_read_status")
    return st.value


def row_info(ws: Workspace, row: int = 0) -> dict:
    info = RowInfo()
    _check(_lib().lapsum_row_info_get(ws.ptr, row, ctypes.byref(info), _stream_ptr(ws.device)),
           "lapsum_row_info_get")
    return {name: getattr(info, name) for name, _ in RowInfo._fields_ if name != "reserved"}


def sample_values(ws: Workspace, row: int, m: int):
    import numpy as np
    out = np.empty(m, dtype=np.float32)
    _check(_lib().lapsum_sample_get(ws.ptr, row, out.ctypes.data, m, _stream_ptr(ws.device)),
           "lapsum_sample_get")
    return out


def profile_enable(on: bool = True):
    """Start (or stop) per-kernel CUDA-event timing inside the library."""
    _check(_lib().lapsum_profile_enable(1 if on else 0), "lapsum_profile_enable")


def profile_read() -> dict:
    """{kernel name: (launches, total device ms)} since profile_enable(True)."""
    buf = (KernelTime * 64)()
    cnt = ctypes.c_int(0)
    _check(_lib().lapsum_profile_read(buf, 64, ctypes.byref(cnt)), "lapsum_profile_read")
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].total_ms))
            for i in range(min(cnt.value, 64))}


class LapSumTopK(torch.autograd.Function):
    """Autograd wrapper.  Rows longer than 4096 go through lapsum_forward_support
    and lapsum_backward_support (the gradient support is kept for backward);
    shorter rows through lapsum_forward and lapsum_backward."""

    @staticmethod
    def forward(ctx, r, k, t, path="auto", seed=0):
        rd = r.detach()
        B = 1 if rd.dim() == 1 else rd.shape[0]
        n = rd.shape[-1]
        per_row = isinstance(k, torch.Tensor) and k.dim() == 1
        ctx.lowp = rd.dtype in (torch.bfloat16, torch.float16)
        if ctx.lowp:
            # 16-bit scores (one shared k): lapsum_forward_lowp; p is fp32, the
            # gradient with respect to r comes back in r's dtype
            if per_row:
                raise ValueError("16-bit scores take one shared k")
            tf = float(t)
            sup = Support(B, n, rd.device) if support_bytes(B, n) > 0 else None
            p, b = forward_lowp(rd, float(k), tf, path=path, seed=seed, support=sup)
            ctx.save_for_backward(r, b)
            ctx.t = tf
            ctx.sup = sup
            ctx.kt_grad = (isinstance(k, torch.Tensor) and k.requires_grad,
                           isinstance(t, torch.Tensor) and t.requires_grad)
            ctx.kt_like = (k, t)
            return p
        kf = k.detach() if per_row else float(k)
        tf = float(t)
        sup = Support(B, n, rd.device) if support_bytes(B, n) > 0 else None
        p, b = forward(rd, kf, tf, path=path, seed=seed, support=sup)
        ctx.save_for_backward(r, b)
        ctx.t = tf
        ctx.sup = sup
        ctx.kt_grad = (isinstance(k, torch.Tensor) and k.requires_grad,
                       isinstance(t, torch.Tensor) and t.requires_grad)
        ctx.kt_like = (k, t)
        return p

    @staticmethod
    def backward(ctx, gp):
        r, b = ctx.saved_tensors
        v = gp.contiguous()
        if ctx.lowp:
            g = backward_lowp(r.detach(), b, v, ctx.t, support=ctx.sup).to(r.dtype)
        else:
            g = backward(r.detach(), b, v, ctx.t, support=ctx.sup)
        ctx.sup = None
        gk = gt = None
        if any(ctx.kt_grad):
            # a shared k or t gets the sum over rows of the per-row gradients;
            # a per-row k (one entry per row) gets them row by row
            r32 = r.detach().float() if ctx.lowp else r.detach()
            gks, gts = backward_kt(r32, b, v, ctx.t)
            k, t = ctx.kt_like
            if ctx.kt_grad[0]:
                if k.dim() == 1:
                    gk = gks.reshape(-1).to(k.dtype)
                else:
                    gk = gks.sum().to(k.dtype).reshape(k.shape)
            if ctx.kt_grad[1]:
                gt = gts.sum().to(t.dtype).reshape(t.shape)
        return g, gk, gt, None, None


def soft_topk(r: torch.Tensor, k, t: float, path="auto", seed: int = 0) -> torch.Tensor:
    """Differentiable soft top-k probabilities p with sum p = k per row (k a number,
    or a 1-D tensor with one budget per row)."""
    return LapSumTopK.apply(r, k, t, path, seed)
