"""One row split over several devices: host orchestration of the split-row
pieces of ``liblapsum.so`` (``lapsum_shard_*`` and ``lapsum_bracket_plan`` in
``include/lapsum.h``), one process per device.

The method ("Fast LapSum: Exact Differentiable Top-k at Million Scale",
gist.science explainer pages, section 2.2) needs only small exchanges when a
row is split: the sample (every device draws the sample entries whose index
falls in its shard; one sum gives the whole sample), the fold's tail sums and
counts, the band, and in the backward the shards' shifted sums.  Every device
combines them in device order and takes the same decisions, so all compute
the same threshold b.  The arithmetic runs in the library's kernels; this
module moves the small tensors between devices (``DistComm`` over
torch.distributed) and runs the widening loop of the bracket.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib, _check, _stream_ptr, LapSumError

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
MAX_ATTEMPTS = 7


def _setup(lib):
    if getattr(lib, "_shard_ready", False):
        return lib
    lib.lapsum_bracket_plan.restype = ctypes.c_int
    lib.lapsum_bracket_plan.argtypes = [_i64, ctypes.c_double, ctypes.POINTER(ctypes.c_int32),
                                        ctypes.POINTER(_i64), ctypes.POINTER(_i64)]
    lib.lapsum_shard_workspace_bytes.restype = ctypes.c_size_t
    lib.lapsum_shard_workspace_bytes.argtypes = [_i64]
    lib.lapsum_shard_band_bytes.restype = ctypes.c_size_t
    lib.lapsum_shard_band_bytes.argtypes = [_i64]
    lib.lapsum_shard_sample.restype = ctypes.c_int
    lib.lapsum_shard_sample.argtypes = [_vp, _i64, _i64, _i64, ctypes.c_double, ctypes.c_uint64,
                                        ctypes.c_int32, _vp, _vp]
    lib.lapsum_sample_bracket.restype = ctypes.c_int
    lib.lapsum_sample_bracket.argtypes = [_vp, ctypes.c_int32, _i64, _i64, _vp, _vp]
    lib.lapsum_shard_fold.restype = ctypes.c_int
    lib.lapsum_shard_fold.argtypes = [_vp, _i64, _vp, ctypes.c_double, _vp, _vp, _vp,
                                      ctypes.c_size_t, _vp]
    lib.lapsum_shard_band_solve.restype = ctypes.c_int
    lib.lapsum_shard_band_solve.argtypes = [_vp, _i64, _vp, ctypes.c_int32, _vp, ctypes.c_double,
                                            ctypes.c_double, _vp, _vp, ctypes.c_size_t, _vp]
    lib.lapsum_shard_emit.restype = ctypes.c_int
    lib.lapsum_shard_emit.argtypes = [_vp, _i64, _vp, ctypes.c_double, _vp, _vp]
    lib.lapsum_shard_vjp_partial.restype = ctypes.c_int
    lib.lapsum_shard_vjp_partial.argtypes = [_vp, _vp, _i64, _vp, ctypes.c_double, _vp, _vp,
                                             ctypes.c_size_t, _vp]
    lib.lapsum_shard_vjp_apply.restype = ctypes.c_int
    lib.lapsum_shard_vjp_apply.argtypes = [_vp, _vp, _i64, _vp, ctypes.c_double, _vp,
                                           ctypes.c_int32, _vp, _vp, ctypes.c_size_t, _vp]
    lib._shard_ready = True
    return lib


def bracket_plan(n: int, k: float):
    """(m, rank_l[4], rank_h[4]) of a row of n scores with budget k (host)."""
    lib = _setup(_lib())
    m = ctypes.c_int32(0)
    rl = (_i64 * 4)()
    rh = (_i64 * 4)()
    _check(lib.lapsum_bracket_plan(n, float(k), ctypes.byref(m), rl, rh), "lapsum_bracket_plan")
    return int(m.value), list(rl), list(rh)


def _aligned(nbytes: int, device):
    buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
    ptr = (buf.data_ptr() + 255) // 256 * 256
    return buf, ptr


class GpuShardOps:
    """The per-shard steps on this process's CUDA device (the C ABI)."""

    def __init__(self, n_shard: int, device):
        self.lib = _setup(_lib())
        self.device = torch.device(device)
        self.n_shard = n_shard
        self.ws_bytes = int(self.lib.lapsum_shard_workspace_bytes(n_shard))
        self.ws_buf, self.ws = _aligned(self.ws_bytes, self.device)
        _check(self.lib.lapsum_workspace_init(self.ws, self.ws_bytes, self._s()),
               "lapsum_workspace_init")

    def _s(self):
        return _stream_ptr(self.device)

    def sample(self, r, offset, n, t, seed, m):
        y = torch.empty(m, dtype=torch.float32, device=self.device)
        _check(self.lib.lapsum_shard_sample(r.data_ptr(), r.numel(), offset, n, float(t), seed, m,
                                            y.data_ptr(), self._s()), "lapsum_shard_sample")
        return y

    def bracket(self, y, m, rank_l, rank_h):
        ends = torch.empty(2, dtype=torch.float32, device=self.device)
        _check(self.lib.lapsum_sample_bracket(y.data_ptr(), m, rank_l, rank_h, ends.data_ptr(),
                                              self._s()), "lapsum_sample_bracket")
        return ends

    def fold(self, r, ends, t):
        rec = torch.empty(5, dtype=torch.float64, device=self.device)
        band = torch.empty(max(1, r.numel()), dtype=torch.float32, device=self.device)
        _check(self.lib.lapsum_shard_fold(r.data_ptr(), r.numel(), ends.data_ptr(), float(t),
                                          rec.data_ptr(), band.data_ptr(), self.ws, self.ws_bytes,
                                          self._s()), "lapsum_shard_fold")
        return rec, band

    def band_solve(self, bands, stride, recs, world, ends, k, t):
        out = torch.empty(4, dtype=torch.float64, device=self.device)
        nbytes = int(self.lib.lapsum_shard_band_bytes(world * stride))
        buf, ptr = _aligned(nbytes, self.device)
        _check(self.lib.lapsum_shard_band_solve(bands.data_ptr(), stride, recs.data_ptr(), world,
                                                ends.data_ptr(), float(k), float(t),
                                                out.data_ptr(), ptr, nbytes, self._s()),
               "lapsum_shard_band_solve")
        return out

    def emit(self, r, b, t):
        p = torch.empty_like(r)
        _check(self.lib.lapsum_shard_emit(r.data_ptr(), r.numel(), b.data_ptr(), float(t),
                                          p.data_ptr(), self._s()), "lapsum_shard_emit")
        return p

    def vjp_partial(self, r, v, b, t):
        rec = torch.empty(3, dtype=torch.float64, device=self.device)
        _check(self.lib.lapsum_shard_vjp_partial(r.data_ptr(), v.data_ptr(), r.numel(),
                                                 b.data_ptr(), float(t), rec.data_ptr(), self.ws,
                                                 self.ws_bytes, self._s()),
               "lapsum_shard_vjp_partial")
        return rec

    def vjp_apply(self, r, v, b, t, recs, world):
        g = torch.empty_like(r)
        _check(self.lib.lapsum_shard_vjp_apply(r.data_ptr(), v.data_ptr(), r.numel(),
                                               b.data_ptr(), float(t), recs.data_ptr(), world,
                                               g.data_ptr(), self.ws, self.ws_bytes, self._s()),
               "lapsum_shard_vjp_apply")
        return g


class DistComm:
    """Sum and gather over a torch.distributed group.  With NCCL the device
    tensors are exchanged directly; with gloo they pass through host memory."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.host = dist.get_backend(group) != "nccl"

    def all_reduce_sum(self, x: torch.Tensor):
        if self.host:
            h = x.cpu()
            self.dist.all_reduce(h, group=self.group)
            x.copy_(h)
        else:
            self.dist.all_reduce(x, group=self.group)

    def all_gather(self, x: torch.Tensor) -> torch.Tensor:
        src = x.cpu() if self.host else x
        parts = [torch.empty_like(src) for _ in range(self.world)]
        self.dist.all_gather(parts, src, group=self.group)
        out = torch.stack(parts)
        return out.to(x.device) if self.host else out


class LocalComm:
    """The collectives of a single device (the whole row in one shard)."""
    world, rank = 1, 0

    def all_reduce_sum(self, x):
        return None

    def all_gather(self, x):
        return x.unsqueeze(0)


def forward(r_shard: torch.Tensor, k: float, t: float, n: int, offset: int, comm, ops=None,
            seed: int = 0):
    """(p of this shard, b as a 1-element fp64 tensor, attempts) for the row of n
    scores whose [offset, offset + len) part this process holds."""
    r = r_shard.reshape(-1)
    if ops is None:
        ops = GpuShardOps(r.numel(), r.device)
    m, rank_l, rank_h = bracket_plan(n, k)
    y = ops.sample(r, offset, n, t, seed, m)
    comm.all_reduce_sum(y)                 # one owner per draw: the sum is the sample
    il = ih = 0
    out = None
    for attempt in range(1, MAX_ATTEMPTS + 1):
        rl = rank_l[il] if rank_l[il] >= 1 else 0
        rh = rank_h[ih] if rank_h[ih] <= m else 0
        ends = ops.bracket(y, m, rl, rh)
        rec, band = ops.fold(r, ends, t)
        recs = comm.all_gather(rec)        # (world, 5)
        sizes = recs[:, 4].cpu()
        stride = max(1, int(sizes.max().item()))
        nb = int(rec[4].item())
        pad = torch.zeros(stride, dtype=band.dtype, device=band.device)
        pad[:nb] = band[:nb]
        bands = comm.all_gather(pad)       # (world, stride)
        out = ops.band_solve(bands, stride, recs, comm.world, ends, k, t)
        o = out.cpu()
        if o[3].item() == 1.0:
            break
        if attempt == MAX_ATTEMPTS:
            raise LapSumError(4, "sharded forward")
        # widen the failing end to its next rung
        if o[1].item() < k:
            ih = min(ih + 1, len(rank_h) - 1)
        else:
            il = min(il + 1, len(rank_l) - 1)
    b = out[0:1].clone()
    p = ops.emit(r, b, t)
    return p.reshape(r_shard.shape), b, attempt


def backward(r_shard: torch.Tensor, v_shard: torch.Tensor, b: torch.Tensor, t: float, comm,
             ops=None):
    """g of this shard: the shards' shifted sums merged in device order."""
    r = r_shard.reshape(-1)
    v = v_shard.reshape(-1).contiguous()
    if ops is None:
        ops = GpuShardOps(r.numel(), r.device)
    rec = ops.vjp_partial(r, v, b, t)
    recs = comm.all_gather(rec)            # (world, 3)
    g = ops.vjp_apply(r, v, b, t, recs, comm.world)
    return g.reshape(r_shard.shape)
