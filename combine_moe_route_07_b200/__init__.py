"""On-GPU MoE token route / layout / dispatch / combine for NVIDIA B200 (sm_100a).

Python binding over the C ABI in include/moe_route07.h.  The functions carry
the ABI's names and only marshal arguments: they check that tensors are CUDA,
contiguous and of the right dtype, allocate outputs with torch when the caller
passes none, and forward data pointers plus torch's current stream.  Every
step of the path runs in the library's kernels.

    shape = MoeShape(tokens=T, hidden=H, experts=E, k=k, ranks=R)
    ws = Workspace(shape)                       # zero-filled device workspace
    ids, gates = moe_route(shape, logits, bias, ws=ws)
    lay = moe_layout(shape, ids, ws=ws)
    xd = moe_dispatch(shape, x, lay.dst_pos, ws=ws)
    ...  experts turn xd into y (same rows) ...
    out = moe_combine(shape, y, lay.dst_pos, gates, ws=ws, residual=x)
    moe_check(ws)                               # raises on a device-side error
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional

import torch

from . import _binding
from ._binding import MoeError, MOE_F_FP8, MOE_F_RENORM, MOE_F_SRC_LAYOUT

__all__ = ["MoeShape", "Workspace", "Layout", "LayoutSrc", "MoeError", "moe_route", "moe_layout",
           "moe_layout_src", "moe_route_limited", "moe_bias_update",
           "moe_layout_remote_first", "moe_route_round_robin",
           "moe_route_layout", "moe_route_layout_dispatch",
           "moe_dispatch", "moe_combine", "moe_get_device_error", "moe_check",
           "moe_layout_rows", "moe_workspace_bytes"]


@dataclasses.dataclass(frozen=True)
class MoeShape:
    tokens: int
    hidden: int
    experts: int
    k: int
    ranks: int
    capacity: int = 0
    align: int = 1
    renorm: bool = True
    fp8: bool = False
    src_layout: bool = False  # rows follow the per-source-rank layout (moe_layout_src)

    @property
    def flags(self) -> int:
        return ((MOE_F_RENORM if self.renorm else 0) | (MOE_F_FP8 if self.fp8 else 0)
                | (MOE_F_SRC_LAYOUT if self.src_layout else 0))

    def c(self) -> _binding.MoeShapeC:
        return _binding.MoeShapeC(self.tokens, self.hidden, self.experts, self.k, self.ranks,
                                  self.capacity, self.align, self.flags)

    @property
    def rows(self) -> int:
        return moe_layout_rows(self)


def moe_layout_rows(shape: MoeShape) -> int:
    n = _binding.lib().moe_layout_rows(ctypes.byref(shape.c()))
    if n < 0:
        raise MoeError(_binding.MOE_ERR_INVALID_ARG, "moe_layout_rows")
    return int(n)


def moe_workspace_bytes(shape: MoeShape) -> int:
    n = _binding.lib().moe_workspace_bytes(ctypes.byref(shape.c()))
    if n == 0:
        raise MoeError(_binding.MOE_ERR_INVALID_ARG, "moe_workspace_bytes")
    return int(n)


def _stream(device=None) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None, shape=None) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


def _check(status: int, what: str):
    if status != _binding.MOE_OK:
        raise MoeError(status, what)


class Workspace:
    """Zero-filled device workspace for the calls of `shape` (or any shape whose
    requirement is not larger)."""

    def __init__(self, shape: MoeShape, device=None):
        self.nbytes = moe_workspace_bytes(shape)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8,
                               device=device if device is not None else "cuda")
        _check(_binding.lib().moe_workspace_init(self.buf.data_ptr(), self.nbytes,
                                                 _stream(self.buf.device)),
               "moe_workspace_init")

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()


@dataclasses.dataclass
class Layout:
    counts: torch.Tensor       # int32 [E]
    expert_off: torch.Tensor   # int32 [E+1]
    rank_off: torch.Tensor     # int32 [R+1]
    rank_counts: torch.Tensor  # int32 [R]
    dst_pos: torch.Tensor      # int32 [T,k]
    src_idx: torch.Tensor      # int32 [N]


def moe_route(shape: MoeShape, logits: torch.Tensor, bias: Optional[torch.Tensor] = None, *,
              ws: Workspace, ids: Optional[torch.Tensor] = None,
              gates: Optional[torch.Tensor] = None):
    T, E, k = shape.tokens, shape.experts, shape.k
    dev = logits.device
    if ids is None:
        ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    if gates is None:
        gates = torch.empty((T, k), dtype=torch.float32, device=dev)
    st = _binding.lib().moe_route(
        ctypes.byref(shape.c()), _ptr(logits, "logits", torch.float32, (T, E)),
        _ptr(bias, "bias", torch.float32, (E,)), _ptr(ids, "ids", torch.int32, (T, k)),
        _ptr(gates, "gates", torch.float32, (T, k)), ws.ptr, ws.nbytes, _stream(dev))
    _check(st, "moe_route")
    return ids, gates


def moe_route_limited(shape: MoeShape, logits: torch.Tensor, max_ranks: int,
                      bias: Optional[torch.Tensor] = None, *, ws: Workspace,
                      ids: Optional[torch.Tensor] = None, gates: Optional[torch.Tensor] = None):
    """moe_route with each token's experts taken from at most `max_ranks` ranks."""
    T, E, k = shape.tokens, shape.experts, shape.k
    dev = logits.device
    if ids is None:
        ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    if gates is None:
        gates = torch.empty((T, k), dtype=torch.float32, device=dev)
    st = _binding.lib().moe_route_limited(
        ctypes.byref(shape.c()), _ptr(logits, "logits", torch.float32, (T, E)),
        _ptr(bias, "bias", torch.float32, (E,)), int(max_ranks),
        _ptr(ids, "ids", torch.int32, (T, k)), _ptr(gates, "gates", torch.float32, (T, k)),
        ws.ptr, ws.nbytes, _stream(dev))
    _check(st, "moe_route_limited")
    return ids, gates


def moe_layout_remote_first(shape: MoeShape, ids: torch.Tensor, home_rank: int, *,
                            ws: Workspace, out: Optional[Layout] = None,
                            tile_expert: Optional[torch.Tensor] = None):
    """Layout with the rank slices ordered home+1, ..., home (remote first);
    returns (Layout, tile_expert int32 [N/align])."""
    T, E, k, R = shape.tokens, shape.experts, shape.k, shape.ranks
    N = shape.rows
    dev = ids.device
    i32 = dict(dtype=torch.int32, device=dev)
    if out is None:
        out = Layout(torch.empty(E, **i32), torch.empty(E + 1, **i32), torch.empty(R + 1, **i32),
                     torch.empty(R, **i32), torch.empty((T, k), **i32), torch.empty(N, **i32))
    if tile_expert is None:
        tile_expert = torch.empty(N // shape.align, **i32)
    st = _binding.lib().moe_layout_remote_first(
        ctypes.byref(shape.c()), _ptr(ids, "ids", torch.int32, (T, k)), int(home_rank),
        _ptr(out.counts, "counts", torch.int32, (E,)),
        _ptr(out.expert_off, "expert_off", torch.int32, (E + 1,)),
        _ptr(out.rank_off, "rank_off", torch.int32, (R + 1,)),
        _ptr(out.rank_counts, "rank_counts", torch.int32, (R,)),
        _ptr(out.dst_pos, "dst_pos", torch.int32, (T, k)),
        _ptr(out.src_idx, "src_idx", torch.int32, (N,)),
        _ptr(tile_expert, "tile_expert", torch.int32, (N // shape.align,)),
        ws.ptr, ws.nbytes, _stream(dev))
    _check(st, "moe_layout_remote_first")
    return out, tile_expert


def moe_route_round_robin(shape: MoeShape, *, device=None, ids: Optional[torch.Tensor] = None,
                          gates: Optional[torch.Tensor] = None):
    """The round-robin router: ids[t,j] = (t*k + j) mod E, gates 1/k."""
    T, k = shape.tokens, shape.k
    dev = device if device is not None else (ids.device if ids is not None else "cuda")
    if ids is None:
        ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    if gates is None:
        gates = torch.empty((T, k), dtype=torch.float32, device=ids.device)
    st = _binding.lib().moe_route_round_robin(
        ctypes.byref(shape.c()), _ptr(ids, "ids", torch.int32, (T, k)),
        _ptr(gates, "gates", torch.float32, (T, k)), _stream(ids.device))
    _check(st, "moe_route_round_robin")
    return ids, gates


def moe_bias_update(shape: MoeShape, counts: torch.Tensor, gamma: float,
                    bias: torch.Tensor) -> torch.Tensor:
    """bias[e] += gamma * sign(T*k/E - counts[e]), in place; returns bias."""
    E = shape.experts
    st = _binding.lib().moe_bias_update(
        ctypes.byref(shape.c()), _ptr(counts, "counts", torch.int32, (E,)), float(gamma),
        _ptr(bias, "bias", torch.float32, (E,)), _stream(bias.device))
    _check(st, "moe_bias_update")
    return bias


def moe_layout(shape: MoeShape, ids: torch.Tensor, *, ws: Workspace,
               out: Optional[Layout] = None) -> Layout:
    T, E, k, R = shape.tokens, shape.experts, shape.k, shape.ranks
    N = shape.rows
    dev = ids.device
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        out = Layout(torch.empty(E, **i32), torch.empty(E + 1, **i32), torch.empty(R + 1, **i32),
                     torch.empty(R, **i32), torch.empty((T, k), **i32), torch.empty(N, **i32))
    st = _binding.lib().moe_layout(
        ctypes.byref(shape.c()), _ptr(ids, "ids", torch.int32, (T, k)),
        _ptr(out.counts, "counts", torch.int32, (E,)),
        _ptr(out.expert_off, "expert_off", torch.int32, (E + 1,)),
        _ptr(out.rank_off, "rank_off", torch.int32, (R + 1,)),
        _ptr(out.rank_counts, "rank_counts", torch.int32, (R,)),
        _ptr(out.dst_pos, "dst_pos", torch.int32, (T, k)),
        _ptr(out.src_idx, "src_idx", torch.int32, (N,)), ws.ptr, ws.nbytes, _stream(dev))
    _check(st, "moe_layout")
    return out


@dataclasses.dataclass
class LayoutSrc:
    src_counts: torch.Tensor   # int32 [R,E]   per (source shard, expert)
    seg_off: torch.Tensor      # int32 [R*E+1] segments in (rank, shard, expert) order
    pair_counts: torch.Tensor  # int32 [R,R]   [source shard][destination rank]
    rank_off: torch.Tensor     # int32 [R+1]
    rank_counts: torch.Tensor  # int32 [R]
    dst_pos: torch.Tensor      # int32 [T,k]
    src_idx: torch.Tensor      # int32 [N]


def moe_layout_src(shape: MoeShape, ids: torch.Tensor, *, ws: Workspace,
                   out: Optional[LayoutSrc] = None) -> LayoutSrc:
    """Per-source-rank layout (shape.src_layout must be set)."""
    T, E, k, R = shape.tokens, shape.experts, shape.k, shape.ranks
    N = shape.rows
    dev = ids.device
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        out = LayoutSrc(torch.empty((R, E), **i32), torch.empty(R * E + 1, **i32),
                        torch.empty((R, R), **i32), torch.empty(R + 1, **i32),
                        torch.empty(R, **i32), torch.empty((T, k), **i32),
                        torch.empty(N, **i32))
    st = _binding.lib().moe_layout_src(
        ctypes.byref(shape.c()), _ptr(ids, "ids", torch.int32, (T, k)),
        _ptr(out.src_counts, "src_counts", torch.int32, (R, E)),
        _ptr(out.seg_off, "seg_off", torch.int32, (R * E + 1,)),
        _ptr(out.pair_counts, "pair_counts", torch.int32, (R, R)),
        _ptr(out.rank_off, "rank_off", torch.int32, (R + 1,)),
        _ptr(out.rank_counts, "rank_counts", torch.int32, (R,)),
        _ptr(out.dst_pos, "dst_pos", torch.int32, (T, k)),
        _ptr(out.src_idx, "src_idx", torch.int32, (N,)), ws.ptr, ws.nbytes, _stream(dev))
    _check(st, "moe_layout_src")
    return out


def moe_route_layout(shape: MoeShape, logits: torch.Tensor, bias: Optional[torch.Tensor] = None,
                     *, ws: Workspace, ids: Optional[torch.Tensor] = None,
                     gates: Optional[torch.Tensor] = None, out: Optional[Layout] = None):
    """moe_route then moe_layout in one launch; returns (ids, gates, Layout)."""
    T, E, k, R = shape.tokens, shape.experts, shape.k, shape.ranks
    N = shape.rows
    dev = logits.device
    i32 = dict(dtype=torch.int32, device=dev)
    if ids is None:
        ids = torch.empty((T, k), **i32)
    if gates is None:
        gates = torch.empty((T, k), dtype=torch.float32, device=dev)
    if out is None:
        out = Layout(torch.empty(E, **i32), torch.empty(E + 1, **i32), torch.empty(R + 1, **i32),
                     torch.empty(R, **i32), torch.empty((T, k), **i32), torch.empty(N, **i32))
    st = _binding.lib().moe_route_layout(
        ctypes.byref(shape.c()), _ptr(logits, "logits", torch.float32, (T, E)),
        _ptr(bias, "bias", torch.float32, (E,)), _ptr(ids, "ids", torch.int32, (T, k)),
        _ptr(gates, "gates", torch.float32, (T, k)),
        _ptr(out.counts, "counts", torch.int32, (E,)),
        _ptr(out.expert_off, "expert_off", torch.int32, (E + 1,)),
        _ptr(out.rank_off, "rank_off", torch.int32, (R + 1,)),
        _ptr(out.rank_counts, "rank_counts", torch.int32, (R,)),
        _ptr(out.dst_pos, "dst_pos", torch.int32, (T, k)),
        _ptr(out.src_idx, "src_idx", torch.int32, (N,)), ws.ptr, ws.nbytes, _stream(dev))
    _check(st, "moe_route_layout")
    return ids, gates, out


def _dispatch_out(shape: MoeShape, dev, out, scales):
    N, H = shape.rows, shape.hidden
    if shape.fp8:
        if out is None:
            out = torch.empty((N, H), dtype=torch.float8_e4m3fn, device=dev)
        if scales is None:
            scales = torch.empty((N, H // 128), dtype=torch.float32, device=dev)
        return out, scales, _ptr(out, "out", torch.float8_e4m3fn, (N, H)), \
            _ptr(scales, "scales", torch.float32, (N, H // 128))
    if out is None:
        out = torch.empty((N, H), dtype=torch.bfloat16, device=dev)
    return out, None, _ptr(out, "out", torch.bfloat16, (N, H)), None


def moe_route_layout_dispatch(shape: MoeShape, logits: torch.Tensor, x: torch.Tensor,
                              bias: Optional[torch.Tensor] = None, *, ws: Workspace,
                              ids: Optional[torch.Tensor] = None,
                              gates: Optional[torch.Tensor] = None, lay: Optional[Layout] = None,
                              out: Optional[torch.Tensor] = None,
                              scales: Optional[torch.Tensor] = None):
    """Steps 1-4 in one call.  Returns (ids, gates, Layout, dispatched) where
    dispatched is as moe_dispatch returns it."""
    T, E, k, R, H = shape.tokens, shape.experts, shape.k, shape.ranks, shape.hidden
    N = shape.rows
    dev = logits.device
    i32 = dict(dtype=torch.int32, device=dev)
    if ids is None:
        ids = torch.empty((T, k), **i32)
    if gates is None:
        gates = torch.empty((T, k), dtype=torch.float32, device=dev)
    if lay is None:
        lay = Layout(torch.empty(E, **i32), torch.empty(E + 1, **i32), torch.empty(R + 1, **i32),
                     torch.empty(R, **i32), torch.empty((T, k), **i32), torch.empty(N, **i32))
    out, scales, optr, sptr = _dispatch_out(shape, dev, out, scales)
    st = _binding.lib().moe_route_layout_dispatch(
        ctypes.byref(shape.c()), _ptr(logits, "logits", torch.float32, (T, E)),
        _ptr(bias, "bias", torch.float32, (E,)), _ptr(x, "x", torch.bfloat16, (T, H)),
        _ptr(ids, "ids", torch.int32, (T, k)), _ptr(gates, "gates", torch.float32, (T, k)),
        _ptr(lay.counts, "counts", torch.int32, (E,)),
        _ptr(lay.expert_off, "expert_off", torch.int32, (E + 1,)),
        _ptr(lay.rank_off, "rank_off", torch.int32, (R + 1,)),
        _ptr(lay.rank_counts, "rank_counts", torch.int32, (R,)),
        _ptr(lay.dst_pos, "dst_pos", torch.int32, (T, k)),
        _ptr(lay.src_idx, "src_idx", torch.int32, (N,)), optr, sptr, ws.ptr, ws.nbytes,
        _stream(dev))
    _check(st, "moe_route_layout_dispatch")
    return ids, gates, lay, ((out, scales) if shape.fp8 else out)


def moe_dispatch(shape: MoeShape, x: torch.Tensor, dst_pos: torch.Tensor, *, ws: Workspace,
                 out: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None):
    """bf16: returns out [N,H] bf16.  FP8: returns (codes [N,H] float8_e4m3fn,
    scales [N,H/128] fp32).  Rows no assignment maps to are left as allocated."""
    T, H, k = shape.tokens, shape.hidden, shape.k
    N = shape.rows
    dev = x.device
    if shape.fp8:
        if out is None:
            out = torch.empty((N, H), dtype=torch.float8_e4m3fn, device=dev)
        if scales is None:
            scales = torch.empty((N, H // 128), dtype=torch.float32, device=dev)
        optr = _ptr(out, "out", torch.float8_e4m3fn, (N, H))
        sptr = _ptr(scales, "scales", torch.float32, (N, H // 128))
    else:
        if out is None:
            out = torch.empty((N, H), dtype=torch.bfloat16, device=dev)
        optr = _ptr(out, "out", torch.bfloat16, (N, H))
        sptr = None
    st = _binding.lib().moe_dispatch(
        ctypes.byref(shape.c()), _ptr(x, "x", torch.bfloat16, (T, H)),
        _ptr(dst_pos, "dst_pos", torch.int32, (T, k)), optr, sptr, ws.ptr, ws.nbytes,
        _stream(dev))
    _check(st, "moe_dispatch")
    return (out, scales) if shape.fp8 else out


def moe_combine(shape: MoeShape, y: torch.Tensor, dst_pos: torch.Tensor, gates: torch.Tensor, *,
                ws: Workspace, shared: Optional[torch.Tensor] = None,
                residual: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None) -> torch.Tensor:
    T, H, k = shape.tokens, shape.hidden, shape.k
    N = shape.rows
    dev = y.device
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    st = _binding.lib().moe_combine(
        ctypes.byref(shape.c()), _ptr(y, "y", torch.bfloat16, (N, H)),
        _ptr(dst_pos, "dst_pos", torch.int32, (T, k)),
        _ptr(gates, "gates", torch.float32, (T, k)),
        _ptr(shared, "shared", torch.bfloat16, (T, H)),
        _ptr(residual, "residual", torch.bfloat16, (T, H)),
        _ptr(out, "out", torch.bfloat16, (T, H)), ws.ptr, ws.nbytes, _stream(dev))
    _check(st, "moe_combine")
    return out


def moe_get_device_error(ws: Workspace):
    """Synchronise the current stream; return (status, detail) of the first
    device-side error since the last read, and clear it."""
    detail = ctypes.c_int32(0)
    st = _binding.lib().moe_get_device_error(ws.ptr, ctypes.byref(detail),
                                             _stream(ws.buf.device))
    return int(st), int(detail.value)


def moe_check(ws: Workspace):
    st, detail = moe_get_device_error(ws)
    if st != _binding.MOE_OK:
        raise MoeError(st, "device", detail)
