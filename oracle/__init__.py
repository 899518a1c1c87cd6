"""CPU oracle for the MoE route / layout / dispatch / combine path.

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  The
product library never calls it and shares no code with it.

Thin numpy wrappers over ``moe_oracle.c``; every rule and its source is stated
in that file's comments.  Arrays are C-contiguous numpy arrays; bf16 values
are carried as their uint16 bit patterns, e4m3 codes as uint8.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        L.orc_route.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp]
        L.orc_route.restype = i32
        L.orc_route_limited.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp, vp]
        L.orc_route_limited.restype = i32
        L.orc_bias_update.argtypes = [i32, i64, vp, ctypes.c_float, vp, vp]
        L.orc_bias_update.restype = None
        L.orc_layout_rows.argtypes = [i32, i32, i32, i32, i32]
        L.orc_layout_rows.restype = i64
        L.orc_layout.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp]
        L.orc_layout.restype = i32
        L.orc_layout_src_rows.argtypes = [i32, i32, i32, i32, i32, i32]
        L.orc_layout_src_rows.restype = i64
        L.orc_layout_src.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp,
                                     vp]
        L.orc_layout_src.restype = i32
        L.orc_layout_remote_first.argtypes = [i32, i32, i32, i32, i32, i32, i32, vp, vp, vp,
                                              vp, vp, vp, vp, vp]
        L.orc_layout_remote_first.restype = i32
        L.orc_route_round_robin.argtypes = [i32, i32, i32, vp, vp]
        L.orc_route_round_robin.restype = None
        L.orc_dispatch_bf16.argtypes = [i32, i32, i32, vp, vp, vp]
        L.orc_dispatch_bf16.restype = None
        L.orc_quantize_row_fp8.argtypes = [i32, vp, vp, vp]
        L.orc_quantize_row_fp8.restype = None
        L.orc_dispatch_fp8.argtypes = [i32, i32, i32, vp, vp, vp, vp]
        L.orc_dispatch_fp8.restype = None
        L.orc_combine.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, i32]
        L.orc_combine.restype = None
        L.orc_combine_f32.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, i32]
        L.orc_combine_f32.restype = None
        L.orc_expert_scale.argtypes = [i32, i32, vp, vp, i32, vp, vp]
        L.orc_expert_scale.restype = None
        L.orc_dequant_fp8.argtypes = [i64, i32, vp, vp, vp]
        L.orc_dequant_fp8.restype = None
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_encode_satfinite.argtypes = [ctypes.c_float]
        L.orc_e4m3_encode_satfinite.restype = ctypes.c_uint8
        L.orc_double_to_bf16.argtypes = [ctypes.c_double]
        L.orc_double_to_bf16.restype = ctypes.c_uint16
        L.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_double.restype = ctypes.c_double
        _lib = L
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


class OracleError(RuntimeError):
    pass


def route(logits, k, bias=None, renorm=True):
    """Top-k expert ids [T,k] int32 and gates [T,k] float32."""
    logits = _c(logits, np.float32)
    T, E = logits.shape
    bias = None if bias is None else _c(bias, np.float32)
    ids = np.empty((T, k), np.int32)
    gates = np.empty((T, k), np.float32)
    rc = lib().orc_route(T, E, k, int(bool(renorm)), _p(logits), _p(bias), _p(ids), _p(gates))
    if rc:
        raise OracleError(f"orc_route status {rc}")
    return ids, gates


def route_limited(logits, k, R, M, bias=None, renorm=True):
    """Rank-limited route: experts from at most M of the R ranks (group score
    = largest key on the rank).  Returns (ids int32 [T,k], gates fp32 [T,k])."""
    logits = _c(logits, np.float32)
    T, E = logits.shape
    b = None if bias is None else _c(bias, np.float32)
    ids = np.empty((T, k), np.int32)
    gates = np.empty((T, k), np.float32)
    rc = lib().orc_route_limited(T, E, k, R, M, 1 if renorm else 0, _p(logits), _p(b), _p(ids),
                                 _p(gates))
    if rc:
        raise OracleError(f"orc_route_limited status {rc}")
    return ids, gates


def bias_update(counts, assignments, gamma, bias):
    """b_e + gamma * sign(assignments/E - counts[e]) (the aux-loss-free
    balancing step); returns the new fp32 bias."""
    counts = _c(counts, np.int32)
    bias = _c(bias, np.float32)
    E = counts.shape[0]
    out = np.empty(E, np.float32)
    lib().orc_bias_update(E, int(assignments), _p(counts), float(gamma), _p(bias), _p(out))
    return out


def layout_rows(T, E, k, capacity=0, align=1):
    return int(lib().orc_layout_rows(T, E, k, capacity, align))


def layout(ids, E, R, capacity=0, align=1):
    """Returns dict(counts, expert_off, rank_off, rank_counts, dst_pos, src_idx)."""
    ids = _c(ids, np.int32)
    T, k = ids.shape
    N = layout_rows(T, E, k, capacity, align)
    out = dict(
        counts=np.empty(E, np.int32),
        expert_off=np.empty(E + 1, np.int32),
        rank_off=np.empty(R + 1, np.int32),
        rank_counts=np.empty(R, np.int32),
        dst_pos=np.empty((T, k), np.int32),
        src_idx=np.empty(N, np.int32),
    )
    rc = lib().orc_layout(T, E, k, R, capacity, align, _p(ids), _p(out["counts"]),
                          _p(out["expert_off"]), _p(out["rank_off"]), _p(out["rank_counts"]),
                          _p(out["dst_pos"]), _p(out["src_idx"]))
    if rc:
        raise OracleError(f"orc_layout status {rc}")
    return out


def layout_src_rows(T, E, k, R, capacity=0, align=1):
    return int(lib().orc_layout_src_rows(T, E, k, R, capacity, align))


def layout_src(ids, E, R, capacity=0, align=1):
    """Per-source-rank layout (rows ordered by destination rank, source shard,
    expert, token).  Returns dict(src_counts [R,E], seg_off [R*E+1],
    pair_counts [R_src,R_dst], rank_off, rank_counts, dst_pos, src_idx)."""
    ids = _c(ids, np.int32)
    T, k = ids.shape
    N = layout_src_rows(T, E, k, R, capacity, align)
    out = dict(
        src_counts=np.empty((R, E), np.int32),
        seg_off=np.empty(R * E + 1, np.int32),
        pair_counts=np.empty((R, R), np.int32),
        rank_off=np.empty(R + 1, np.int32),
        rank_counts=np.empty(R, np.int32),
        dst_pos=np.empty((T, k), np.int32),
        src_idx=np.empty(N, np.int32),
    )
    rc = lib().orc_layout_src(T, E, k, R, capacity, align, _p(ids), _p(out["src_counts"]),
                              _p(out["seg_off"]), _p(out["pair_counts"]), _p(out["rank_off"]),
                              _p(out["rank_counts"]), _p(out["dst_pos"]), _p(out["src_idx"]))
    if rc:
        raise OracleError(f"orc_layout_src status {rc}")
    return out


def layout_remote_first(ids, E, R, home, capacity=0, align=1):
    """Remote-first, tile-aligned layout seen from rank `home`.  Returns the
    orc_layout dict plus tile_expert [N/align]."""
    ids = _c(ids, np.int32)
    T, k = ids.shape
    N = layout_rows(T, E, k, capacity, align)
    out = dict(
        counts=np.empty(E, np.int32),
        expert_off=np.empty(E + 1, np.int32),
        rank_off=np.empty(R + 1, np.int32),
        rank_counts=np.empty(R, np.int32),
        dst_pos=np.empty((T, k), np.int32),
        src_idx=np.empty(N, np.int32),
        tile_expert=np.empty(N // align, np.int32),
    )
    rc = lib().orc_layout_remote_first(T, E, k, R, capacity, align, home, _p(ids),
                                       _p(out["counts"]), _p(out["expert_off"]),
                                       _p(out["rank_off"]), _p(out["rank_counts"]),
                                       _p(out["dst_pos"]), _p(out["src_idx"]),
                                       _p(out["tile_expert"]))
    if rc:
        raise OracleError(f"orc_layout_remote_first status {rc}")
    return out


def route_round_robin(T, E, k):
    ids = np.empty((T, k), np.int32)
    gates = np.empty((T, k), np.float32)
    lib().orc_route_round_robin(T, E, k, _p(ids), _p(gates))
    return ids, gates


def dispatch_bf16(x_bits, dst_pos, N):
    """x_bits uint16 [T,H] -> out uint16 [N,H]; rows nobody writes stay 0."""
    x_bits = _c(x_bits, np.uint16)
    dst_pos = _c(dst_pos, np.int32)
    T, H = x_bits.shape
    k = dst_pos.shape[1]
    out = np.zeros((N, H), np.uint16)
    lib().orc_dispatch_bf16(T, H, k, _p(x_bits), _p(dst_pos), _p(out))
    return out


def quantize_row_fp8(x_row_bits):
    x_row_bits = _c(x_row_bits, np.uint16)
    H = x_row_bits.shape[0]
    q = np.empty(H, np.uint8)
    s = np.empty(H // 128, np.float32)
    lib().orc_quantize_row_fp8(H, _p(x_row_bits), _p(q), _p(s))
    return q, s


def dispatch_fp8(x_bits, dst_pos, N):
    """x_bits uint16 [T,H] -> (codes uint8 [N,H], scales float32 [N,H/128])."""
    x_bits = _c(x_bits, np.uint16)
    dst_pos = _c(dst_pos, np.int32)
    T, H = x_bits.shape
    k = dst_pos.shape[1]
    out = np.zeros((N, H), np.uint8)
    scales = np.zeros((N, H // 128), np.float32)
    lib().orc_dispatch_fp8(T, H, k, _p(x_bits), _p(dst_pos), _p(out), _p(scales))
    return out, scales


def _combine(fn, y_bits, dst_pos, gates, T, shared_bits, residual_bits, tokens):
    y_bits = _c(y_bits, np.uint16)
    dst_pos = _c(dst_pos, np.int32)
    gates = _c(gates, np.float32)
    H = y_bits.shape[1]
    k = dst_pos.shape[1]
    sh = None if shared_bits is None else _c(shared_bits, np.uint16)
    rs = None if residual_bits is None else _c(residual_bits, np.uint16)
    out = np.zeros((T, H), np.uint16)
    tk = None if tokens is None else _c(tokens, np.int32)
    fn(T, H, k, _p(y_bits), _p(dst_pos), _p(gates), _p(sh), _p(rs), _p(out), _p(tk),
       0 if tk is None else int(tk.shape[0]))
    return out


def combine(y_bits, dst_pos, gates, T, shared_bits=None, residual_bits=None, tokens=None):
    """The combine's exact sum (fp64), rounded once to bf16; uint16 [T,H]
    bf16 bits.  With `tokens`, only those rows are computed."""
    return _combine(lib().orc_combine, y_bits, dst_pos, gates, T, shared_bits, residual_bits,
                    tokens)


def combine_f32(y_bits, dst_pos, gates, T, shared_bits=None, residual_bits=None, tokens=None):
    """The combine accumulated in binary32 in fixed order (slot fmaf's, then
    shared, then residual), rounded once to bf16; arguments as combine()."""
    return _combine(lib().orc_combine_f32, y_bits, dst_pos, gates, T, shared_bits,
                    residual_bits, tokens)


def expert_scale(xd_bits, expert_off, counts, capacity=0):
    """Stand-in expert: rows of expert e scaled by (e+1)/E (bf16 bits)."""
    xd_bits = _c(xd_bits, np.uint16)
    expert_off = _c(expert_off, np.int32)
    counts = _c(counts, np.int32)
    E = counts.shape[0]
    H = xd_bits.shape[1]
    y = xd_bits.copy()
    lib().orc_expert_scale(E, H, _p(expert_off), _p(counts), capacity, _p(xd_bits), _p(y))
    return y


def dequant_fp8(q, scales):
    q = _c(q, np.uint8)
    scales = _c(scales, np.float32)
    rows, H = q.shape
    y = np.empty((rows, H), np.uint16)
    lib().orc_dequant_fp8(rows, H, _p(q), _p(scales), _p(y))
    return y


def e4m3_decode(code):
    return lib().orc_e4m3_decode(int(code))


def e4m3_encode(f):
    return int(lib().orc_e4m3_encode_satfinite(float(f)))


def double_to_bf16(v):
    return int(lib().orc_double_to_bf16(float(v)))


def bf16_to_double(b):
    return float(lib().orc_bf16_to_double(int(b)))
