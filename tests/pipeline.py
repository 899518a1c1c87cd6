"""Test helpers: run the CUDA path (through the C ABI binding) and the CPU
oracle on the same seeded inputs, plus comparison helpers.

The expert FFN is outside the path; between dispatch and combine both sides
apply the same stand-in expert (identity, "row of expert e times (e+1)/E", or
FP8 dequantisation).  On the GPU side the stand-in uses plain torch ops; on
the oracle side the oracle's own stand-in functions.
"""
import functools

import numpy as np
import torch

import oracle
from combine_moe_route_07_b200.workloads import (WORKLOADS, Workload, bf16_bits, bits_to_bf16,
                                                 make_inputs)


@functools.lru_cache(maxsize=2)
def _inputs_cached(T, H, E, zipf_s, bias, shared, seed):
    w = Workload("tmp", T=T, H=H, E=E, R=1, k=1, zipf_s=zipf_s, bias=bias, shared=shared,
                 seed=seed)
    return make_inputs(w)


def inputs_for(w: Workload):
    """The workload's seeded inputs.  With a shared expert, `shared` is its own
    draw (taken after x, logits and bias, which therefore do not change), so
    the combine's shared and residual operands are different tensors."""
    return _inputs_cached(w.T, w.H, w.E, w.zipf_s, w.bias, w.shared, w.seed)


def shape_of(w: Workload):
    from combine_moe_route_07_b200 import MoeShape
    return MoeShape(tokens=w.T, hidden=w.H, experts=w.E, k=w.k, ranks=w.R, capacity=w.capacity,
                    align=w.align, renorm=w.renorm, fp8=w.fp8)


# ------------------------------------------------------------- stand-ins ----

def row_expert(expert_off: torch.Tensor, N: int) -> torch.Tensor:
    rows = torch.arange(N, device=expert_off.device, dtype=torch.int32)
    return (torch.searchsorted(expert_off, rows, right=True) - 1).clamp(min=0)


def standin_gpu(w: Workload, dispatched, lay):
    if w.expert == "identity":
        return dispatched
    if w.expert == "scale":
        e = row_expert(lay.expert_off, dispatched.shape[0])
        s = (torch.arange(1, w.E + 1, dtype=torch.float32, device=e.device)
             / torch.tensor(float(w.E), device=e.device))[e]
        return (dispatched.float() * s[:, None]).to(torch.bfloat16)
    if w.expert == "dequant":
        q, sc = dispatched
        return (q.float() * sc.repeat_interleave(128, dim=1)).to(torch.bfloat16)
    raise ValueError(w.expert)


def standin_oracle(w: Workload, disp, L):
    if w.expert == "identity":
        return disp
    if w.expert == "scale":
        return oracle.expert_scale(disp, L["expert_off"], L["counts"], w.capacity)
    if w.expert == "dequant":
        q, s = disp
        return oracle.dequant_fp8(q, s)
    raise ValueError(w.expert)


# ------------------------------------------------------------ the paths ----

def run_gpu(w: Workload, inp, ids=None, gates=None, fused=False):
    """Run route (unless ids/gates are given), layout, dispatch, stand-in and
    combine on cuda:0.  fused=True: route and layout in one moe_route_layout
    call; fused="dispatch": steps 1-4 in one moe_route_layout_dispatch call.
    Returns a dict of CUDA tensors and the workspace."""
    import combine_moe_route_07_b200 as m
    dev = torch.device("cuda:0")
    shape = shape_of(w)
    ws = m.Workspace(shape, dev)
    x = inp.x.to(dev)
    res = {"ws": ws, "x": x}
    disp = None
    if fused == "dispatch":
        logits = inp.logits.to(dev)
        bias = None if inp.bias is None else inp.bias.to(dev)
        ids, gates, lay, disp = m.moe_route_layout_dispatch(shape, logits, x, bias, ws=ws)
    elif fused:
        logits = inp.logits.to(dev)
        bias = None if inp.bias is None else inp.bias.to(dev)
        ids, gates, lay = m.moe_route_layout(shape, logits, bias, ws=ws)
    elif ids is None:
        logits = inp.logits.to(dev)
        bias = None if inp.bias is None else inp.bias.to(dev)
        ids, gates = m.moe_route(shape, logits, bias, ws=ws)
        lay = m.moe_layout(shape, ids, ws=ws)
    else:
        ids = torch.from_numpy(np.ascontiguousarray(ids)).to(dev)
        gates = torch.from_numpy(np.ascontiguousarray(gates)).to(dev)
        lay = m.moe_layout(shape, ids, ws=ws)
    res["ids"], res["gates"] = ids, gates
    res["layout"] = lay
    if disp is None:
        disp = m.moe_dispatch(shape, x, lay.dst_pos, ws=ws)
    res["dispatch"] = disp
    y = standin_gpu(w, disp, lay)
    res["y"] = y
    res["shared"] = inp.shared.to(dev) if w.shared else None
    res["out"] = m.moe_combine(shape, y, lay.dst_pos, gates, ws=ws, shared=res["shared"],
                               residual=x if w.residual else None)
    torch.cuda.synchronize()
    return res


def run_oracle(w: Workload, inp, through="combine"):
    """The oracle's whole path on the host (numpy)."""
    x = bf16_bits(inp.x)
    logits = inp.logits.numpy()
    bias = None if inp.bias is None else inp.bias.numpy()
    ids, gates = oracle.route(logits, w.k, bias, renorm=w.renorm)
    res = {"ids": ids, "gates": gates, "x": x}
    if through == "route":
        return res
    L = oracle.layout(ids, w.E, w.R, capacity=w.capacity, align=w.align)
    res["layout"] = L
    if through == "layout":
        return res
    N = L["src_idx"].shape[0]
    disp = oracle.dispatch_fp8(x, L["dst_pos"], N) if w.fp8 else oracle.dispatch_bf16(
        x, L["dst_pos"], N)
    res["dispatch"] = disp
    y = standin_oracle(w, disp, L)
    res["y"] = y
    res["shared"] = bf16_bits(inp.shared) if w.shared else None
    res.update(oracle_combines(y, L["dst_pos"], gates, w.T, res["shared"],
                               x if w.residual else None))
    return res


def _abs_bits(b):
    return None if b is None else (np.asarray(b) & 0x7FFF).astype(np.uint16)


def oracle_combines(y, dst_pos, gates, T, shared_bits=None, residual_bits=None):
    """The oracle's combine three ways: `out` the exact sum rounded once to
    bf16; `out_f32` the fixed-order binary32 accumulation (slot fmaf's, then
    shared, then residual) rounded once; `mag` the bf16 of the sum of the
    terms' magnitudes (for the binary32 error bound)."""
    return {
        "out": oracle.combine(y, dst_pos, gates, T, shared_bits=shared_bits,
                              residual_bits=residual_bits),
        "out_f32": oracle.combine_f32(y, dst_pos, gates, T, shared_bits=shared_bits,
                                      residual_bits=residual_bits),
        "mag": oracle.combine(_abs_bits(y), dst_pos, np.abs(gates), T,
                              shared_bits=_abs_bits(shared_bits),
                              residual_bits=_abs_bits(residual_bits)),
    }


def oracle_chunk(w: Workload, x_bits, ids, gates, dst_pos, tokens, shared_bits=None):
    """The oracle's dispatch and combine for a subset of tokens, building only
    those tokens' rows.  Assignment (i, j) of the i-th listed token is placed
    in local row i*k + j (its dropped slots nowhere), so the local rows hold
    what the full dispatch writes at dst_pos[tokens[i], j]; the stand-in expert
    then turns them into expert outputs for the combine.  shared_bits: the
    shared-expert output of the whole batch (uint16 [T,H]) when the workload
    has one; the residual is x.  Returns dict(keep [n,k] bool, dispatch (bf16
    rows, or e4m3 codes and scales, local rows), out [n,H] bf16 bits)."""
    tokens = np.asarray(tokens, np.int32)
    n, k = len(tokens), w.k
    xs = x_bits[tokens]
    dp = dst_pos[tokens]
    keep = dp >= 0
    local = np.where(keep, np.arange(n * k, dtype=np.int32).reshape(n, k), -1).astype(np.int32)
    if w.fp8:
        disp = oracle.dispatch_fp8(xs, local, n * k)
        y = oracle.dequant_fp8(*disp)
    else:
        disp = oracle.dispatch_bf16(xs, local, n * k)
        y = disp
        if w.expert == "scale":
            y = _scale_rows(w, y, ids[tokens].reshape(-1).astype(np.int32))
    sh = None
    if w.shared:
        assert shared_bits is not None, "the workload has a shared expert: pass its output"
        sh = shared_bits[tokens]
    res = {"keep": keep, "dispatch": disp}
    res.update(oracle_combines(y, local, gates[tokens], n, sh, xs if w.residual else None))
    if w.fp8:  # the same combine over the unquantised rows, and the recipe's error bound
        y16 = oracle.dispatch_bf16(xs, local, n * k)
        res["out_unquantised"] = oracle.combine(y16, local, gates[tokens], n, shared_bits=sh,
                                                residual_bits=xs if w.residual else None)
        # e4m3 rounding of the scaled value (16/448 of the block's max at worst),
        # plus the bf16 rounding of the dequantised row (half a quantum of it)
        amax = np.repeat(np.abs(bf16_value(xs)).reshape(n, -1, 128).max(axis=2), 128, axis=1)
        res["fp8_bound"] = amax * (16.0 / 448.0) + bf16_quantum(amax)
    return res


def _scale_rows(w, y, e_of_row):
    """oracle.expert_scale on rows whose experts are given one by one."""
    out = y.copy()
    for e in np.unique(e_of_row):
        rows = np.nonzero(e_of_row == e)[0]
        counts = np.zeros(w.E, np.int32)
        counts[e] = len(rows)
        off = np.zeros(w.E + 1, np.int32)
        off[e + 1:] = len(rows)
        out[rows] = oracle.expert_scale(y[rows], off, counts)
    return out


# ------------------------------------------------------------ comparisons --

def to_np(t: torch.Tensor):
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def bf16_ulp_diff(a_bits, b_bits):
    """|ordered(a) - ordered(b)| for bf16 bit patterns (+0 and -0 coincide)."""
    def ordered(v):
        v = v.astype(np.int32)
        mag = v & 0x7FFF
        return np.where(v & 0x8000, -mag, mag)
    return np.abs(ordered(np.asarray(a_bits)) - ordered(np.asarray(b_bits)))


def assert_bf16_close(got_bits, want_bits, ulps=1, what=""):
    d = bf16_ulp_diff(got_bits, want_bits)
    bad = int((d > ulps).sum())
    assert bad == 0, f"{what}: {bad} of {d.size} values differ by more than {ulps} bf16 ulp " \
                     f"(max {int(d.max())})"
    return d


def bf16_value(bits):
    """bf16 bit patterns -> float64 values."""
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_quantum(v):
    """Spacing of the bf16 numbers at |v| (2^-133 at zero and below the
    normal range)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (np.maximum(e, -126) - 7), 2.0 ** -133)


def assert_combine(got_bits, want, k, what, exact_rows=None):
    """The combine tolerance, derived from the arithmetic.  The kernels
    accumulate in binary32 in fixed order (slot FMAs, then shared, then
    residual) and round once to bf16, so they must equal the oracle's
    fixed-order accumulation `out_f32` bit for bit (+0 and -0 alike) on the
    rows in `exact_rows` (all rows by default; the whole-path tests leave out
    tokens whose gates came out one fp32 ulp away from the oracle's).  Every
    value must also lie within one bf16 quantum plus the binary32 bound
    (k+2) * 2^-24 * (sum of the terms' magnitudes) of the exact sum `out`: one
    bf16 ulp wherever the terms do not cancel.  Returns the ulp distance to
    the exact sum."""
    got_bits = np.asarray(got_bits)
    d32 = bf16_ulp_diff(got_bits, want["out_f32"])
    sel = d32 if exact_rows is None else d32[exact_rows]
    bad = int((sel != 0).sum())
    assert bad == 0, f"{what}: {bad} of {sel.size} values differ from the fixed-order binary32 " \
                     f"accumulation (max {int(sel.max())} ulp)"
    g = bf16_value(got_bits)
    e = bf16_value(want["out"])
    mag = bf16_value(want["mag"]) * (1 + 2.0 ** -7)
    allow = np.maximum(bf16_quantum(g), bf16_quantum(e)) + (k + 2) * 2.0 ** -24 * mag * (1 + 1e-6)
    over = int((np.abs(g - e) > allow).sum())
    assert over == 0, f"{what}: {over} values outside the binary32 bound of the exact sum"
    return bf16_ulp_diff(got_bits, want["out"])


def gate_rows_equal(gpu_gates, oracle_gates):
    """Tokens whose gates are bit-identical on both sides."""
    a = np.ascontiguousarray(gpu_gates, np.float32).view(np.uint32)
    b = np.ascontiguousarray(oracle_gates, np.float32).view(np.uint32)
    return (a == b).all(axis=1)


def assert_gates_close(got, want, rel=1e-6, what="gates"):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want) / np.maximum(np.abs(want), 1e-300)
    assert float(err.max(initial=0.0)) <= rel, f"{what}: max relative error {err.max()}"
