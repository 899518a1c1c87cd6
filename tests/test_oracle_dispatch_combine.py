"""Pins for the oracle's dispatch (bf16 copy, FP8 quantisation) and combine
("GPU MoE all-to-all", section "Two collectives per layer": k copies out,
inverse permutation back, scaled by the router's gate weights; section
"Latency-bound at decode, bandwidth-bound at prefill": lower-precision
dispatch; "MoE All-to-All Dispatch and Ragged Routing", section "Returning
Tokens to the Original GPU": residual x + dx)."""
import math

import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_07_b200.workloads import bf16_bits, bits_to_bf16
from conftest import read_golden


def _bf16_rand(shape, rng, scale=1.0):
    x = torch.from_numpy((rng.standard_normal(shape) * scale).astype(np.float32))
    return bf16_bits(x.to(torch.bfloat16))


def _bits_to_f64(b):
    return bits_to_bf16(b).to(torch.float64).numpy()


def _ids(T, E, k, rng):
    return np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)


def test_dispatch_bf16_is_index_select():
    rng = np.random.default_rng(11)
    T, H, E, R, k = 40, 24, 8, 2, 3
    x = _bf16_rand((T, H), rng)
    L = oracle.layout(_ids(T, E, k, rng), E, R)
    out = oracle.dispatch_bf16(x, L["dst_pos"], T * k)
    ref = x[L["src_idx"] // k]          # library gather: row p <- token src/k
    assert np.array_equal(out, ref)


def test_dispatch_bf16_capacity_leaves_empty_rows():
    rng = np.random.default_rng(12)
    T, H, E, R, k, C = 30, 8, 4, 2, 2, 5
    x = _bf16_rand((T, H), rng)
    L = oracle.layout(_ids(T, E, k, rng), E, R, capacity=C)
    out = oracle.dispatch_bf16(x, L["dst_pos"], E * C)
    src = L["src_idx"]
    assert np.array_equal(out[src >= 0], x[src[src >= 0] // k])
    assert np.all(out[src < 0] == 0)


def test_quantize_row_matches_torch_recipe():
    # Library special case: torch's fp32 division for 448/amax and amax/448, an
    # fp32 multiply and torch's float8_e4m3fn cast (nearest-even; inputs stay
    # within +-448 so its non-saturating cast agrees with satfinite).
    rng = np.random.default_rng(13)
    H = 512
    for trial in range(20):
        x = _bf16_rand((H,), rng, scale=10.0 ** rng.integers(-3, 3))
        q, s = oracle.quantize_row_fp8(x)
        xf = bits_to_bf16(x).to(torch.float32).view(H // 128, 128)
        amax = xf.abs().amax(dim=1, keepdim=True)
        inv = torch.tensor(448.0, dtype=torch.float32) / amax
        scaled = xf * inv
        assert float(scaled.abs().max()) <= 448.0 * (1 + 2 ** -22)
        scaled = scaled.clamp(-448.0, 448.0)
        qref = scaled.to(torch.float8_e4m3fn).view(torch.uint8).reshape(-1).numpy()
        sref = (amax / torch.tensor(448.0)).reshape(-1).numpy()
        assert np.array_equal(q, qref)
        assert np.array_equal(s, sref)


def test_quantize_row_invariants():
    rng = np.random.default_rng(14)
    H = 256
    x = _bf16_rand((H,), rng)
    x[128:] = 0            # second block all zero
    q, s = oracle.quantize_row_fp8(x)
    assert s[1] == 0 and np.all(q[128:] == 0)
    xf = _bits_to_f64(x)
    blk = xf[:128]
    i = int(np.argmax(np.abs(blk)))
    assert q[i] & 0x7F == 0x7E              # the block's amax maps to 448
    deq = np.array([oracle.e4m3_decode(c) for c in q[:128]]) * float(s[0])
    # error bound: half an e4m3 quantum of the scaled value (relative 2^-4,
    # absolute 2^-10 in the subnormal range), times the scale
    scaled = np.abs(blk) * 448.0 / float(np.abs(blk).max())
    bound = np.maximum(scaled * 2.0 ** -4, 2.0 ** -10) * float(s[0]) * (1 + 1e-6)
    assert np.all(np.abs(deq - blk) <= bound + 1e-12)


def test_dispatch_fp8_copies_codes_to_every_slot():
    rng = np.random.default_rng(15)
    T, H, E, R, k = 12, 256, 8, 4, 3
    x = _bf16_rand((T, H), rng)
    L = oracle.layout(_ids(T, E, k, rng), E, R)
    q, s = oracle.dispatch_fp8(x, L["dst_pos"], T * k)
    for t in range(T):
        qr, sr = oracle.quantize_row_fp8(x[t])
        for j in range(k):
            p = L["dst_pos"][t, j]
            assert np.array_equal(q[p], qr) and np.array_equal(s[p], sr)


def test_combine_identity_experts_returns_input_exactly():
    rng = np.random.default_rng(16)
    T, H, E, R, k = 50, 16, 16, 4, 6
    x = _bf16_rand((T, H), rng)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    ids, gates = oracle.route(logits, k)
    L = oracle.layout(ids, E, R)
    y = oracle.dispatch_bf16(x, L["dst_pos"], T * k)
    out = oracle.combine(y, L["dst_pos"], gates, T)
    assert np.array_equal(_bits_to_f64(out), _bits_to_f64(x))
    # + residual: x * sum(g) + x == 2x exactly
    out2 = oracle.combine(y, L["dst_pos"], gates, T, residual_bits=x)
    assert np.array_equal(_bits_to_f64(out2), 2 * _bits_to_f64(x))


def test_combine_is_nearest_bf16_of_exact_sum():
    rng = np.random.default_rng(17)
    T, H, E, R, k = 40, 32, 8, 2, 4
    x = _bf16_rand((T, H), rng)
    y = _bf16_rand((T * k, H), rng)
    sh = _bf16_rand((T, H), rng)
    ids = _ids(T, E, k, rng)
    gates = rng.random((T, k)).astype(np.float32)
    L = oracle.layout(ids, E, R)
    out = oracle.combine(y, L["dst_pos"], gates, T, shared_bits=sh, residual_bits=x)
    # numpy fp64 sum of the same terms (exact products, tiny summation error)
    yf = _bits_to_f64(y)
    exact = np.einsum("tk,tkh->th", gates.astype(np.float64), yf[L["dst_pos"]])
    exact += _bits_to_f64(sh) + _bits_to_f64(x)
    got = _bits_to_f64(out)
    # nearest bf16: |got - exact| <= half a bf16 quantum of exact
    quantum = 2.0 ** (np.floor(np.log2(np.abs(exact) + 1e-300)) - 7)
    assert np.all(np.abs(got - exact) <= 0.5 * quantum * (1 + 1e-9))


def test_combine_drops_contribute_nothing():
    T, H, E, R, k, C = 6, 8, 2, 1, 2, 2
    ids = np.tile(np.array([0, 1], np.int32), (T, 1))  # every token picks both
    rng = np.random.default_rng(18)
    x = _bf16_rand((T, H), rng)
    gates = np.full((T, k), 0.5, np.float32)
    L = oracle.layout(ids, E, R, capacity=C)
    y = oracle.dispatch_bf16(x, L["dst_pos"], E * C)
    out = oracle.combine(y, L["dst_pos"], gates, T, residual_bits=x)
    xf = _bits_to_f64(x)
    got = _bits_to_f64(out)
    # tokens 0,1 kept both slots: 0.5x + 0.5x + x = 2x; others dropped both: x
    assert np.array_equal(got[:2], 2 * xf[:2])
    assert np.array_equal(got[2:], xf[2:])
    out0 = oracle.combine(y, L["dst_pos"], gates, T)
    assert np.all(_bits_to_f64(out0)[2:] == 0)


def test_combine_token_subset_matches_full():
    rng = np.random.default_rng(19)
    T, H, E, R, k = 30, 16, 8, 2, 2
    x = _bf16_rand((T, H), rng)
    ids = _ids(T, E, k, rng)
    gates = rng.random((T, k)).astype(np.float32)
    L = oracle.layout(ids, E, R)
    y = _bf16_rand((T * k, H), rng)
    full = oracle.combine(y, L["dst_pos"], gates, T)
    sub = np.array([3, 17, 29], np.int32)
    part = oracle.combine(y, L["dst_pos"], gates, T, tokens=sub)
    assert np.array_equal(part[sub], full[sub])


def test_expert_scale_standin_matches_torch():
    rng = np.random.default_rng(20)
    T, H, E, R, k = 20, 16, 8, 2, 3
    x = _bf16_rand((T, H), rng)
    L = oracle.layout(_ids(T, E, k, rng), E, R)
    xd = oracle.dispatch_bf16(x, L["dst_pos"], T * k)
    y = oracle.expert_scale(xd, L["expert_off"], L["counts"])
    e_of_row = np.repeat(np.arange(E), L["counts"])
    s = (torch.arange(1, E + 1, dtype=torch.float32) / torch.tensor(float(E)))[e_of_row]
    ref = (bits_to_bf16(xd).to(torch.float32) * s[:, None]).to(torch.bfloat16)
    assert np.array_equal(y, bf16_bits(ref))


def test_dequant_standin_matches_torch():
    rng = np.random.default_rng(21)
    q = rng.integers(0, 256, size=(7, 256), dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0  # no NaN codes
    s = (rng.random((7, 2)) * 3).astype(np.float32)
    y = oracle.dequant_fp8(q, s)
    qt = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float32)
    ref = (qt * torch.from_numpy(s).repeat_interleave(128, dim=1)).to(torch.bfloat16)
    assert np.array_equal(y, bf16_bits(ref))


def test_hand_worked_combine():
    g = read_golden("hand_route_layout.txt")
    logits = np.array([[float(v) for v in g["logits_t0"]],
                       [float(v) for v in g["logits_t1"]]], np.float32)
    bias = np.array([float(v) for v in g["bias"]], np.float32)
    x = bf16_bits(torch.tensor([[float(v) for v in g["x_t0"]],
                                [float(v) for v in g["x_t1"]]]).to(torch.bfloat16))
    ids, gates = oracle.route(logits, 2, bias)
    for cap, tag in ((0, "dropless"), (1, "capacity")):
        L = oracle.layout(ids, 4, 2, capacity=cap)
        y = oracle.dispatch_bf16(x, L["dst_pos"], L["src_idx"].shape[0])
        out = _bits_to_f64(oracle.combine(y, L["dst_pos"], gates, 2))
        assert out[0].tolist() == [float(v) for v in g[f"out_{tag}_t0"]]
        assert out[1].tolist() == [float(v) for v in g[f"out_{tag}_t1"]]


# ---- the combine in fixed-order binary32 accumulation (orc_combine_f32) ----

def _one_token_case(g, tag):
    vals = lambda key: [float(v) for v in g[key]]  # noqa: E731
    gates = np.array([vals(f"{tag}_gates")], np.float32)
    y = bf16_bits(torch.tensor(vals(f"{tag}_y"))[:, None].to(torch.bfloat16))
    dst = np.array([[int(v) for v in g[f"{tag}_dst"]]], np.int32)
    extra = {}
    for key in ("shared", "residual"):
        if f"{tag}_{key}" in g:
            extra[f"{key}_bits"] = bf16_bits(torch.tensor([vals(f"{tag}_{key}")]).to(torch.bfloat16))
    return y, dst, gates, extra


@pytest.mark.parametrize("tag", ["c1", "c2", "c3", "c4", "c5"])
def test_hand_worked_combine_accumulation_order(tag):
    """Hand-worked cases where the binary32 order decides the result (a tie
    at 2^24 lost in one slot order and kept in another; shared before
    residual; one rounding per fused multiply-add; a dropped slot)."""
    g = read_golden("hand_combine_f32.txt")
    y, dst, gates, extra = _one_token_case(g, tag)
    f32 = _bits_to_f64(oracle.combine_f32(y, dst, gates, 1, **extra))[0, 0]
    exact = _bits_to_f64(oracle.combine(y, dst, gates, 1, **extra))[0, 0]
    assert f32 == float(g[f"{tag}_f32"][0])
    assert exact == float(g[f"{tag}_exact"][0])


def test_combine_f32_equals_exact_sum_when_every_step_is_exact():
    """Gates that are powers of two and small integer rows keep every binary32
    partial sum exact, so the fixed-order accumulation is the exact sum."""
    rng = np.random.default_rng(31)
    T, H, E, R, k = 64, 32, 16, 4, 6
    x = bf16_bits(torch.from_numpy(rng.integers(-64, 65, (T, H)).astype(np.float32))
                  .to(torch.bfloat16))
    sh = bf16_bits(torch.from_numpy(rng.integers(-64, 65, (T, H)).astype(np.float32))
                   .to(torch.bfloat16))
    y = bf16_bits(torch.from_numpy(rng.integers(-64, 65, (T * k, H)).astype(np.float32))
                  .to(torch.bfloat16))
    gates = (2.0 ** -rng.integers(0, 4, (T, k))).astype(np.float32)
    L = oracle.layout(_ids(T, E, k, rng), E, R)
    for extra in ({}, {"shared_bits": sh}, {"residual_bits": x},
                  {"shared_bits": sh, "residual_bits": x}):
        a = oracle.combine_f32(y, L["dst_pos"], gates, T, **extra)
        b = oracle.combine(y, L["dst_pos"], gates, T, **extra)
        assert np.array_equal(a, b)


def _bf16_quantum(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (np.maximum(e, -126) - 7), 2.0 ** -133)


@pytest.mark.parametrize("case", ["random", "identity_experts", "cancelling"])
def test_combine_f32_within_the_binary32_bound_of_the_exact_sum(case):
    """|out - exact| <= half a bf16 quantum of out + n * 2^-24 * (sum of the
    terms' magnitudes) * (1 + 1e-6), n = roundings (kept slots + shared +
    residual): the standard bound for n binary32 steps.  A dropped term, a
    wrong sign or a wrong row breaks it by orders of magnitude."""
    rng = np.random.default_rng({"random": 41, "identity_experts": 42, "cancelling": 43}[case])
    T, H, E, R, k = 300, 64, 32, 4, 8
    x = _bf16_rand((T, H), rng)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    ids, gates = oracle.route(logits, k)
    L = oracle.layout(ids, E, R)
    if case == "identity_experts":
        y = oracle.dispatch_bf16(x, L["dst_pos"], T * k)
        sh = _bf16_rand((T, H), rng)
    elif case == "cancelling":
        y = oracle.dispatch_bf16(x, L["dst_pos"], T * k)
        # shared = -(2x) up to bf16 rounding: the sum nearly cancels
        sh = bf16_bits((-2.0 * bits_to_bf16(x).to(torch.float32)
                        + torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)) * 1e-3)
                       .to(torch.bfloat16))
    else:
        y = _bf16_rand((T * k, H), rng)
        sh = _bf16_rand((T, H), rng)
    out = _bits_to_f64(oracle.combine_f32(y, L["dst_pos"], gates, T, shared_bits=sh,
                                          residual_bits=x))
    yf = _bits_to_f64(y)[L["dst_pos"]]                # [T,k,H]
    terms = gates.astype(np.float64)[:, :, None] * yf  # exact products
    exact = terms.sum(1) + _bits_to_f64(sh) + _bits_to_f64(x)
    mag = np.abs(terms).sum(1) + np.abs(_bits_to_f64(sh)) + np.abs(_bits_to_f64(x))
    n = k + 2
    allow = 0.5 * _bf16_quantum(out) + n * 2.0 ** -24 * mag * (1 + 1e-6)
    assert np.all(np.abs(out - exact) <= allow)
    # and the bound has teeth: against the exact sum with slot 0 left out, or
    # with the residual counted twice, most values break it
    assert (np.abs(out - (exact - terms[:, 0])) > allow).mean() > 0.9
    assert (np.abs(out - (exact + _bits_to_f64(x))) > allow).mean() > 0.9


def test_combine_f32_identity_experts_return_the_input_exactly():
    """Identity experts with renormalised gates return x, also in the
    fixed-order binary32 accumulation (the gates' sum is 1 to within a few
    2^-24, far inside half a bf16 quantum)."""
    rng = np.random.default_rng(44)
    T, H, E, R, k = 200, 32, 64, 8, 10
    x = _bf16_rand((T, H), rng)
    ids, gates = oracle.route(rng.standard_normal((T, E)).astype(np.float32), k)
    L = oracle.layout(ids, E, R)
    y = oracle.dispatch_bf16(x, L["dst_pos"], T * k)
    out = oracle.combine_f32(y, L["dst_pos"], gates, T)
    assert np.array_equal(_bits_to_f64(out), _bits_to_f64(x))


def test_fp8_recipe_error_reaches_16_of_448_of_the_block_max():
    """The FP8 recipe (per-128-channel scale = amax/448, e4m3 round to nearest
    even) can be off by half an e4m3 step of the top binade: 16/448 (3.57 %)
    of the block's max.  Worked by hand: a block whose max is 448 (scale 1)
    holding 432, the midpoint of the e4m3 values 416 (mantissa 101) and 448
    (mantissa 110), which rounds to the even 448.  Where that block holds the
    tensor's largest value, the error is 3.57 % of max|x| -- above a 2 % of
    max|x| bound against the unquantised rows, which no encoding with these
    scales can meet; the FP8 path is therefore checked against the quantised
    oracle, and against the unquantised rows within this bound."""
    row = np.zeros(128, np.float32)
    row[0], row[1] = 448.0, 432.0
    xb = bf16_bits(torch.from_numpy(row).to(torch.bfloat16))
    q, s = oracle.quantize_row_fp8(xb)
    assert s[0] == np.float32(1.0)
    deq = _bits_to_f64(oracle.dequant_fp8(q[None, :], s[None, :]))[0]
    assert deq[0] == 448.0 and deq[1] == 448.0
    err = abs(deq[1] - 432.0)
    assert err == 16.0 and err / 448.0 > 0.035


def test_fp8_path_within_the_recipe_bound_of_the_unquantised_combine():
    """Identity experts behind the FP8 dispatch: every output is within
    16/448 of its 128-channel block's max (the recipe's rounding) of the
    unquantised path's output, plus the bf16 roundings of the dequantised row
    and of the two outputs."""
    rng = np.random.default_rng(46)
    T, H, E, R, k = 120, 512, 32, 4, 6
    x = _bf16_rand((T, H), rng, scale=2.0)
    ids, gates = oracle.route(rng.standard_normal((T, E)).astype(np.float32), k)
    L = oracle.layout(ids, E, R)
    q, s = oracle.dispatch_fp8(x, L["dst_pos"], T * k)
    y8 = oracle.dequant_fp8(q, s)
    y16 = oracle.dispatch_bf16(x, L["dst_pos"], T * k)
    a = _bits_to_f64(oracle.combine(y8, L["dst_pos"], gates, T, residual_bits=x))
    b = _bits_to_f64(oracle.combine(y16, L["dst_pos"], gates, T, residual_bits=x))
    amax = np.repeat(np.abs(_bits_to_f64(x)).reshape(T, H // 128, 128).max(axis=2), 128, axis=1)
    q = lambda v: 2.0 ** (np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -126))) - 7)  # noqa: E731
    # e4m3 rounding (16/448 of the block's max at worst) + the bf16 rounding of the
    # dequantised row (half a quantum of the block's max) + each output's rounding
    bound = amax * 16.0 / 448.0 + q(amax) + q(a) + q(b)
    assert np.all(np.abs(a - b) <= bound)
