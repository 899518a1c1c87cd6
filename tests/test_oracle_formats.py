"""Pins for the oracle's number formats (bf16 rounding, OCP E4M3 encode/decode).

Each check reaches the oracle from outside its own formula: the OCP table's
printed values, torch's independent conversions, and brute-force nearest-value
search over every representable value.
"""
import math
import struct

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden


def _f32(v):
    return struct.unpack("<f", struct.pack("<f", v))[0]


# ---------------------------------------------------------------- E4M3 ----


def test_e4m3_decode_matches_ocp_table():
    g = read_golden("e4m3_ocp_table.txt")
    for name, (code, val) in g.items():
        got = oracle.e4m3_decode(int(code, 16))
        if val == "nan":
            assert math.isnan(got), name
        else:
            assert got == float(val), name
            assert math.copysign(1.0, got) == math.copysign(1.0, float(val)), name


def test_e4m3_decode_all_codes_match_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle.e4m3_decode(c)
        if math.isnan(ref[c]):
            assert math.isnan(got)
        else:
            assert got == ref[c], hex(c)


def test_e4m3_roundtrip_every_finite_code():
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if math.isnan(v):
            continue
        assert oracle.e4m3_encode(v) == c, hex(c)


def _all_finite_e4m3():
    vals = sorted({oracle.e4m3_decode(c) for c in range(256)} - {float("nan")})
    return np.array([v for v in vals if not math.isnan(v)])


def test_e4m3_encode_is_nearest_even_brute_force():
    table = _all_finite_e4m3()
    rng = np.random.default_rng(1)
    samples = np.concatenate([
        rng.standard_normal(4000) * 50,
        rng.standard_normal(2000) * 0.01,
        (rng.random(1000) - 0.5) * 900,
    ]).astype(np.float32)
    for v in samples:
        if abs(float(v)) >= 448:
            continue
        code = oracle.e4m3_encode(float(v))
        got = oracle.e4m3_decode(code)
        d = np.abs(table - float(v))
        best = d.min()
        assert abs(got - float(v)) == best, v
        ties = table[d == best]
        if len(ties) > 1:  # nearest-even: the tied value with an even mantissa
            assert (code & 1) == 0, v


def test_e4m3_encode_midpoints_round_to_even():
    # 1 + 1/16 lies midway between 1 (M=0, even) and 1.125 (M=1) -> 1
    assert oracle.e4m3_encode(1.0625) == 0x38
    # 1.125 + 1/16 = 1.1875 midway between 1.125 (M=1) and 1.25 (M=2) -> 1.25
    assert oracle.e4m3_encode(1.1875) == 0x3A
    # subnormal midpoint 1.5 * 2^-9 between 2^-9 (M=1) and 2^-8 (M=2) -> 2^-8
    assert oracle.e4m3_encode(1.5 * 2.0 ** -9) == 0x02
    # half the smallest subnormal -> 0 (tie to even zero)
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00


def test_e4m3_encode_saturates_and_keeps_nan():
    assert oracle.e4m3_encode(448.0) == 0x7E
    assert oracle.e4m3_encode(449.0) == 0x7E
    assert oracle.e4m3_encode(1e30) == 0x7E
    assert oracle.e4m3_encode(float("inf")) == 0x7E
    assert oracle.e4m3_encode(-float("inf")) == 0xFE
    assert oracle.e4m3_encode(-500.0) == 0xFE
    assert oracle.e4m3_encode(float("nan")) & 0x7F == 0x7F


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.standard_normal(20000) * 30, rng.standard_normal(5000) * 1e-3])
    v = v.astype(np.float32)
    v = v[np.abs(v) < 448]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(a)) for a in v], np.uint8)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- bf16 ----


def test_float_to_bf16_matches_torch():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(20000), rng.standard_normal(2000) * 1e-38,
                        rng.standard_normal(2000) * 1e37]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.double_to_bf16(float(a)) for a in v], np.uint16)
    assert np.array_equal(got, ref)


def _bf16_val(bits):
    return oracle.bf16_to_double(bits)


def test_double_to_bf16_is_single_nearest_even_rounding():
    # Brute force: the result is no farther from v than either bf16 neighbour,
    # and on an exact tie the mantissa is even.  Values are chosen so that a
    # double -> float -> bf16 double rounding would go wrong.
    rng = np.random.default_rng(4)
    vals = list(rng.standard_normal(3000) * 10)
    one_tie_plus = 1.0 + 2.0 ** -8 + 2.0 ** -40   # just above a bf16 midpoint
    vals += [one_tie_plus, -one_tie_plus, 1.0 + 2.0 ** -8, 3.0 * 2.0 ** -134]
    for v in vals:
        b = oracle.double_to_bf16(v)
        got = _bf16_val(b)
        lo, hi = _bf16_val((b - 1) & 0xFFFF), _bf16_val((b + 1) & 0xFFFF)
        for nb in (lo, hi):
            if math.isfinite(nb) and (nb > 0) == (got > 0):
                assert abs(got - v) <= abs(nb - v), v
                if abs(got - v) == abs(nb - v):
                    assert b & 1 == 0, v
    assert oracle.double_to_bf16(one_tie_plus) == 0x3F81       # up, not to even
    assert oracle.double_to_bf16(1.0 + 2.0 ** -8) == 0x3F80    # exact tie -> even
    assert oracle.double_to_bf16(3.0 * 2.0 ** -134) == 0x0002  # subnormal tie -> even
    assert oracle.double_to_bf16(1e39) == 0x7F80               # overflow -> inf
