"""A CPU model of the decisions of the float-key top-k (the staged route form
for more than 224 experts), searched for counterexamples against the oracle.

The GPU tests compare the kernel with the oracle on chosen inputs; this file
checks the argument the form rests on, on inputs built to break it (few
distinct values, +0 and -0, infinities, NaN, partial last lanes, any k):

  - at least k keys reach tau (the k-th largest lane maximum, taken on order
    codes whose low 5 bits carry the lane, then lowered to the bottom of its
    32-code bucket), so the top-k are all candidates;
  - when no two candidates among the first k slots share a slot, every slot
    0..k-1 is written (the kernel reads them without a check);
  - whenever the form answers (no NaN, at most 32 candidates, no shared
    slot), its answer is the oracle's.

The model follows the kernel's steps (lane l holds experts l, l+32, ...;
candidates are compacted in ballot-round order; a candidate's slot is the
number of strictly larger values); it shares no code with the kernel or the
oracle."""
import math

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import oracle


def _f32_bits(x):
    return int(np.array([x], np.float32).view(np.uint32)[0])


def _bits_f32(u):
    return float(np.array([u], np.uint32).view(np.float32)[0])


def order_code(x):
    if x == 0.0:
        x = 0.0  # -0 folds onto +0
    u = _f32_bits(x)
    return (~u) & 0xFFFFFFFF if u & 0x80000000 else u | 0x80000000


def code_float(c):
    return _bits_f32(c & 0x7FFFFFFF if c & 0x80000000 else (~c) & 0xFFFFFFFF)


def model_select(row, bias, k):
    """The float-key form's selection, or None where it hands the token to
    the exact form.  Also returns the facts the tests check."""
    E = len(row)
    nk = 1
    while 32 * nk < E:
        nk *= 2
    f32 = np.float32
    keys = [[-math.inf] * nk for _ in range(32)]
    valid = [[False] * nk for _ in range(32)]
    for l in range(32):
        for i in range(nk):
            e = l + 32 * i
            if e < E:
                v = f32(row[e]) if bias is None else f32(f32(row[e]) + f32(bias[e]))
                keys[l][i] = float(v)
                valid[l][i] = True
    if any(math.isnan(v) for l in range(32) for v in keys[l]):
        return None, {"why": "nan"}
    mm = [max(keys[l]) for l in range(32)]
    packed = [(order_code(mm[l]) & ~31 & 0xFFFFFFFF) | (31 - l) for l in range(32)]
    top = 0
    for _ in range(k):
        top = max(packed)
        packed = [0 if p == top else p for p in packed]
    tau = -math.inf if top < 0x00800000 else code_float(top & ~31 & 0xFFFFFFFF)
    cand_lanes = [[i for i in range(nk) if valid[l][i] and keys[l][i] >= tau] for l in range(32)]
    total = sum(len(c) for c in cand_lanes)
    facts = {"total": total}
    if total > 32:
        return None, dict(facts, why="many")
    cv, ce = [], []
    r = 0
    while any(len(c) > r for c in cand_lanes):  # ballot round r: each lane's r-th candidate
        for l in range(32):
            if len(cand_lanes[l]) > r:
                i = cand_lanes[l][r]
                cv.append(keys[l][i])
                ce.append(l + 32 * i)
        r += 1
    slot = {}
    clash = False
    for p, v in enumerate(cv):
        n = sum(1 for w in cv if w > v)
        if n < k:
            if n in slot:
                clash = True
            slot[n] = p
    if clash:
        return None, dict(facts, why="tie")
    facts["filled"] = all(j in slot for j in range(k))
    return [ce[slot[j]] for j in range(k)], facts


def _check_row(row, bias, k):
    lg = np.asarray(row, np.float32)[None, :]
    b = None if bias is None else np.asarray(bias, np.float32)
    sel, facts = model_select(list(lg[0]), None if b is None else list(b), k)
    if facts.get("why") == "nan":
        return facts
    assert facts["total"] >= k, facts
    if sel is not None:
        assert facts["filled"], facts
        ids, _ = oracle.route(lg, k, b)
        assert sel == ids[0].tolist(), (sel, ids[0].tolist())
    return facts


VALUES = [0.0, -0.0, 1.0, -1.0, 0.5, 2.0, 1e-30, -1e-30, math.inf, -math.inf, 3.4e38, -3.4e38]


@settings(max_examples=400, deadline=None)
@given(
    E=st.sampled_from([225, 256, 260, 300, 512, 996, 1024]),
    k=st.integers(1, 32),
    data=st.data(),
)
def test_model_matches_the_oracle_on_few_distinct_values(E, k, data):
    vals = data.draw(st.lists(st.sampled_from(VALUES), min_size=1, max_size=4, unique_by=repr))
    seed = data.draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    row = np.array(vals, np.float32)[rng.integers(len(vals), size=E)]
    if data.draw(st.booleans()):  # a few distinct values on top of the ties
        pos = rng.choice(E, size=min(E, data.draw(st.integers(1, 40))), replace=False)
        row[pos] = rng.standard_normal(len(pos)).astype(np.float32)
    _check_row(list(row), None, k)


@settings(max_examples=400, deadline=None)
@given(
    E=st.sampled_from([225, 256, 260, 512, 1024]),
    k=st.integers(1, 32),
    data=st.data(),
)
def test_model_matches_the_oracle_on_ties_among_few_candidates(E, k, data):
    """Up to 24 keys drawn from a tiny set above a row of distinct lower
    values: equal values inside a candidate set small enough for the form,
    at, above and below slot k."""
    seed = data.draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    row = (-10.0 - rng.random(E)).astype(np.float32)
    top = data.draw(st.lists(st.sampled_from([2.0, 1.0, 0.0, -0.0, math.inf]), min_size=1,
                             max_size=24))
    pos = rng.choice(E, size=len(top), replace=False)
    row[pos] = np.array(top, np.float32)
    _check_row(list(row), None, k)


@settings(max_examples=300, deadline=None)
@given(
    E=st.sampled_from([256, 260, 512, 1024]),
    k=st.integers(1, 32),
    scale=st.sampled_from([1e-3, 1.0, 30.0]),
    seed=st.integers(0, 2**31 - 1),
    use_bias=st.booleans(),
)
def test_model_matches_the_oracle_on_random_rows(E, k, scale, seed, use_bias):
    rng = np.random.default_rng(seed)
    row = (rng.standard_normal(E) * scale).astype(np.float32)
    bias = (rng.random(E) * 0.2 - 0.1).astype(np.float32) if use_bias else None
    facts = _check_row(list(row), None if bias is None else list(bias), k)
    assert "why" not in facts or facts["why"] in ("many", "tie")


def test_model_takes_the_fast_answer_on_typical_rows():
    """On N(0,1) rows of 512 experts with k = 10 the form answers for nearly
    every token (the exact form is the rare path)."""
    rng = np.random.default_rng(0)
    fast = 0
    for _ in range(300):
        row = rng.standard_normal(512).astype(np.float32)
        sel, facts = model_select(list(row), None, 10)
        fast += sel is not None
        _check_row(list(row), None, 10)
    assert fast >= 295


@pytest.mark.parametrize("finite", [0, 1, 9])
def test_model_with_fewer_than_k_finite_lane_maxima(finite):
    """tau is -inf (the truncated code of -inf would read as a NaN), every key
    is a candidate, and the token goes to the exact form."""
    row = [-math.inf] * 512
    for e in range(finite):
        row[e * 32] = float(e)  # all on lane 0
    sel, facts = model_select(row, None, 10)
    assert sel is None and facts["why"] == "many"
