"""The float-key top-k for rows staged in shared memory (more than 224
experts, E a multiple of 4) against the oracle.

Lane l of the routing warp holds experts l, l+32, l+64, ... (NK of them, NK
the power of two >= E/32).  The float form takes tau, the k-th largest lane
maximum, ranks at most 32 keys >= tau by value and hands a token to the exact
code form when a key is NaN, more than 32 keys reach tau, or two of the first
k values are equal.  The cases: random keys with and without a bias and in
both gate modes (E with partial last lanes included); equal values at, across
and below slot k; +0 against -0; one NaN token among routed ones;
candidate sets of exactly 32, 33, 55 and more than 64 keys, built from the
lane layout.  Every token is compared with the oracle, through moe_route and
through the fused moe_route_layout (whose route kernel also fills the
layout's tile table)."""
import numpy as np
import pytest
import torch

import oracle
from pipeline import assert_gates_close, to_np

pytestmark = pytest.mark.gpu


def _nk(E):
    nk = 1
    while 32 * nk < E:
        nk *= 2
    return nk


def _route_both(lg, k, bias=None, renorm=True, R=4):
    import combine_moe_route_07_b200 as m
    T, E = lg.shape
    dev = torch.device("cuda:0")
    shape = m.MoeShape(tokens=T, hidden=16, experts=E, k=k, ranks=R, renorm=renorm)
    ws = m.Workspace(shape, dev)
    lgd = torch.from_numpy(np.ascontiguousarray(lg)).to(dev)
    bd = None if bias is None else torch.from_numpy(bias).to(dev)
    ids, gates = m.moe_route(shape, lgd, bd, ws=ws)
    torch.cuda.synchronize()
    err1 = m.moe_get_device_error(ws)
    ids2, gates2, _ = m.moe_route_layout(shape, lgd, bd, ws=ws)
    torch.cuda.synchronize()
    err2 = m.moe_get_device_error(ws)
    return [(to_np(ids), to_np(gates), err1), (to_np(ids2), to_np(gates2), err2)]


def _check(lg, k, bias=None, renorm=True):
    ids_o, gates_o = oracle.route(lg, k, bias, renorm=renorm)
    for ids, gates, err in _route_both(lg, k, bias, renorm):
        assert err == (0, 0)
        assert np.array_equal(ids, ids_o)
        assert_gates_close(gates, gates_o)


@pytest.mark.parametrize("E", [256, 260, 512, 996, 1024])
@pytest.mark.parametrize("k", [1, 10, 32])
def test_random_keys(E, k):
    rng = np.random.default_rng(E * 100 + k)
    T = 3000
    lg = rng.standard_normal((T, E)).astype(np.float32)
    for use_bias in (False, True):
        bias = (rng.random(E) * 0.2 - 0.1).astype(np.float32) if use_bias else None
        for renorm in (True, False):
            _check(lg, k, bias, renorm)


def _sorted_row(rng, E):
    """A row of distinct values, and its experts in descending order."""
    row = rng.permutation(E).astype(np.float32) / 8.0 - E / 16.0
    return row, np.argsort(-row, kind="stable")


@pytest.mark.parametrize("E,k", [(256, 8), (512, 10), (1024, 32)])
def test_equal_values_at_and_around_slot_k(E, k):
    """Rows with two equal values at slots (p, p+1): both below k (exact form),
    straddling k-1 and k (exact form, the lower id wins the last slot) and at
    or beyond k (no effect on the result)."""
    rng = np.random.default_rng(E + k)
    places = [0, k // 2, k - 2, k - 1, k, k + 3]
    places = [p for p in places if 0 <= p and p + 1 < E]
    T = 400 * len(places)
    lg = np.empty((T, E), np.float32)
    for t in range(T):
        row, order = _sorted_row(rng, E)
        p = places[t % len(places)]
        row[order[p + 1]] = row[order[p]]
        lg[t] = row
    _check(lg, k)


def test_plus_and_minus_zero_are_equal_keys():
    """The k-th and (k+1)-th largest keys are +0 and -0 (either order of ids):
    they tie, and the lower expert id takes the last slot."""
    rng = np.random.default_rng(5)
    E, k, T = 512, 10, 600
    lg = np.empty((T, E), np.float32)
    for t in range(T):
        row = -1.0 - rng.random(E).astype(np.float32)  # all negative
        top = rng.choice(E, size=k + 1, replace=False)
        row[top[: k - 1]] = 1.0 + rng.random(k - 1).astype(np.float32)
        row[top[k - 1]] = 0.0 if t % 2 else -0.0
        row[top[k]] = -0.0 if t % 2 else 0.0
        lg[t] = row
    _check(lg, k)


@pytest.mark.parametrize("e_nan", [0, 15, 77, 79, 236, 511])
def test_a_nan_token_is_reported_and_the_others_are_exact(e_nan):
    """One NaN key, at experts that fall on different places of a lane's
    keys (first, last, middle of a 16-byte chunk, under every rotation)."""
    from combine_moe_route_07_b200._binding import MOE_ERR_DEVICE_NAN
    rng = np.random.default_rng(9 + e_nan)
    E, k, T = 512, 10, 3000
    lg = rng.standard_normal((T, E)).astype(np.float32)
    clean = lg.copy()
    lg[1234, e_nan] = np.nan
    ids_o, gates_o = oracle.route(clean, k)
    keep = np.setdiff1d(np.arange(T), [1234])
    for ids, gates, err in _route_both(lg, k):
        assert err == (MOE_ERR_DEVICE_NAN, 1234)
        assert np.array_equal(ids[keep], ids_o[keep])
        assert_gates_close(gates[keep], gates_o[keep])


def _lane_rows(rng, E, k, full_lanes, partial_keys):
    """Rows whose candidate count is set by the lane layout (lane L holds
    experts L, L+32, ...): `full_lanes` lanes with every key in (101, 200),
    one lane with `partial_keys` keys there, and single keys in (150, 200) on
    further lanes, up to k-1 lanes with a large maximum; the k-th lane
    maximum (tau) is 100.5 on one more lane, so every large key is a
    candidate.  All other keys are in (-2, -1)."""
    nk = _nk(E)
    lanes = rng.permutation(32)
    row = (-1.0 - rng.random(E)).astype(np.float32)
    keys = lambda L: L + 32 * np.arange(nk)
    used = 0
    for _ in range(full_lanes):
        L = lanes[used]; used += 1
        row[keys(L)] = 101.0 + 99.0 * rng.random(nk)
    if partial_keys:
        L = lanes[used]; used += 1
        pos = keys(L)[rng.choice(nk, size=partial_keys, replace=False)]
        row[pos] = 101.0 + 99.0 * rng.random(partial_keys)
    while used < k - 1:
        L = lanes[used]; used += 1
        row[keys(L)[rng.integers(nk)]] = 150.0 + 50.0 * rng.random()
    L = lanes[used]
    row[keys(L)[rng.integers(nk)]] = 100.5
    return row


@pytest.mark.parametrize("E,k", [(512, 10), (1024, 12), (256, 10)])
@pytest.mark.parametrize("count", [32, 33, 55, 70])
def test_candidate_counts_around_the_limits(E, k, count):
    nk = _nk(E)
    rng = np.random.default_rng(count * 1000 + E + k)
    # f full lanes, k-1-f single-key lanes and the tau lane give f*nk + k - f
    # candidates; a partial lane of p keys in place of one single-key lane adds p-1
    base = lambda f: f * nk + k - f
    full = min((count - k) // (nk - 1), k - 2)
    partial = 0 if base(full) == count else count - base(full) + 1
    assert partial == 0 or (2 <= partial <= nk and full + 1 <= k - 1)
    T = 1500
    lg = np.stack([_lane_rows(rng, E, k, full, partial) for _ in range(T)])
    n = (lg >= 100.5).sum(axis=1)  # the construction's count
    assert (n == count).all(), (n.min(), n.max(), count)
    _check(lg, k)


@pytest.mark.parametrize("E,k,T", [(8, 2, 100), (128, 8, 3000), (512, 10, 3000), (256, 8, 120)])
@pytest.mark.parametrize("renorm", [True, False])
def test_gates_over_the_exponent_range(E, k, T, renorm):
    """The gates' fp64 softmax over exponential arguments from 0 down past
    -700: logits scaled by 0.01 up to 300, so the smallest gates underflow
    in fp32.  Every route form (one-launch cluster for small T,
    register rows for E <= 224, staged rows above) must stay within the gate
    tolerance, and the fp32 gates must equal the oracle's (libm fp64
    exponential, the same rounding) in all but a few cases near an fp32
    rounding boundary."""
    rng = np.random.default_rng(E + T + renorm)
    scales = np.array([0.01, 1.0, 30.0, 300.0], np.float32)
    lg = (rng.standard_normal((T, E)).astype(np.float32)
          * scales[np.arange(T) % 4, None]).astype(np.float32)
    ids_o, gates_o = oracle.route(lg, k, renorm=renorm)
    for ids, gates, err in _route_both(lg, k, renorm=renorm):
        assert err == (0, 0)
        assert np.array_equal(ids, ids_o)
        assert_gates_close(gates, gates_o)
        same = (gates.view(np.uint32) == gates_o.view(np.uint32)).mean()
        assert same >= 0.999, same
        assert (gates_o == 0).any() == (gates == 0).any()


@pytest.mark.parametrize("finite", [1, 5, 10, 40])
def test_rows_with_few_finite_keys(finite):
    """All but `finite` keys of each row are -inf, so with finite < k fewer
    than k lanes have a finite maximum and tau is -inf (every key a
    candidate: the exact form); the selection runs on into the -inf keys by
    expert id and their gates are 0."""
    rng = np.random.default_rng(finite)
    E, k, T = 512, 10, 2000
    lg = np.full((T, E), -np.inf, np.float32)
    for t in range(T):
        lg[t, rng.choice(E, size=finite, replace=False)] = rng.standard_normal(finite)
    _check(lg, k)
