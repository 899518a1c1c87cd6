"""Pins for the oracle's rank-limited route (each token's experts from at
most M of the R ranks; group score = the largest key on the rank).

Pinned by a hand-worked fixture, by the special cases that reduce to
something already pinned or to a library routine (M >= R is the unrestricted
route; M = 1 takes the top-k of the rank holding the largest key, a stable
numpy argsort), and by properties every output must have."""
import numpy as np
import pytest

import oracle
from conftest import read_golden


def _logits(T, E, seed, ties=False):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, E)).astype(np.float32)
    if ties:
        x = np.round(x * 2).astype(np.float32) / 2
    return x


def test_hand_worked_example():
    g = read_golden("hand_route_limited.txt")
    logits = np.array([float(v) for v in g["logits"]], np.float32).reshape(2, 8)
    ids, gates = oracle.route_limited(logits, 3, 4, 2)
    assert ids.ravel().tolist() == [int(v) for v in g["ids"]]
    np.testing.assert_allclose(gates.ravel(), [float(v) for v in g["gates"]], rtol=1e-6)
    ids4, gates4 = oracle.route_limited(logits[:1], 3, 4, 4)
    assert ids4.ravel().tolist() == [int(v) for v in g["unlimited_ids_token0"]]
    np.testing.assert_allclose(gates4.ravel(), [float(v) for v in g["unlimited_gates_token0"]],
                               rtol=1e-6)


@pytest.mark.parametrize("T,E,k,R,M", [(50, 16, 4, 4, 4), (40, 32, 8, 8, 9), (30, 64, 6, 64, 64)])
@pytest.mark.parametrize("renorm", [True, False])
def test_no_limit_is_the_unrestricted_route(T, E, k, R, M, renorm):
    lg = _logits(T, E, seed=E)
    bias = (np.random.default_rng(1).random(E).astype(np.float32) * 0.2 - 0.1)
    a = oracle.route_limited(lg, k, R, M, bias=bias, renorm=renorm)
    b = oracle.route(lg, k, bias=bias, renorm=renorm)
    assert np.array_equal(a[0], b[0])
    assert np.array_equal(a[1], b[1])


@pytest.mark.parametrize("ties", [False, True])
def test_one_rank_takes_the_top_k_of_the_best_rank(ties):
    T, E, k, R = 60, 32, 3, 8
    Er = E // R
    lg = _logits(T, E, seed=5, ties=ties)
    ids, _ = oracle.route_limited(lg, k, R, 1)
    for t in range(T):
        keys = lg[t]
        r = int(np.argmax(keys)) // Er  # first maximum: the lower id among equals
        want = r * Er + np.argsort(-keys[r * Er:(r + 1) * Er], kind="stable")[:k]
        assert ids[t].tolist() == want.tolist(), t


@pytest.mark.parametrize("T,E,k,R,M", [(200, 64, 8, 8, 2), (200, 256, 8, 32, 4),
                                       (100, 512, 10, 64, 4), (100, 24, 6, 6, 3)])
@pytest.mark.parametrize("ties", [False, True])
def test_properties(T, E, k, R, M, ties):
    Er = E // R
    lg = _logits(T, E, seed=T + E, ties=ties)
    bias = (np.random.default_rng(2).random(E).astype(np.float32) * 0.2 - 0.1)
    ids, gates = oracle.route_limited(lg, k, R, M, bias=bias)
    keys = lg + bias  # one fp32 add, as the route defines
    for t in range(T):
        sel = ids[t]
        assert len(set(sel.tolist())) == k
        used = set((sel // Er).tolist())
        assert len(used) <= M
        score = keys[t].reshape(R, Er).max(axis=1)
        mth = np.sort(score)[::-1][M - 1]
        assert all(score[r] >= mth for r in used)          # only top-M ranks are used
        # slot order: keys non-increasing, equal keys by increasing id
        ks = keys[t][sel]
        assert np.all(ks[:-1] >= ks[1:])
        for j in range(k - 1):
            if ks[j] == ks[j + 1]:
                assert sel[j] < sel[j + 1]
        # nothing left out on a used rank beats the last selected key
        last = ks[-1]
        for r in used:
            for e in range(r * Er, (r + 1) * Er):
                if e not in sel:
                    assert keys[t][e] < last or (keys[t][e] == last and e > sel[-1])
    np.testing.assert_allclose(gates.sum(axis=1), 1.0, rtol=1e-6)


def test_gates_ignore_the_bias():
    T, E, k, R, M = 80, 32, 4, 8, 2
    lg = _logits(T, E, seed=9)
    b1 = np.zeros(E, np.float32)
    b2 = np.full(E, 0.25, np.float32)  # a constant shift changes no selection
    i1, g1 = oracle.route_limited(lg, k, R, M, bias=b1)
    i2, g2 = oracle.route_limited(lg, k, R, M, bias=b2)
    assert np.array_equal(i1, i2)
    assert np.array_equal(g1, g2)


def test_too_few_eligible_experts_is_rejected():
    with pytest.raises(oracle.OracleError):
        oracle.route_limited(_logits(4, 16, 0), 5, 8, 2)   # 2 ranks x 2 experts < 5
