"""Pins for the oracle's router ("19. All-to-all", section "Why the router can
ruin your day": the per-expert bias only takes part in the top-k decision, the
mix weights come from the router without it)."""
import math

import numpy as np
import pytest
import scipy.special

import oracle
from conftest import read_golden


def _brute_topk(logits, bias, k):
    """Full sort by (key descending, id ascending) -- a different route to the
    same set than the oracle's k rounds of selection."""
    T, E = logits.shape
    b = np.zeros(E, np.float32) if bias is None else bias
    keys = (logits + b).astype(np.float32)  # one fp32 add per element
    out = np.empty((T, k), np.int32)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(keys[t, e]), e))
        out[t] = order[:k]
    return out


@pytest.mark.parametrize("T,E,k", [(7, 8, 2), (13, 16, 5), (5, 33, 33), (9, 64, 1), (4, 3, 2)])
@pytest.mark.parametrize("with_bias", [False, True])
def test_route_ids_brute_force(T, E, k, with_bias):
    rng = np.random.default_rng(T * 1000 + E * 10 + k)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    bias = (rng.random(E).astype(np.float32) * 0.6 - 0.3) if with_bias else None
    ids, gates = oracle.route(logits, k, bias)
    assert np.array_equal(ids, _brute_topk(logits, bias, k))


def test_route_ties_go_to_lower_id_and_signed_zero_is_equal():
    logits = np.array([[0.0, -0.0, 1.0, 1.0, -0.0, 0.0],
                       [-0.0, 0.0, -0.0, 0.0, -1.0, -1.0]], np.float32)
    ids, _ = oracle.route(logits, 4)
    assert ids[0].tolist() == [2, 3, 0, 1]
    assert ids[1].tolist() == [0, 1, 2, 3]


def test_route_no_bias_equals_stable_argsort():
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((50, 40)).astype(np.float32)
    # quantise so that exact ties are common
    logits = np.round(logits * 4) / 4
    ids, _ = oracle.route(logits, 6)
    ref = np.argsort(-logits, axis=1, kind="stable")[:, :6]
    assert np.array_equal(ids, ref)


def test_gates_are_softmax_of_selected_raw_logits():
    rng = np.random.default_rng(6)
    logits = rng.standard_normal((64, 32)).astype(np.float32) * 3
    bias = rng.random(32).astype(np.float32) - 0.5
    ids, gates = oracle.route(logits, 8, bias)
    sel = np.take_along_axis(logits.astype(np.float64), ids, axis=1)
    ref = scipy.special.softmax(sel, axis=1).astype(np.float32)
    assert np.array_equal(gates, ref)
    assert np.all(np.abs(gates.astype(np.float64).sum(1) - 1.0) <= 1e-6)


def test_gates_without_renorm_are_full_softmax():
    rng = np.random.default_rng(7)
    logits = rng.standard_normal((20, 16)).astype(np.float32)
    ids, gates = oracle.route(logits, 3, renorm=False)
    full = scipy.special.softmax(logits.astype(np.float64), axis=1)
    ref = np.take_along_axis(full, ids, axis=1).astype(np.float32)
    assert np.array_equal(gates, ref)


def test_k_equals_e_renorm_equals_full_softmax():
    rng = np.random.default_rng(8)
    logits = rng.standard_normal((10, 12)).astype(np.float32)
    ids1, g1 = oracle.route(logits, 12, renorm=True)
    ids2, g2 = oracle.route(logits, 12, renorm=False)
    assert np.array_equal(ids1, ids2)
    assert np.array_equal(g1, g2)


def test_k1_gate_is_one():
    rng = np.random.default_rng(9)
    logits = rng.standard_normal((30, 9)).astype(np.float32)
    ids, gates = oracle.route(logits, 1)
    assert np.all(gates == 1.0)
    assert np.array_equal(ids[:, 0], np.argmax(logits, axis=1))


def test_bias_never_enters_the_gates():
    rng = np.random.default_rng(10)
    logits = rng.standard_normal((40, 16)).astype(np.float32)
    b1 = np.zeros(16, np.float32)
    b2 = np.full(16, 0.25, np.float32)  # shifts every key equally: same selection
    i1, g1 = oracle.route(logits, 4, b1)
    i2, g2 = oracle.route(logits, 4, b2)
    assert np.array_equal(i1, i2) and np.array_equal(g1, g2)
    # a bias that changes the selection: gates follow the raw logits of the
    # newly selected experts, not their keys
    b3 = np.zeros(16, np.float32)
    b3[0] = 100.0
    i3, g3 = oracle.route(logits, 4, b3)
    assert np.all(i3[:, 0] == 0)
    sel = np.take_along_axis(logits.astype(np.float64), i3, axis=1)
    assert np.array_equal(g3, scipy.special.softmax(sel, axis=1).astype(np.float32))


def test_hand_worked_example():
    g = read_golden("hand_route_layout.txt")
    logits = np.array([[float(v) for v in g["logits_t0"]],
                       [float(v) for v in g["logits_t1"]]], np.float32)
    bias = np.array([float(v) for v in g["bias"]], np.float32)
    ids, gates = oracle.route(logits, 2, bias)
    assert ids.tolist() == [[int(v) for v in g["ids_t0"]], [int(v) for v in g["ids_t1"]]]
    e = math.e
    assert gates[0].tolist() == [0.5, 0.5]
    assert gates[1].tolist() == [np.float32(e / (e + 1)), np.float32(1 / (e + 1))]
