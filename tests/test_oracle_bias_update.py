"""Pins for the oracle's aux-loss-free bias update (b_e += gamma *
sign(mean - load_e)): hand-worked exact cases, the no-op cases, and the
method's purpose -- repeated updates on a skewed router even out the load,
which a flipped sign or a wrong mean would not."""
import numpy as np
import pytest

import oracle
from conftest import read_golden


def _f(v):
    return np.array([float(x) for x in v], np.float32)


@pytest.mark.parametrize("case", ["c1", "c2", "c3"])
def test_hand_worked_cases(case):
    g = read_golden("hand_bias_update.txt")
    counts = np.array([int(x) for x in g[f"{case}_counts"]], np.int32)
    out = oracle.bias_update(counts, int(g[f"{case}_assignments"][0]), 0.125,
                             _f(g[f"{case}_bias"]))
    assert np.array_equal(out, _f(g[f"{case}_out"]))


def test_zero_gamma_and_perfect_balance_change_nothing():
    rng = np.random.default_rng(0)
    b = rng.standard_normal(64).astype(np.float32)
    counts = rng.integers(0, 100, 64).astype(np.int32)
    assert np.array_equal(oracle.bias_update(counts, int(counts.sum()), 0.0, b), b)
    flat = np.full(64, 7, np.int32)
    assert np.array_equal(oracle.bias_update(flat, 7 * 64, 0.01, b), b)


def test_repeated_updates_balance_a_skewed_router():
    """Zipf-skewed logits (the skewed workload's recipe at a small size): the
    most loaded expert's share falls steadily as the bias learns."""
    T, E, k = 2048, 32, 4
    rng = np.random.default_rng(1)
    p = (np.arange(1, E + 1, dtype=np.float64) ** -1.2)
    p /= p.sum()
    logits = (rng.standard_normal((T, E)) + 2 * np.log(p)).astype(np.float32)
    bias = np.zeros(E, np.float32)
    mean = T * k / E
    imbalance = []
    for _ in range(60):
        ids, _ = oracle.route(logits, k, bias=bias)
        counts = np.bincount(ids.ravel(), minlength=E).astype(np.int32)
        imbalance.append(counts.max() / mean)
        bias = oracle.bias_update(counts, T * k, 0.2, bias)
    assert imbalance[0] > 4.0
    assert imbalance[-1] < 1.6
    assert imbalance[-1] < imbalance[0] / 3
