"""GPU parity of the aux-loss-free bias update (moe_bias_update) against the
oracle, bit for bit: single updates on hand-worked and random histograms,
then the balancing loop itself -- route (with the bias) -> layout counts ->
bias update, repeated -- where every step's ids, counts and bias must match
the oracle's loop exactly."""
import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden
from pipeline import to_np

pytestmark = pytest.mark.gpu


def _shape(T, E, k, R=1):
    import combine_moe_route_07_b200 as m
    return m.MoeShape(tokens=T, hidden=16, experts=E, k=k, ranks=R)


@pytest.mark.parametrize("case", ["c1", "c2", "c3"])
def test_hand_worked_cases(case):
    import combine_moe_route_07_b200 as m
    g = read_golden("hand_bias_update.txt")
    counts = np.array([int(x) for x in g[f"{case}_counts"]], np.int32)
    bias = np.array([float(x) for x in g[f"{case}_bias"]], np.float32)
    A = int(g[f"{case}_assignments"][0])
    E = counts.shape[0]
    dev = torch.device("cuda:0")
    b = torch.from_numpy(bias).to(dev)
    m.moe_bias_update(_shape(A, E, 1), torch.from_numpy(counts).to(dev), 0.125, b)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(b), np.array([float(x) for x in g[f"{case}_out"]], np.float32))


@pytest.mark.parametrize("E,T,k,gamma", [(8, 100, 2, 0.001), (256, 32768, 8, 1e-3),
                                         (1024, 4097, 7, 0.03), (1, 10, 1, 0.5)])
def test_random_histograms(E, T, k, gamma):
    import combine_moe_route_07_b200 as m
    rng = np.random.default_rng(E)
    counts = rng.multinomial(T * k, np.ones(E) / E).astype(np.int32)
    bias = rng.standard_normal(E).astype(np.float32)
    dev = torch.device("cuda:0")
    b = torch.from_numpy(bias.copy()).to(dev)
    m.moe_bias_update(_shape(T, E, k), torch.from_numpy(counts).to(dev), gamma, b)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(b), oracle.bias_update(counts, T * k, gamma, bias))


def test_bad_gamma_is_rejected():
    import combine_moe_route_07_b200 as m
    dev = torch.device("cuda:0")
    c = torch.zeros(8, dtype=torch.int32, device=dev)
    b = torch.zeros(8, dtype=torch.float32, device=dev)
    for gamma in (-0.1, float("nan"), float("inf")):
        with pytest.raises(m.MoeError):
            m.moe_bias_update(_shape(4, 8, 2), c, gamma, b)


def test_balancing_loop_matches_the_oracle_step_by_step():
    import combine_moe_route_07_b200 as m
    T, E, k, R, gamma, steps = 4096, 64, 6, 8, 0.25, 40
    rng = np.random.default_rng(11)
    p = (np.arange(1, E + 1, dtype=np.float64) ** -1.2)
    p /= p.sum()
    logits = (rng.standard_normal((T, E)) + 2 * np.log(p)).astype(np.float32)
    shape = _shape(T, E, k, R)
    dev = torch.device("cuda:0")
    ws = m.Workspace(shape, dev)
    lg = torch.from_numpy(logits).to(dev)
    bias = torch.zeros(E, dtype=torch.float32, device=dev)
    ob = np.zeros(E, np.float32)
    first = last = None
    for step in range(steps):
        ids, gates, lay = m.moe_route_layout(shape, lg, bias, ws=ws)
        m.moe_bias_update(shape, lay.counts, gamma, bias)
        torch.cuda.synchronize()
        oi, _ = oracle.route(logits, k, bias=ob)
        oc = np.bincount(oi.ravel(), minlength=E).astype(np.int32)
        assert np.array_equal(to_np(ids), oi), step
        assert np.array_equal(to_np(lay.counts), oc), step
        ob = oracle.bias_update(oc, T * k, gamma, ob)
        assert np.array_equal(to_np(bias), ob), step
        imb = oc.max() / (T * k / E)
        first = imb if first is None else first
        last = imb
    assert m.moe_get_device_error(ws) == (0, 0)
    assert last < first / 2  # the loop balances the load
