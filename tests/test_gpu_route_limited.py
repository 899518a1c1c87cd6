"""GPU parity of the rank-limited route (moe_route_limited) against the
oracle: ids bit-exact, gates within 1e-6 relative, on every selection path of
the kernel (full scan for E <= 224, threshold selection above, shared-memory
row staging for E a multiple of 4 above 224), with ties, a bias, one expert
per rank, the largest E, and the unrestricted special case."""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_07_b200.workloads import WORKLOADS, make_inputs
from pipeline import assert_gates_close, to_np

pytestmark = pytest.mark.gpu


def _run(logits, k, R, M, bias=None, renorm=True):
    import combine_moe_route_07_b200 as m
    T, E = logits.shape
    shape = m.MoeShape(tokens=T, hidden=16, experts=E, k=k, ranks=R, renorm=renorm)
    dev = torch.device("cuda:0")
    ws = m.Workspace(shape, dev)
    b = None if bias is None else torch.from_numpy(bias).to(dev)
    ids, gates = m.moe_route_limited(shape, torch.from_numpy(logits).to(dev), M, b, ws=ws)
    torch.cuda.synchronize()
    assert m.moe_get_device_error(ws) == (0, 0)
    return to_np(ids), to_np(gates)


CASES = [  # T, E, k, R, M, ties, bias, renorm
    (4096, 512, 10, 64, 4, False, False, True),    # staged threshold path
    (2000, 256, 8, 32, 4, False, True, True),      # threshold path, bias
    (1000, 128, 8, 16, 2, False, False, True),     # full-scan path
    (1000, 128, 8, 16, 2, True, False, True),      # ties
    (500, 64, 6, 8, 1, True, False, True),         # one rank
    (300, 32, 1, 32, 1, False, False, True),       # one expert per rank
    (200, 1024, 32, 1024, 32, False, False, True),  # largest E, k = M * E/R
    (400, 24, 6, 6, 3, False, False, False),       # E not a multiple of 32, no renorm
    (777, 300, 5, 10, 3, True, True, True),        # E > 224 with ties and a bias
    (333, 226, 4, 2, 1, False, False, True),       # E > 224 and E % 4 != 0: threshold, no staging
]


@pytest.mark.parametrize("case", CASES, ids=[f"T{c[0]}_E{c[1]}_k{c[2]}_R{c[3]}_M{c[4]}"
                                             + ("_ties" if c[5] else "") for c in CASES])
def test_route_limited_matches_oracle(case):
    T, E, k, R, M, ties, use_bias, renorm = case
    rng = np.random.default_rng(T + E + M)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    if ties:
        lg = (np.round(lg * 2) / 2).astype(np.float32)
    bias = (rng.random(E).astype(np.float32) * 0.2 - 0.1) if use_bias else None
    ids, gates = _run(lg, k, R, M, bias, renorm)
    oi, og = oracle.route_limited(lg, k, R, M, bias=bias, renorm=renorm)
    assert np.array_equal(ids, oi)
    assert_gates_close(gates, og)


def test_no_limit_equals_moe_route():
    import combine_moe_route_07_b200 as m
    rng = np.random.default_rng(3)
    lg = rng.standard_normal((512, 256)).astype(np.float32)
    ids, gates = _run(lg, 8, 32, 32)
    shape = m.MoeShape(tokens=512, hidden=16, experts=256, k=8, ranks=32)
    dev = torch.device("cuda:0")
    ws = m.Workspace(shape, dev)
    i2, g2 = m.moe_route(shape, torch.from_numpy(lg).to(dev), ws=ws)
    assert np.array_equal(ids, to_np(i2))
    assert np.array_equal(gates, to_np(g2))


def test_too_few_eligible_experts_is_rejected():
    import combine_moe_route_07_b200 as m
    shape = m.MoeShape(tokens=4, hidden=16, experts=16, k=5, ranks=8)
    dev = torch.device("cuda:0")
    ws = m.Workspace(shape, dev)
    with pytest.raises(m.MoeError):
        m.moe_route_limited(shape, torch.zeros((4, 16), device=dev), 2, ws=ws)


@pytest.mark.slow
def test_full_size_finegrained_limited_to_four_ranks():
    w = WORKLOADS["finegrained"]
    inp = make_inputs(w)
    lg = inp.logits.numpy()
    ids, gates = _run(lg, w.k, w.R, 4)
    oi, og = oracle.route_limited(lg, w.k, w.R, 4)
    assert np.array_equal(ids, oi)
    assert_gates_close(gates, og)
    used = (ids // (w.E // w.R))
    assert max(len(set(row.tolist())) for row in used) <= 4
