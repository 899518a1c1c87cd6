"""The threshold route's candidate set at its size limits, against the oracle.

For more than 224 experts the route first takes tau, the k-th largest of the
32 lane maxima, compacts every key >= tau (at most 64 of them) and ranks them;
with more than 64 it scans every key instead.  Here each token has n keys tied
at the top value and the rest well below, so exactly n keys reach tau: n = k
(no tie to break), 32 and 33 (one and two candidates per lane), 64 (the
largest ranked set) and 65 (the full scan).  The ties must go to the lowest
ids.  Three paths meet these inputs: rows staged in shared memory (E a multiple
of 4), rows read from global memory (E not a multiple of 4) and the one-launch
cluster path for small batches (T*k <= 1024)."""
import numpy as np
import pytest
import torch

import oracle
from pipeline import assert_gates_close, to_np

pytestmark = pytest.mark.gpu


def _tied_logits(T, E, n, seed):
    """n keys of each row tied at 1.5, the rest near -6.  The tied keys sit on
    min(n, 32) different lanes (expert e is held by lane e % 32), so at least
    k lane maxima are tied and tau is the tied value: exactly n candidates."""
    rng = np.random.default_rng(seed)
    lg = (rng.standard_normal((T, E)) - 6.0).astype(np.float32)
    for t in range(T):
        lanes = rng.permutation(32)
        slots = [rng.permutation(8) for _ in range(32)]  # distinct key index per lane
        tied = [int(lanes[j % 32] + 32 * slots[lanes[j % 32]][j // 32]) for j in range(n)]
        lg[t, tied] = 1.5
    return lg


@pytest.mark.parametrize("E,k", [(256, 8), (512, 10), (258, 8)])
@pytest.mark.parametrize("n", ["k", 32, 33, 64, 65])
@pytest.mark.parametrize("T", [100, 3000])
def test_tied_candidates_match_the_oracle(E, k, n, T):
    import combine_moe_route_07_b200 as m
    n = k if n == "k" else n
    lg = _tied_logits(T, E, n, seed=E * 7 + n)
    bias = np.zeros(E, np.float32)
    ids_o, gates_o = oracle.route(lg, k, bias)
    # the selected experts are the k lowest ids among the tied ones
    for t in range(0, T, max(1, T // 7)):
        tied = np.flatnonzero(lg[t] == 1.5)
        assert ids_o[t].tolist() == tied[:k].tolist()

    dev = torch.device("cuda:0")
    shape = m.MoeShape(tokens=T, hidden=16, experts=E, k=k, ranks=2)
    ws = m.Workspace(shape, dev)
    lgd = torch.from_numpy(lg).to(dev)
    bd = torch.from_numpy(bias).to(dev)
    ids, gates = m.moe_route(shape, lgd, bd, ws=ws)
    ids2, gates2, _ = m.moe_route_layout(shape, lgd, bd, ws=ws)  # cluster path when small
    torch.cuda.synchronize()
    assert m.moe_get_device_error(ws) == (0, 0)
    for got_ids, got_gates in ((ids, gates), (ids2, gates2)):
        assert np.array_equal(to_np(got_ids), ids_o)
        assert_gates_close(to_np(got_gates), gates_o)
