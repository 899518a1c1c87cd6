"""Route + layout of decode-sized batches against the oracle.

Batches of at most 1024 assignments (and at most 512 experts) take the
one-launch path: an 8-CTA thread-block cluster that shares its per-CTA
histograms over distributed shared memory.  Larger batches take the route and
layout kernels.  Every case here is compared with the oracle (ids, counts,
offsets, dst_pos and src_idx bit-exact, gates within 1e-6 relative) and with
the separate moe_route + moe_layout calls on the same device (identical bits),
on both sides of the size boundary, with fewer tokens than CTAs in the
cluster, token counts that split unevenly over the CTAs, the largest expert
count, padding rows (alignment, unused capacity) and capacity drops."""
import numpy as np
import pytest
import torch

import oracle
from pipeline import assert_gates_close, to_np

pytestmark = pytest.mark.gpu

LAYOUT_KEYS = ("counts", "expert_off", "rank_off", "rank_counts", "dst_pos", "src_idx")

# T, E, k, R, capacity, align, bias, renorm, skew (hot-expert logit offset)
CASES = [
    (128, 256, 8, 32, 0, 1, True, True, 0.0),     # the decode shape
    (1, 8, 2, 2, 0, 1, False, True, 0.0),         # one token: seven CTAs without tokens
    (5, 64, 4, 8, 0, 1, True, True, 0.0),         # fewer tokens than CTAs
    (9, 48, 3, 4, 0, 1, False, False, 0.0),       # uneven split, two keys per lane, full softmax
    (128, 512, 8, 64, 0, 1, True, True, 0.0),     # largest expert count, 1024 assignments
    (100, 100, 10, 4, 0, 128, True, True, 1.0),   # alignment padding rows
    (128, 256, 8, 32, 4, 1, False, True, 2.0),    # capacity: drops and unused slots
    (64, 16, 16, 4, 0, 1, False, True, 0.0),      # k = E
    (73, 32, 6, 32, 3, 1, True, True, 1.5),       # one expert per rank, capacity
    (129, 256, 8, 32, 0, 1, True, True, 0.0),     # 1032 assignments: the two-kernel path
    (256, 256, 8, 32, 0, 1, True, True, 0.0),     # the two-kernel path
]


def _inputs(T, E, bias, skew, seed):
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    if skew:
        logits += (skew * np.arange(E, 0, -1) / E).astype(np.float32)  # low ids run hot
    b = (rng.random(E) * 0.2 - 0.1).astype(np.float32) if bias else None
    return logits, b


@pytest.mark.parametrize("T,E,k,R,C,align,bias,renorm,skew", CASES)
def test_route_layout_matches_oracle_and_separate_calls(T, E, k, R, C, align, bias, renorm,
                                                        skew):
    import combine_moe_route_07_b200 as m
    logits, b = _inputs(T, E, bias, skew, seed=T * 131 + E)
    ids_o, gates_o = oracle.route(logits, k, b, renorm=renorm)
    L = oracle.layout(ids_o, E, R, capacity=C, align=align)
    if C > 0:  # the capacity cases drop slots and leave rows unused
        assert (L["dst_pos"] < 0).any() and (L["src_idx"] < 0).any()
    if align > 1:
        assert (L["src_idx"] < 0).any()

    dev = torch.device("cuda:0")
    shape = m.MoeShape(tokens=T, hidden=16, experts=E, k=k, ranks=R, capacity=C, align=align,
                       renorm=renorm)
    ws = m.Workspace(shape, dev)
    lg = torch.from_numpy(logits).to(dev)
    bt = torch.from_numpy(b).to(dev) if b is not None else None
    ids, gates, lay = m.moe_route_layout(shape, lg, bt, ws=ws)
    torch.cuda.synchronize()
    assert m.moe_get_device_error(ws) == (0, 0)
    assert np.array_equal(to_np(ids), ids_o)
    assert_gates_close(to_np(gates), gates_o)
    for key in LAYOUT_KEYS:
        assert np.array_equal(to_np(getattr(lay, key)), L[key]), key

    ids2, gates2 = m.moe_route(shape, lg, bt, ws=ws)
    lay2 = m.moe_layout(shape, ids2, ws=ws)
    assert torch.equal(ids, ids2) and torch.equal(gates, gates2)
    for key in LAYOUT_KEYS:
        assert torch.equal(getattr(lay, key), getattr(lay2, key)), key

