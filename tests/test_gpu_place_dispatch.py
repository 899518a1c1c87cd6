"""Steps 1-4 through moe_route_layout_dispatch on dropless bf16 batches of at
least 2048 tokens with rows of 1-32 KiB and at most 512 assignments in each
CTA's range of tokens: the route kernel fills the per-tile
count table, then one kernel places each CTA's contiguous range of tokens
(from the table, plus the ids of the range's first, partial tile) and streams
its rows by bulk copy.  Against the oracle, and bit for bit against the
separate moe_route, moe_layout and moe_dispatch calls on the same inputs.

The shapes cover the kernel's branches: ranges that start inside a tile (the
partial-tile count), vector and scalar reads of the table (E a multiple of 4
or not), alignment padding rows, k = 1 and k = 32, bias and no
renormalisation, rings that hold every row of a range and rings that refill,
the widest rows that give two stages (24 KiB), the smallest batch it serves
(2048 tokens) and a last range of one token.  A capacity case checks that
the call keeps the separate calls' bits when it takes the other form."""
import numpy as np
import pytest
import torch

from combine_moe_route_07_b200.workloads import WORKLOADS, Workload, make_inputs
from pipeline import assert_gates_close, run_gpu, run_oracle, to_np

pytestmark = pytest.mark.gpu

LAYOUT_KEYS = ("counts", "expert_off", "rank_off", "rank_counts", "dst_pos", "src_idx")

CASES = [
    WORKLOADS["prefill"],                                              # ranges of 28 tokens, tiles of 32
    WORKLOADS["skewed_dropless"].with_(name="skewed_dropless_8k", T=8192),
    Workload("prefill_bias_capacity", T=4096, H=4096, E=128, R=16, k=8, bias=True,
             capacity_factor=1.0),                                     # the other form
    Workload("e_not_mult4", T=3000, H=512, E=30, R=5, k=3),
    Workload("k1", T=2100, H=512, E=64, R=8, k=1),
    Workload("k32", T=2048, H=512, E=64, R=4, k=32),                  # 448 assignments a range
    Workload("align128", T=2500, H=1024, E=64, R=8, k=4, align=128),
    Workload("no_renorm_bias", T=2400, H=1024, E=48, R=6, k=6, renorm=False, bias=True),
    Workload("ring_refill", T=8192, H=8192, E=128, R=16, k=8),         # 56 tokens a range, 2 stages
    Workload("wide_row", T=2500, H=12288, E=64, R=8, k=2),             # 24 KiB rows, 2 stages
    Workload("smallest_batch", T=2048, H=512, E=64, R=8, k=4),
    Workload("last_range_one_token", T=2206, H=512, E=64, R=8, k=4),   # 147 ranges of 15, then 1
]


def _separate(w, inp):
    import combine_moe_route_07_b200 as m
    from pipeline import shape_of
    shape = shape_of(w)
    dev = torch.device("cuda:0")
    ws = m.Workspace(shape, dev)
    bias = None if inp.bias is None else inp.bias.to(dev)
    ids, gates = m.moe_route(shape, inp.logits.to(dev), bias, ws=ws)
    lay = m.moe_layout(shape, ids, ws=ws)
    xd = m.moe_dispatch(shape, inp.x.to(dev), lay.dst_pos, ws=ws)
    torch.cuda.synchronize()
    assert m.moe_get_device_error(ws) == (0, 0)
    return ids, gates, lay, xd


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_fused_steps_1_to_4(w):
    import combine_moe_route_07_b200 as m
    inp = make_inputs(w)
    o = run_oracle(w, inp, through="layout")
    g = run_gpu(w, inp, fused="dispatch")
    assert m.moe_get_device_error(g["ws"]) == (0, 0)
    assert np.array_equal(to_np(g["ids"]), o["ids"])
    assert_gates_close(to_np(g["gates"]), o["gates"])
    for key in LAYOUT_KEYS:
        assert np.array_equal(to_np(getattr(g["layout"], key)), o["layout"][key]), key
    # every kept copy is its token's row (the oracle's dispatch is this copy)
    dst = o["layout"]["dst_pos"]
    kept = dst >= 0
    rows = torch.from_numpy(dst[kept]).long().cuda()
    tok = torch.from_numpy(np.nonzero(kept)[0]).long().cuda()
    assert torch.equal(g["dispatch"].index_select(0, rows), g["x"].index_select(0, tok))
    # the same bits as the separate calls
    ids, gates, lay, xd = _separate(w, inp)
    assert torch.equal(ids, g["ids"]) and torch.equal(gates, g["gates"])
    for key in LAYOUT_KEYS:
        assert torch.equal(getattr(lay, key), getattr(g["layout"], key)), key
    used = lay.src_idx >= 0
    assert torch.equal(xd[used], g["dispatch"][used])


def test_fused_steps_twice_and_after_other_calls():
    """The tile tables alternate between calls and the placing kernel clears
    the one the previous call filled: calls in a row, interleaved with the
    other entry points on the same workspace, give the same bits."""
    import combine_moe_route_07_b200 as m
    from pipeline import shape_of
    w = WORKLOADS["prefill"]
    inp = make_inputs(w)
    dev = torch.device("cuda:0")
    shape = shape_of(w)
    ws = m.Workspace(shape, dev)
    x, logits = inp.x.to(dev), inp.logits.to(dev)
    first = m.moe_route_layout_dispatch(shape, logits, x, None, ws=ws)
    for _ in range(3):
        ids, gates = m.moe_route(shape, logits, None, ws=ws)
        m.moe_layout(shape, ids, ws=ws)
        again = m.moe_route_layout_dispatch(shape, logits, x, None, ws=ws)
        torch.cuda.synchronize()
        assert torch.equal(again[0], first[0]) and torch.equal(again[1], first[1])
        assert torch.equal(again[2].dst_pos, first[2].dst_pos)
        assert torch.equal(again[3], first[3])
    assert m.moe_get_device_error(ws) == (0, 0)
