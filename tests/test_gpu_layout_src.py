"""GPU parity of the per-source-rank layout (moe_layout_src) against the
oracle: every output bit-exact (integer work), on the workloads' shapes
(full size included), ragged and empty shards, capacity and alignment, the
largest segment count, and the device error word; then the whole path
(dispatch and combine over the new rows) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_07_b200.workloads import WORKLOADS, Workload, bf16_bits, make_inputs
from pipeline import _scale_rows, assert_combine, gate_rows_equal, oracle_combines, to_np

pytestmark = pytest.mark.gpu

KEYS = ("src_counts", "seg_off", "pair_counts", "rank_off", "rank_counts", "dst_pos", "src_idx")


def _shape(T, H, E, k, R, capacity=0, align=1, fp8=False):
    import combine_moe_route_07_b200 as m
    return m.MoeShape(tokens=T, hidden=H, experts=E, k=k, ranks=R, capacity=capacity,
                      align=align, fp8=fp8, src_layout=True)


def _random_ids(T, E, k, seed, skew=0.0):
    rng = np.random.default_rng(seed)
    p = (np.arange(1, E + 1, dtype=np.float64) ** -skew) if skew else np.ones(E)
    p /= p.sum()
    ids = np.empty((T, k), np.int32)
    for t in range(T):
        ids[t] = rng.choice(E, size=k, replace=False, p=p)
    return ids


def _run(T, E, k, R, ids, capacity=0, align=1):
    import combine_moe_route_07_b200 as m
    shape = _shape(T, 16, E, k, R, capacity, align)
    dev = torch.device("cuda:0")
    ws = m.Workspace(shape, dev)
    lay = m.moe_layout_src(shape, torch.from_numpy(ids).to(dev), ws=ws)
    torch.cuda.synchronize()
    return lay, ws


def _compare(lay, o, what):
    for key in KEYS:
        got = to_np(getattr(lay, key))
        assert np.array_equal(got.reshape(o[key].shape), o[key]), f"{what}: {key} differs"


CASES = [  # name, T, E, k, R, capacity, align, skew
    ("prefill_shape", 4096, 128, 8, 16, 0, 1, 0.0),
    ("decode_shape", 128, 256, 8, 32, 0, 1, 0.0),
    ("tiny_shape", 256, 8, 2, 4, 0, 1, 0.0),
    ("ragged_shards", 1000, 64, 4, 16, 0, 1, 0.0),
    ("fewer_tokens_than_ranks", 5, 16, 3, 8, 0, 1, 0.0),
    ("one_rank", 777, 32, 4, 1, 0, 1, 0.0),
    ("skewed", 5000, 64, 4, 8, 0, 1, 1.2),
    ("capacity_1", 600, 32, 4, 8, 1, 1, 0.0),
    ("capacity_skewed", 3000, 64, 6, 8, 5, 1, 1.2),
    ("align_4", 900, 32, 3, 4, 0, 4, 0.0),
    ("align_128", 700, 16, 2, 4, 0, 128, 0.0),
    ("many_segments", 3000, 1024, 4, 1024, 0, 1, 0.0),   # R*E = 2^20 segments
    ("many_parts", 20000, 64, 6, 2, 0, 1, 0.5),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_layout_src_matches_oracle(case):
    import combine_moe_route_07_b200 as m
    name, T, E, k, R, C, align, skew = case
    ids = _random_ids(T, E, k, seed=T + E, skew=skew)
    lay, ws = _run(T, E, k, R, ids, C, align)
    assert m.moe_get_device_error(ws) == (0, 0)
    _compare(lay, oracle.layout_src(ids, E, R, capacity=C, align=align), name)


@pytest.mark.slow
@pytest.mark.parametrize("wname", ["skewed_dropless", "skewed_capacity", "finegrained"])
def test_layout_src_full_size_on_routed_ids(wname):
    """The workloads' own router output at full size (the oracle's layout is
    integer work and finishes in well under a second)."""
    import combine_moe_route_07_b200 as m
    w = WORKLOADS[wname]
    inp = make_inputs(w)
    dev = torch.device("cuda:0")
    shape = _shape(w.T, w.H, w.E, w.k, w.R, w.capacity_src, w.align, w.fp8)
    ws = m.Workspace(shape, dev)
    ids, _ = m.moe_route(shape, inp.logits.to(dev),
                         inp.bias.to(dev) if inp.bias is not None else None, ws=ws)
    ids_np = to_np(ids)
    # the router itself is checked elsewhere; here its ids feed both layouts
    lay = m.moe_layout_src(shape, ids, ws=ws)
    torch.cuda.synchronize()
    assert m.moe_get_device_error(ws) == (0, 0)
    _compare(lay, oracle.layout_src(ids_np, w.E, w.R, capacity=w.capacity_src, align=w.align),
             wname)


def test_empty_batch():
    import combine_moe_route_07_b200 as m
    for C, align in ((0, 1), (3, 1), (0, 4)):
        ids = np.empty((0, 2), np.int32)
        lay, ws = _run(0, 8, 2, 4, ids, C, align)
        assert m.moe_get_device_error(ws) == (0, 0)
        o = oracle.layout_src(ids, 8, 4, capacity=C, align=align)
        _compare(lay, o, f"empty C={C} align={align}")


def test_bad_ids_set_the_device_error_and_are_dropped():
    import combine_moe_route_07_b200 as m
    ids = _random_ids(64, 16, 2, seed=1)
    ids[3, 1] = 16
    ids[40, 0] = -5
    lay, ws = _run(64, 16, 2, 4, ids)
    status, _ = m.moe_get_device_error(ws)
    assert status == m._binding.MOE_ERR_DEVICE_RANGE
    dst = to_np(lay.dst_pos)
    assert dst[3, 1] == -1 and dst[40, 0] == -1


def test_flag_required_and_standard_calls_refuse_it():
    import combine_moe_route_07_b200 as m
    dev = torch.device("cuda:0")
    plain = m.MoeShape(tokens=8, hidden=16, experts=8, k=2, ranks=2)
    ws = m.Workspace(plain, dev)
    ids = torch.zeros((8, 2), dtype=torch.int32, device=dev)
    ids[:, 1] = 1
    with pytest.raises(m.MoeError):
        m.moe_layout_src(plain, ids, ws=ws)
    src = _shape(8, 16, 8, 2, 2)
    ws2 = m.Workspace(src, dev)
    with pytest.raises(m.MoeError):
        m.moe_layout(src, ids, ws=ws2)


@pytest.mark.parametrize("capacity_factor", [None, 0.5])
def test_dispatch_and_combine_over_the_src_layout(capacity_factor):
    """route -> moe_layout_src -> dispatch -> (identity / scaled experts) ->
    combine, against the oracle on the same inputs."""
    import combine_moe_route_07_b200 as m
    w = Workload("src_path", T=1500, H=256, E=32, R=8, k=4, capacity_factor=capacity_factor,
                 shared=True, residual=True, expert="scale")
    inp = make_inputs(w)
    dev = torch.device("cuda:0")
    C = w.capacity_src
    shape = _shape(w.T, w.H, w.E, w.k, w.R, C)
    ws = m.Workspace(shape, dev)
    x = inp.x.to(dev)
    ids, gates = m.moe_route(shape, inp.logits.to(dev), None, ws=ws)
    lay = m.moe_layout_src(shape, ids, ws=ws)
    xd = m.moe_dispatch(shape, x, lay.dst_pos, ws=ws)
    # expert stand-in: row of expert e scaled by (e+1)/E in fp32, rounded to bf16
    ids_np, src = to_np(ids), to_np(lay.src_idx)
    e_of_row = np.where(src >= 0, ids_np.ravel()[np.maximum(src, 0)], 0)
    scale = ((torch.arange(1, w.E + 1, dtype=torch.float32) / float(w.E))[e_of_row]).to(dev)
    y = (xd.float() * scale[:, None]).to(torch.bfloat16)
    sh = inp.shared.to(dev)  # the shared expert's output: its own draw, not x
    out = m.moe_combine(shape, y, lay.dst_pos, gates, ws=ws, shared=sh, residual=x)
    torch.cuda.synchronize()
    assert m.moe_get_device_error(ws) == (0, 0)

    # the oracle's own path: route, per-source-rank layout, dispatch
    o_ids, o_gates = oracle.route(inp.logits.numpy(), w.k, renorm=w.renorm)
    assert np.array_equal(o_ids, ids_np)
    o = oracle.layout_src(o_ids, w.E, w.R, capacity=C)
    _compare(lay, o, "path")
    xb = bf16_bits(inp.x)
    rows = oracle.dispatch_bf16(xb, o["dst_pos"], shape.rows)
    used = o["src_idx"] >= 0
    assert np.array_equal(to_np(xd).view(np.uint16)[used], rows[used])
    # the oracle's combine over its own expert rows: the same stand-in expert
    # (row of expert e times (e+1)/E) applied to the oracle's dispatch
    o_src = o["src_idx"]
    o_e = np.where(o_src >= 0, o_ids.ravel()[np.maximum(o_src, 0)], 0).astype(np.int32)
    o_y = _scale_rows(w, rows, o_e)
    want = oracle_combines(o_y, o["dst_pos"], o_gates, w.T,
                           shared_bits=bf16_bits(inp.shared), residual_bits=xb)
    assert_combine(to_np(out), want, w.k, "src_path",
                   exact_rows=gate_rows_equal(to_np(gates), o_gates))
