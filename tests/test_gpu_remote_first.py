"""GPU parity of the remote-first tile-aligned layout (moe_layout_remote_first)
and of the round-robin router (moe_route_round_robin) against the oracle:
integer outputs bit-exact, on the workloads' shapes with 128-row tiles,
capacity, ragged and skewed batches, every home rank position, and the
whole path behind the round-robin router."""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_07_b200.workloads import Workload, bf16_bits, make_inputs
from pipeline import assert_combine, oracle_combines, to_np

pytestmark = pytest.mark.gpu

KEYS = ("counts", "expert_off", "rank_off", "rank_counts", "dst_pos", "src_idx")


def _random_ids(T, E, k, seed, skew=0.0):
    rng = np.random.default_rng(seed)
    p = (np.arange(1, E + 1, dtype=np.float64) ** -skew) if skew else np.ones(E)
    p /= p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


def _shape(T, E, k, R, capacity=0, align=1, H=16):
    import combine_moe_route_07_b200 as m
    return m.MoeShape(tokens=T, hidden=H, experts=E, k=k, ranks=R, capacity=capacity, align=align)


CASES = [  # name, T, E, k, R, capacity, align, skew
    ("prefill_tiles128", 4096, 128, 8, 16, 0, 128, 0.0),
    ("decode_tiles128", 128, 256, 8, 32, 0, 128, 0.0),
    ("decode_rows", 128, 256, 8, 32, 0, 1, 0.0),
    ("skewed_tiles128", 6000, 64, 8, 8, 0, 128, 1.2),
    ("capacity", 3000, 32, 4, 8, 100, 1, 1.2),
    ("ragged", 301, 24, 3, 6, 0, 4, 0.0),
    ("odd_E", 500, 30, 4, 5, 0, 8, 0.0),
    ("one_rank", 200, 16, 2, 1, 0, 16, 0.0),
    ("many_tiles", 20000, 64, 6, 8, 0, 128, 0.5),
]


@pytest.mark.parametrize("where", ["first", "middle", "last"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_remote_first_matches_oracle(case, where):
    import combine_moe_route_07_b200 as m
    name, T, E, k, R, C, align, skew = case
    home = {"first": 0, "middle": R // 2, "last": R - 1}[where]
    ids = _random_ids(T, E, k, seed=T + E + home, skew=skew)
    shape = _shape(T, E, k, R, C, align)
    dev = torch.device("cuda:0")
    ws = m.Workspace(shape, dev)
    lay, tiles = m.moe_layout_remote_first(shape, torch.from_numpy(ids).to(dev), home, ws=ws)
    torch.cuda.synchronize()
    assert m.moe_get_device_error(ws) == (0, 0)
    o = oracle.layout_remote_first(ids, E, R, home, capacity=C, align=align)
    for key in KEYS:
        assert np.array_equal(to_np(getattr(lay, key)), o[key]), f"{name} home={home}: {key}"
    assert np.array_equal(to_np(tiles), o["tile_expert"]), f"{name} home={home}: tile_expert"


def test_last_home_equals_moe_layout():
    import combine_moe_route_07_b200 as m
    T, E, k, R = 2000, 64, 4, 8
    ids = torch.from_numpy(_random_ids(T, E, k, 5)).cuda()
    shape = _shape(T, E, k, R, align=16)
    ws = m.Workspace(shape, ids.device)
    a, _ = m.moe_layout_remote_first(shape, ids, R - 1, ws=ws)
    b = m.moe_layout(shape, ids, ws=ws)
    torch.cuda.synchronize()
    for key in KEYS:
        assert torch.equal(getattr(a, key), getattr(b, key)), key


def test_bad_home_rank_is_rejected():
    import combine_moe_route_07_b200 as m
    shape = _shape(8, 8, 2, 4)
    ws = m.Workspace(shape, torch.device("cuda:0"))
    ids = torch.zeros((8, 2), dtype=torch.int32, device="cuda")
    ids[:, 1] = 1
    for home in (-1, 4):
        with pytest.raises(m.MoeError):
            m.moe_layout_remote_first(shape, ids, home, ws=ws)


@pytest.mark.parametrize("T,E,k", [(4096, 128, 8), (7, 5, 5), (1, 8, 3), (65536, 512, 10)])
def test_round_robin_matches_oracle(T, E, k):
    import combine_moe_route_07_b200 as m
    shape = _shape(T, E, k, 1)
    ids, gates = m.moe_route_round_robin(shape, device=torch.device("cuda:0"))
    torch.cuda.synchronize()
    oi, og = oracle.route_round_robin(T, E, k)
    assert np.array_equal(to_np(ids), oi)
    assert np.array_equal(to_np(gates), og)


def test_path_behind_the_round_robin_router():
    """round-robin ids -> remote-first layout (128-row tiles) -> dispatch ->
    stand-in expert -> combine, against the oracle."""
    import combine_moe_route_07_b200 as m
    w = Workload("rr_path", T=1024, H=256, E=32, R=8, k=4, align=128, residual=True)
    inp = make_inputs(w)
    dev = torch.device("cuda:0")
    shape = _shape(w.T, w.E, w.k, w.R, align=w.align, H=w.H)
    ws = m.Workspace(shape, dev)
    x = inp.x.to(dev)
    ids, gates = m.moe_route_round_robin(shape, device=dev)
    lay, _ = m.moe_layout_remote_first(shape, ids, 3, ws=ws)
    xd = m.moe_dispatch(shape, x, lay.dst_pos, ws=ws)
    out = m.moe_combine(shape, xd, lay.dst_pos, gates, ws=ws, residual=x)  # identity experts
    torch.cuda.synchronize()
    assert m.moe_get_device_error(ws) == (0, 0)
    oi, og = oracle.route_round_robin(w.T, w.E, w.k)
    o = oracle.layout_remote_first(oi, w.E, w.R, 3, align=w.align)
    xb = bf16_bits(inp.x)
    rows = oracle.dispatch_bf16(xb, o["dst_pos"], shape.rows)
    used = o["src_idx"] >= 0
    assert np.array_equal(to_np(xd)[used], rows[used])
    want = oracle_combines(rows, o["dst_pos"], og, w.T, residual_bits=xb)
    assert_combine(to_np(out), want, w.k, "rr_path")
