"""Pins for the oracle's remote-first tile-aligned layout and the round-robin
router: hand-worked fixtures, the home rank whose order is the natural one
(equal to the pinned plain layout), a relabelling of the experts that turns
any home into the natural order, invariants of the tile map, and numpy
bincount for the round-robin balance."""
import numpy as np
import pytest

import oracle
from conftest import read_golden


def _ints(v):
    return [int(x) for x in v]


def _random_ids(T, E, k, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)


def test_hand_worked_layout():
    g = read_golden("hand_remote_first.txt")
    ids = np.array(_ints(g["ids"]), np.int32).reshape(3, 2)
    o = oracle.layout_remote_first(ids, 4, 2, home=0, align=2)
    for key in ("counts", "expert_off", "rank_off", "rank_counts", "src_idx", "tile_expert"):
        assert o[key].tolist() == _ints(g[key]), key
    assert o["dst_pos"].ravel().tolist() == _ints(g["dst_pos"])


def test_hand_worked_round_robin():
    g = read_golden("hand_remote_first.txt")
    ids, gates = oracle.route_round_robin(3, 4, 2)
    assert ids.ravel().tolist() == _ints(g["rr_ids"])
    assert gates.ravel().tolist() == [float(x) for x in g["rr_gates"]]


@pytest.mark.parametrize("capacity,align", [(0, 1), (0, 4), (3, 1)])
def test_last_home_is_the_plain_layout(capacity, align):
    T, E, k, R = 200, 16, 3, 4
    ids = _random_ids(T, E, k, 1)
    a = oracle.layout_remote_first(ids, E, R, home=R - 1, capacity=capacity, align=align)
    b = oracle.layout(ids, E, R, capacity=capacity, align=align)
    for key in b:
        assert np.array_equal(a[key], b[key]), key


@pytest.mark.parametrize("home", [0, 1, 2])
@pytest.mark.parametrize("capacity,align", [(0, 1), (0, 8), (2, 1)])
def test_any_home_is_a_relabelled_plain_layout(home, capacity, align):
    """Renumber the experts so that ranks home+1, ..., home come out as
    0, 1, ..., R-1: the plain layout of the renumbered ids has the same rows."""
    T, E, k, R = 300, 24, 4, 4
    Er = E // R
    ids = _random_ids(T, E, k, home + 10)
    a = oracle.layout_remote_first(ids, E, R, home=home, capacity=capacity, align=align)
    r = ids // Er
    relabel = ((r - home - 1) % R) * Er + ids % Er
    b = oracle.layout(relabel.astype(np.int32), E, R, capacity=capacity, align=align)
    assert np.array_equal(a["dst_pos"], b["dst_pos"])
    assert np.array_equal(a["src_idx"], b["src_idx"])
    e = np.arange(E)
    e2 = ((e // Er - home - 1) % R) * Er + e % Er
    assert np.array_equal(a["expert_off"][:E], b["expert_off"][e2])


@pytest.mark.parametrize("home", [0, 3, 5])
def test_tile_map_and_slice_order(home):
    T, E, k, R, A = 500, 48, 4, 6, 16
    Er = E // R
    ids = _random_ids(T, E, k, home)
    o = oracle.layout_remote_first(ids, E, R, home=home, align=A)
    used = o["expert_off"][E]
    # slices in order home+1, ..., home, contiguous
    order = [(home + q) % R for q in range(1, R + 1)]
    starts = [o["rank_off"][r] for r in order]
    assert starts[0] == 0 and list(starts) == sorted(starts)
    assert order[-1] == home
    # every kept row sits in a tile of its own expert, every tile inside one rank
    src = o["src_idx"]
    rows = np.nonzero(src >= 0)[0]
    assert np.array_equal(o["tile_expert"][rows // A], ids.ravel()[src[rows]])
    assert np.all(o["tile_expert"][: used // A] >= 0)
    assert np.all(o["tile_expert"][used // A:] == -1)


@pytest.mark.parametrize("T,E,k", [(64, 8, 2), (1000, 256, 8), (7, 5, 5), (33, 16, 3)])
def test_round_robin_is_balanced_and_distinct(T, E, k):
    ids, gates = oracle.route_round_robin(T, E, k)
    for row in ids:
        assert len(set(row.tolist())) == k
    counts = np.bincount(ids.ravel(), minlength=E)
    assert counts.max() - counts.min() <= 1
    if (T * k) % E == 0:
        assert np.all(counts == T * k // E)
    assert np.all(gates == np.float32(1.0 / k))
