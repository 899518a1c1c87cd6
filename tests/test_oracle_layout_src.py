"""Pins for the oracle's per-source-rank layout (receive-side rows ordered by
destination rank, source shard, expert, token).

Each pin comes from something other than the oracle: a hand-worked fixture,
numpy's stable lexsort / argsort / bincount, brute force in Python, and
invariants that hold for any input.  A swapped sort key, an off-by-one shard
boundary or a wrong capacity rule fails at least one of them."""
import numpy as np
import pytest

import oracle
from conftest import read_golden


def _ints(v):
    return np.array([int(x) for x in v], np.int64)


def _random_ids(T, E, k, seed):
    rng = np.random.default_rng(seed)
    ids = np.empty((T, k), np.int32)
    for t in range(T):
        ids[t] = rng.choice(E, size=k, replace=False)
    return ids


def test_hand_worked_example():
    g = read_golden("hand_layout_src.txt")
    ids = _ints(g["ids"]).reshape(4, 2).astype(np.int32)
    o = oracle.layout_src(ids, 4, 2)
    assert o["src_counts"].ravel().tolist() == _ints(g["src_counts"]).tolist()
    assert o["seg_off"].tolist() == _ints(g["seg_off"]).tolist()
    assert o["dst_pos"].ravel().tolist() == _ints(g["dst_pos"]).tolist()
    assert o["src_idx"].tolist() == _ints(g["src_idx"]).tolist()
    assert o["pair_counts"].ravel().tolist() == _ints(g["pair_counts"]).tolist()
    assert o["rank_off"].tolist() == _ints(g["rank_off"]).tolist()
    assert o["rank_counts"].tolist() == _ints(g["rank_counts"]).tolist()
    c = oracle.layout_src(ids, 4, 2, capacity=1)
    assert c["dst_pos"].ravel().tolist() == _ints(g["cap1_dst_pos"]).tolist()
    assert c["src_idx"].tolist() == _ints(g["cap1_src_idx"]).tolist()
    assert c["pair_counts"].ravel().tolist() == _ints(g["cap1_pair_counts"]).tolist()
    assert c["rank_counts"].tolist() == _ints(g["cap1_rank_counts"]).tolist()


SHAPES = [  # T, E, k, R
    (64, 8, 2, 4),
    (100, 16, 3, 4),     # T not a multiple of R: short last shard
    (7, 8, 2, 4),        # Ts = 2: shards 0..2 full or short, shard 3 short
    (3, 8, 2, 4),        # T < R: empty trailing shards
    (257, 32, 4, 8),
    (50, 6, 6, 3),       # k = E
    (40, 12, 1, 1),      # one rank: the plain expert layout
]


@pytest.mark.parametrize("T,E,k,R", SHAPES)
def test_dropless_order_is_a_stable_lexsort(T, E, k, R):
    ids = _random_ids(T, E, k, seed=T * 31 + E)
    o = oracle.layout_src(ids, E, R)
    Ts = -(-T // R)
    t = np.repeat(np.arange(T), k)
    e = ids.ravel().astype(np.int64)
    s = t // Ts
    r = e // (E // R)
    order = np.lexsort((t, e, s, r))  # primary key last: rank, shard, expert, token
    dst = o["dst_pos"].ravel()
    assert np.array_equal(dst[order], np.arange(T * k))
    assert np.array_equal(o["src_idx"][: T * k], order)


@pytest.mark.parametrize("T,E,k", [(90, 16, 3), (33, 5, 5)])
def test_one_rank_is_a_stable_argsort_of_expert_ids(T, E, k):
    ids = _random_ids(T, E, k, seed=7)
    o = oracle.layout_src(ids, E, 1)
    order = np.argsort(ids.ravel(), kind="stable")
    assert np.array_equal(o["src_idx"], order)


@pytest.mark.parametrize("T,E,k,R", SHAPES)
def test_counts_and_message_sizes(T, E, k, R):
    ids = _random_ids(T, E, k, seed=3)
    o = oracle.layout_src(ids, E, R)
    Ts = -(-T // R)
    Er = E // R
    for s in range(R):
        want = np.bincount(ids[s * Ts:(s + 1) * Ts].ravel(), minlength=E)
        assert np.array_equal(o["src_counts"][s], want)
        for r in range(R):
            assert o["pair_counts"][s, r] == want[r * Er:(r + 1) * Er].sum()
    assert o["pair_counts"].sum() == T * k
    assert np.array_equal(o["rank_counts"], o["pair_counts"].sum(axis=0))
    # rank slices are contiguous and hold exactly their experts' rows
    for r in range(R):
        lo, hi = o["rank_off"][r], o["rank_off"][r + 1]
        rows = o["src_idx"][lo:hi]
        assert np.all(ids.ravel()[rows] // Er == r)
        assert hi - lo == o["rank_counts"][r]


@pytest.mark.parametrize("C", [1, 2, 5])
@pytest.mark.parametrize("T,E,k,R", [(64, 8, 2, 4), (100, 16, 3, 4), (7, 8, 2, 4)])
def test_capacity_keeps_the_first_C_of_each_shard_expert_pair(T, E, k, R, C):
    ids = _random_ids(T, E, k, seed=11 + C)
    o = oracle.layout_src(ids, E, R, capacity=C)
    Ts = -(-T // R)
    Er = E // R
    seen = {}
    for t in range(T):
        for j in range(k):
            e = int(ids[t, j])
            s = t // Ts
            c = seen.get((s, e), 0)
            seen[(s, e)] = c + 1
            r = e // Er
            seg = (r * R + s) * Er + (e - r * Er)
            want = seg * C + c if c < C else -1
            assert o["dst_pos"][t, j] == want, (t, j)
    kept = np.minimum(o["src_counts"], C)
    for s in range(R):
        for r in range(R):
            assert o["pair_counts"][s, r] == kept[s, r * Er:(r + 1) * Er].sum()
    assert len(o["src_idx"]) == R * E * C
    assert (o["src_idx"] >= 0).sum() == kept.sum()


@pytest.mark.parametrize("align", [2, 4, 16])
def test_alignment_pads_every_segment(align):
    T, E, k, R = 120, 16, 3, 4
    ids = _random_ids(T, E, k, seed=align)
    o = oracle.layout_src(ids, E, R, align=align)
    seg = np.diff(o["seg_off"])
    assert np.all(seg % align == 0)
    Er = E // R
    sizes = [o["src_counts"][s, r * Er + el] for r in range(R) for s in range(R)
             for el in range(Er)]
    assert np.array_equal(seg, [-(-c // align) * align for c in sizes])
    # every segment: its kept rows first, then padding (-1)
    for i, c in enumerate(sizes):
        rows = o["src_idx"][o["seg_off"][i]:o["seg_off"][i + 1]]
        assert np.all(rows[:c] >= 0) and np.all(rows[c:] == -1)
    assert len(o["src_idx"]) == T * k + R * E * (align - 1)
