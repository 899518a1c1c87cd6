"""Pins for the oracle's histogram and layout ("GPU MoE all-to-all", sections
"Two collectives per layer" and "Bucketing"; "MoE All-to-All Dispatch and
Ragged Routing", section "Fixed Capacity vs. Ragged Routing")."""
import numpy as np
import pytest

import oracle
from conftest import read_golden


def _random_ids(T, E, k, rng, skew=None):
    """Rows of k distinct experts, optionally skewed towards low ids."""
    ids = np.empty((T, k), np.int32)
    p = None
    if skew:
        w = np.arange(1, E + 1, dtype=np.float64) ** -skew
        p = w / w.sum()
    for t in range(T):
        ids[t] = rng.choice(E, size=k, replace=False, p=p)
    return ids


def _check_invariants(ids, E, R, L, capacity, align):
    T, k = ids.shape
    counts = L["counts"]
    assert counts.sum() == T * k
    assert np.array_equal(counts, np.bincount(ids.ravel(), minlength=E))
    off = L["expert_off"]
    assert off[0] == 0 and np.all(np.diff(off) >= 0)
    Er = E // R
    assert np.array_equal(L["rank_off"][:R], off[0:E:Er])
    assert L["rank_off"][R] == off[E]
    kept = np.minimum(counts, capacity) if capacity else counts
    assert np.array_equal(L["rank_counts"], kept.reshape(R, Er).sum(1))
    dst = L["dst_pos"].ravel()
    src = L["src_idx"]
    # inverse relation on kept assignments
    keep = dst >= 0
    assert np.array_equal(src[dst[keep]], np.nonzero(keep)[0])
    # each row of an expert segment belongs to that expert
    for e in range(E):
        seg = src[off[e]:off[e + 1]]
        used = seg[seg >= 0]
        assert np.all(ids.ravel()[used] == e)
        assert np.all(np.diff(used) > 0)          # token order inside a segment
        assert len(used) == kept[e]
        assert np.all(seg[:kept[e]] >= 0) and np.all(seg[kept[e]:] == -1)
    assert (src >= 0).sum() == kept.sum()


@pytest.mark.parametrize("T,E,R,k", [(37, 8, 4, 2), (100, 16, 4, 4), (1, 4, 2, 4),
                                     (64, 32, 8, 8), (0, 8, 2, 2)])
def test_dropless_equals_stable_argsort(T, E, R, k):
    rng = np.random.default_rng(T + E)
    ids = _random_ids(T, E, k, rng)
    L = oracle.layout(ids, E, R)
    _check_invariants(ids, E, R, L, 0, 1)
    # library special case: a stable sort by expert id is the whole layout
    assert np.array_equal(L["src_idx"], np.argsort(ids.ravel(), kind="stable"))
    assert np.array_equal(L["expert_off"], np.concatenate([[0], np.cumsum(L["counts"])]))
    # dropless is a bijection onto [0, T*k)
    assert np.array_equal(np.sort(L["dst_pos"].ravel()), np.arange(T * k))


@pytest.mark.parametrize("align", [2, 8, 128])
def test_dropless_aligned_segments(align):
    rng = np.random.default_rng(align)
    T, E, R, k = 90, 16, 4, 3
    ids = _random_ids(T, E, k, rng, skew=1.0)
    L = oracle.layout(ids, E, R, align=align)
    _check_invariants(ids, E, R, L, 0, align)
    seg = np.diff(L["expert_off"])
    assert np.all(seg % align == 0)
    assert np.array_equal(seg, -(-L["counts"] // align) * align)
    assert L["src_idx"].shape[0] == T * k + E * (align - 1)
    assert np.all(L["src_idx"][L["expert_off"][E]:] == -1)


@pytest.mark.parametrize("C", [1, 3, 7, 50])
def test_capacity_brute_force(C):
    rng = np.random.default_rng(C)
    T, E, R, k = 60, 8, 2, 3
    ids = _random_ids(T, E, k, rng, skew=1.5)
    L = oracle.layout(ids, E, R, capacity=C)
    _check_invariants(ids, E, R, L, C, 1)
    flat = ids.ravel()
    for i, e in enumerate(flat):
        rank = int(np.sum(flat[:i] == e))  # predecessors in token order
        want = e * C + rank if rank < C else -1
        assert L["dst_pos"].ravel()[i] == want
    assert np.array_equal(L["expert_off"], np.arange(E + 1) * C)


def test_all_tokens_on_the_same_experts_and_empty_experts():
    T, E, R, k = 33, 16, 4, 3
    ids = np.tile(np.array([5, 0, 9], np.int32), (T, 1))
    L = oracle.layout(ids, E, R)
    _check_invariants(ids, E, R, L, 0, 1)
    assert L["counts"][5] == T and L["counts"][1] == 0
    Lc = oracle.layout(ids, E, R, capacity=4)
    _check_invariants(ids, E, R, Lc, 4, 1)
    assert (Lc["dst_pos"] >= 0).sum() == 12


def test_out_of_range_ids_are_rejected():
    ids = np.array([[0, 8]], np.int32)
    with pytest.raises(oracle.OracleError):
        oracle.layout(ids, 8, 2)


def test_hand_worked_example():
    g = read_golden("hand_route_layout.txt")
    ids = np.array([[int(v) for v in g["ids_t0"]], [int(v) for v in g["ids_t1"]]], np.int32)
    L = oracle.layout(ids, 4, 2)
    for key in ("counts", "expert_off", "rank_off", "rank_counts", "src_idx"):
        assert L[key].tolist() == [int(v) for v in g[key]], key
    assert L["dst_pos"].ravel().tolist() == [int(v) for v in g["dst_pos"]]
    Lc = oracle.layout(ids, 4, 2, capacity=1)
    for key in ("expert_off", "rank_off", "rank_counts", "src_idx", "dst_pos"):
        assert Lc[key].ravel().tolist() == [int(v) for v in g["cap_" + key]], key
