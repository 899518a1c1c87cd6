"""GPU edge cases against the oracle: empty and ragged inputs, extreme k and E,
minimum widths, alignment, tiny capacity, degenerate routing, and the device
error word (bad ids, bad rows, NaN keys) -- all without faulting the GPU: every
bad input here is one the host checks or the kernels' own bounds checks turn
into a status."""
import numpy as np
import pytest
import torch

from combine_moe_route_07_b200.workloads import Workload, make_inputs
from pipeline import (assert_combine, assert_gates_close, gate_rows_equal, run_gpu, run_oracle,
                      shape_of, to_np)

pytestmark = pytest.mark.gpu

LAYOUT_KEYS = ("counts", "expert_off", "rank_off", "rank_counts", "dst_pos", "src_idx")


def _check_all(w, inp=None, fused=False):
    import combine_moe_route_07_b200 as m
    inp = inp or make_inputs(w)
    o = run_oracle(w, inp)
    g = run_gpu(w, inp, fused=fused)
    assert m.moe_get_device_error(g["ws"]) == (0, 0)
    assert np.array_equal(to_np(g["ids"]), o["ids"])
    assert_gates_close(to_np(g["gates"]), o["gates"])
    for key in LAYOUT_KEYS:
        assert np.array_equal(to_np(getattr(g["layout"], key)), o["layout"][key]), key
    src = o["layout"]["src_idx"]
    used = src >= 0
    if w.fp8:
        q, s = g["dispatch"]
        assert np.array_equal(to_np(q)[used], o["dispatch"][0][used])
        assert np.array_equal(to_np(s)[used], o["dispatch"][1][used])
    else:
        assert np.array_equal(to_np(g["dispatch"])[used], o["dispatch"][used])
    assert_combine(to_np(g["out"]), o, w.k, w.name,
                   exact_rows=gate_rows_equal(to_np(g["gates"]), o["gates"]))


CASES = [
    Workload("ragged_tiles", T=300, H=64, E=16, R=4, k=3),
    Workload("one_token", T=1, H=128, E=8, R=2, k=2),
    Workload("tile_plus_one", T=129, H=16, E=8, R=8, k=4),
    Workload("k_equals_e", T=200, H=32, E=8, R=2, k=8),
    Workload("k1", T=257, H=40, E=32, R=4, k=1),
    Workload("one_expert", T=70, H=24, E=1, R=1, k=1),
    Workload("max_experts_k32", T=150, H=16, E=1024, R=1, k=32),
    Workload("max_experts_ranks", T=300, H=16, E=1024, R=1024, k=5),
    Workload("h8", T=500, H=8, E=16, R=2, k=2),
    Workload("fp8_h128", T=333, H=128, E=16, R=4, k=4, fp8=True, expert="dequant"),
    Workload("fp8_capacity", T=400, H=256, E=8, R=2, k=2, fp8=True, expert="dequant",
             capacity_factor=1, residual=True),
    # H % 512 == 0: the FP8 path that stages codes and scales in shared memory
    Workload("fp8_bulk_h512", T=137, H=512, E=16, R=4, k=3, fp8=True, expert="dequant"),
    Workload("fp8_bulk_h1536_capacity", T=300, H=1536, E=8, R=2, k=4, fp8=True,
             expert="dequant", capacity_factor=0.5, residual=True),
    Workload("fp8_bulk_h8192", T=41, H=8192, E=8, R=2, k=2, fp8=True, expert="dequant"),
    Workload("fp8_h8704", T=19, H=8704, E=8, R=2, k=2, fp8=True, expert="dequant"),
    Workload("align128", T=700, H=32, E=16, R=4, k=2, align=128),
    Workload("align3_odd", T=77, H=16, E=6, R=3, k=2, align=3),
    Workload("capacity_c1", T=300, H=16, E=64, R=8, k=4, capacity_factor=0.0001),
    Workload("capacity_skewed", T=1000, H=64, E=32, R=4, k=4, capacity_factor=1.2, zipf_s=1.2),
    Workload("no_renorm", T=90, H=32, E=16, R=4, k=4, renorm=False),
    Workload("bias_shared_residual", T=260, H=48, E=24, R=6, k=3, bias=True, shared=True,
             residual=True),
    Workload("scale_expert_capacity", T=512, H=64, E=16, R=4, k=2, expert="scale",
             capacity_factor=0.8),
    Workload("many_tiles", T=20000, H=16, E=64, R=8, k=6),
    # more 128-token tiles than CTAs that fit at once: the launch widens tiles
    Workload("wide_tiles", T=120000, H=8, E=1024, R=8, k=2),
]


@pytest.mark.parametrize("fused", [False, True, "dispatch"], ids=["separate", "fused", "fused3"])
@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_edge_case_parity(w, fused):
    _check_all(w, fused=fused)


def test_empty_batch():
    import combine_moe_route_07_b200 as m
    for cap, align in ((0, 1), (3, 1), (0, 4)):
        shape = m.MoeShape(tokens=0, hidden=16, experts=8, k=2, ranks=2, capacity=cap,
                           align=align)
        dev = torch.device("cuda:0")
        ws = m.Workspace(shape, dev)
        ids = torch.empty((0, 2), dtype=torch.int32, device=dev)
        lay = m.moe_layout(shape, ids, ws=ws)
        torch.cuda.synchronize()
        assert to_np(lay.counts).tolist() == [0] * 8
        want_off = [e * cap for e in range(9)] if cap else [0] * 9
        assert to_np(lay.expert_off).tolist() == want_off
        assert np.all(to_np(lay.src_idx) == -1)
        assert to_np(lay.rank_counts).tolist() == [0, 0]
        x = torch.empty((0, 16), dtype=torch.bfloat16, device=dev)
        out = m.moe_dispatch(shape, x, lay.dst_pos, ws=ws)
        g = torch.empty((0, 2), dtype=torch.float32, device=dev)
        comb = m.moe_combine(shape, out, lay.dst_pos, g, ws=ws)
        assert comb.shape == (0, 16)
        assert m.moe_get_device_error(ws) == (0, 0)


def test_all_tokens_on_the_same_experts():
    # a large bias on experts 5, 2, 7 makes every token pick exactly them
    w = Workload("same_experts", T=1000, H=32, E=16, R=4, k=3)
    inp = make_inputs(w)
    bias = torch.zeros(16)
    bias[5], bias[2], bias[7] = 300.0, 200.0, 100.0
    inp.bias = bias
    for fused in (False, True, "dispatch"):
        _check_all(w, inp, fused)
        wc = w.with_(name="same_experts_capacity", capacity_factor=0.25)
        _check_all(wc, inp, fused)


@pytest.mark.parametrize("H", [256, 1024])
def test_fp8_zero_blocks_get_zero_codes_and_scale(H):
    """A 128-channel block that is all zeros (or all -0) quantises to code 0
    and scale 0; its neighbours in the same row are unaffected."""
    w = Workload(f"fp8_zero_{H}", T=200, H=H, E=16, R=4, k=3, fp8=True, expert="dequant")
    inp = make_inputs(w)
    inp.x[::3, :128] = 0.0
    inp.x[1::7, 128:256] = -0.0
    inp.x[5] = 0.0
    for fused in (False, "dispatch"):
        _check_all(w, inp, fused)


@pytest.mark.parametrize("E,k", [(256, 8), (512, 10), (1024, 32)])
def test_heavy_ties_take_the_full_scan(E, k):
    """Keys with few distinct values: the threshold selection sees more than
    64 candidates and must fall back to the full scan; ties go to the lower id."""
    w = Workload(f"ties_{E}", T=300, H=16, E=E, R=8, k=k)
    inp = make_inputs(w)
    inp.logits = torch.round(inp.logits * 2) / 2
    inp.logits[:50] = 0.0  # all keys equal
    _check_all(w, inp)


def test_bad_ids_set_the_device_error_and_are_dropped():
    import combine_moe_route_07_b200 as m
    from combine_moe_route_07_b200._binding import MOE_ERR_DEVICE_RANGE
    w = Workload("bad", T=300, H=16, E=8, R=2, k=2)
    shape = shape_of(w)
    dev = torch.device("cuda:0")
    ws = m.Workspace(shape, dev)
    ids = torch.tensor([[0, 1]] * 300, dtype=torch.int32)
    ids[7, 1] = 8     # out of range
    ids[200, 0] = -3  # out of range
    lay = m.moe_layout(shape, ids.to(dev), ws=ws)
    st, detail = m.moe_get_device_error(ws)
    assert st == MOE_ERR_DEVICE_RANGE
    dp = to_np(lay.dst_pos)
    assert dp[7, 1] == -1 and dp[200, 0] == -1
    # the valid assignments keep their token-order rows
    assert dp[0, 0] == 0 and dp[0, 1] == 299
    assert m.moe_get_device_error(ws) == (0, 0)  # the read cleared it


def test_bad_rows_in_dispatch_and_combine_are_skipped():
    import combine_moe_route_07_b200 as m
    from combine_moe_route_07_b200._binding import MOE_ERR_DEVICE_RANGE
    w = Workload("badrow", T=4, H=16, E=4, R=1, k=1)
    shape = shape_of(w)
    dev = torch.device("cuda:0")
    ws = m.Workspace(shape, dev)
    x = torch.ones((4, 16), dtype=torch.bfloat16, device=dev)
    dst = torch.tensor([[0], [1], [2], [4]], dtype=torch.int32, device=dev)  # N = 4
    out = torch.zeros((4, 16), dtype=torch.bfloat16, device=dev)
    m.moe_dispatch(shape, x, dst, ws=ws, out=out)
    st, detail = m.moe_get_device_error(ws)
    assert st == MOE_ERR_DEVICE_RANGE and detail == 4
    assert to_np(out.float()).sum() == 3 * 16
    g = torch.ones((4, 1), dtype=torch.float32, device=dev)
    comb = m.moe_combine(shape, out, dst, g, ws=ws)
    st, _ = m.moe_get_device_error(ws)
    assert st == MOE_ERR_DEVICE_RANGE
    assert to_np(comb.float())[3].sum() == 0


def test_nan_logit_sets_the_device_error():
    import combine_moe_route_07_b200 as m
    from combine_moe_route_07_b200._binding import MOE_ERR_DEVICE_NAN
    w = Workload("nan", T=64, H=16, E=8, R=2, k=2)
    shape = shape_of(w)
    dev = torch.device("cuda:0")
    ws = m.Workspace(shape, dev)
    logits = torch.randn(64, 8)
    logits[17, 3] = float("nan")
    m.moe_route(shape, logits.to(dev), None, ws=ws)
    st, detail = m.moe_get_device_error(ws)
    assert st == MOE_ERR_DEVICE_NAN and detail == 17


def test_workspace_reuse_across_shapes_and_calls():
    """One workspace sized for the largest shape serves smaller ones, call
    after call (the layout leaves its lookback table zeroed)."""
    import combine_moe_route_07_b200 as m
    big = Workload("big", T=5000, H=16, E=64, R=8, k=4)
    ws = m.Workspace(shape_of(big), torch.device("cuda:0"))
    for T, E, k in ((5000, 64, 4), (130, 8, 2), (4999, 64, 4), (1, 16, 16), (5000, 64, 4)):
        w = Workload("reuse", T=T, H=16, E=E, R=2, k=k)
        inp = make_inputs(w)
        o = run_oracle(w, inp, through="layout")
        shape = shape_of(w)
        ids = torch.from_numpy(o["ids"]).cuda()
        lay = m.moe_layout(shape, ids, ws=ws)
        for key in LAYOUT_KEYS:
            assert np.array_equal(to_np(getattr(lay, key)), o["layout"][key]), (T, key)
    assert m.moe_get_device_error(ws) == (0, 0)
