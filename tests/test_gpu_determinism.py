"""Determinism of the whole path and the failure path of the bounded waits.

Every entry point runs twice on the same inputs and must give identical bits
(integer layouts under heavy contention included, and the floating-point
combine, whose per-element slot order is fixed).  The timeout self-test makes
one bounded wait run out -- on a barrier nothing completes, no fault -- and
the error word must say so while the context stays usable."""
import numpy as np
import pytest
import torch

from combine_moe_route_07_b200.workloads import WORKLOADS, make_inputs
from pipeline import shape_of, to_np

pytestmark = pytest.mark.gpu


def _path(w, inp, dev):
    import combine_moe_route_07_b200 as m
    shape = shape_of(w)
    ws = m.Workspace(shape, dev)
    x = inp.x.to(dev)
    bias = inp.bias.to(dev) if inp.bias is not None else None
    ids, gates, lay = m.moe_route_layout(shape, inp.logits.to(dev), bias, ws=ws)
    xd = m.moe_dispatch(shape, x, lay.dst_pos, ws=ws)
    y = xd if not w.fp8 else (xd[0].float() * xd[1].repeat_interleave(128, dim=1)).to(torch.bfloat16)
    shared = inp.shared.to(dev) if w.shared else None
    out = m.moe_combine(shape, y, lay.dst_pos, gates, ws=ws, shared=shared,
                        residual=x if w.residual else None)
    torch.cuda.synchronize()
    assert m.moe_get_device_error(ws) == (0, 0)
    res = [to_np(ids), to_np(gates), to_np(lay.dst_pos), to_np(lay.src_idx), to_np(out)]
    if w.fp8:
        res += [to_np(xd[0].view(torch.uint8)), to_np(xd[1])]
    return res


@pytest.mark.parametrize("name,T", [("skewed_dropless", 6000), ("skewed_capacity", 6000),
                                    ("prefill", 4096), ("finegrained", 8192)])
def test_whole_path_twice_is_bit_identical(name, T):
    w = WORKLOADS[name].with_(T=T)
    inp = make_inputs(w)
    dev = torch.device("cuda:0")
    a = _path(w, inp, dev)
    b = _path(w, inp, dev)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_further_layouts_twice_are_bit_identical():
    import combine_moe_route_07_b200 as m
    T, E, k, R = 20000, 64, 8, 8
    rng = np.random.default_rng(0)
    p = np.arange(1, E + 1, dtype=np.float64) ** -1.2
    p /= p.sum()
    ids = torch.from_numpy(np.stack([rng.choice(E, size=k, replace=False, p=p)
                                     for _ in range(T)]).astype(np.int32)).cuda()
    src = m.MoeShape(tokens=T, hidden=16, experts=E, k=k, ranks=R, src_layout=True)
    ws = m.Workspace(src, ids.device)
    a = m.moe_layout_src(src, ids, ws=ws)
    b = m.moe_layout_src(src, ids, ws=ws)
    for key in ("dst_pos", "src_idx", "pair_counts", "seg_off"):
        assert torch.equal(getattr(a, key), getattr(b, key)), key
    plain = m.MoeShape(tokens=T, hidden=16, experts=E, k=k, ranks=R, align=128)
    ws2 = m.Workspace(plain, ids.device)
    c, tc = m.moe_layout_remote_first(plain, ids, 2, ws=ws2)
    d, td = m.moe_layout_remote_first(plain, ids, 2, ws=ws2)
    assert torch.equal(c.dst_pos, d.dst_pos) and torch.equal(tc, td)
    assert m.moe_get_device_error(ws) == (0, 0) and m.moe_get_device_error(ws2) == (0, 0)


def test_bounded_wait_that_runs_out_reports_a_timeout():
    import combine_moe_route_07_b200 as m
    from combine_moe_route_07_b200 import _binding
    dev = torch.device("cuda:0")
    shape = m.MoeShape(tokens=256, hidden=128, experts=8, k=2, ranks=4)
    ws = m.Workspace(shape, dev)
    st = _binding.lib().moe_selftest_wait_timeout(ws.ptr, 100000, torch.cuda.current_stream().cuda_stream)
    assert st == 0
    status, waited_us = m.moe_get_device_error(ws)
    assert status == _binding.MOE_ERR_DEVICE_TIMEOUT
    assert 50000 <= waited_us <= 2000000
    assert m.moe_get_device_error(ws) == (0, 0)  # read and cleared
    # the context is still usable: the whole path runs and matches itself
    w = WORKLOADS["tiny"]
    inp = make_inputs(w)
    assert all(np.array_equal(u, v) for u, v in zip(_path(w, inp, dev), _path(w, inp, dev)))


def test_timeout_selftest_rejects_bad_limits():
    import combine_moe_route_07_b200 as m
    from combine_moe_route_07_b200 import _binding
    shape = m.MoeShape(tokens=8, hidden=16, experts=8, k=2, ranks=2)
    ws = m.Workspace(shape, torch.device("cuda:0"))
    s = torch.cuda.current_stream().cuda_stream
    assert _binding.lib().moe_selftest_wait_timeout(ws.ptr, 0, s) == _binding.MOE_ERR_INVALID_ARG
    assert _binding.lib().moe_selftest_wait_timeout(ws.ptr, 3000000, s) == \
        _binding.MOE_ERR_INVALID_ARG
    assert _binding.lib().moe_selftest_wait_timeout(None, 100, s) == _binding.MOE_ERR_WORKSPACE
