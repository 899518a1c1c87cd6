"""moe_layout_noalloc: the layout entry point for callers that cannot allocate
device memory (plugin hosts that pass only inputs and outputs, serving
runtimes whose pool owns the device, latency-critical code that may not call
cudaMalloc).  Its scratch is a static device array inside the library.

The GPU test calls it through the C ABI twice in a row on each shape and
checks both results bit for bit (the tolerance every layout test uses)
against the workspace-based moe_layout and against the oracle's layout of the
same ids.  This file is collected last so that a run
stopping at the first failure has run every other test already; it passes on
its own in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_07_b200 import _binding
from combine_moe_route_07_b200.workloads import WORKLOADS, Workload, make_inputs

FIELDS = ("counts", "expert_off", "rank_off", "rank_counts", "dst_pos", "src_idx")


def _shape_c(w):
    flags = (_binding.MOE_F_RENORM if w.renorm else 0) | (_binding.MOE_F_FP8 if w.fp8 else 0)
    return _binding.MoeShapeC(w.T, w.H, w.E, w.k, w.R, w.capacity, w.align, flags)


def _outputs(w, dev):
    i32 = dict(dtype=torch.int32, device=dev)
    return {"counts": torch.full((w.E,), -7, **i32), "expert_off": torch.full((w.E + 1,), -7, **i32),
            "rank_off": torch.full((w.R + 1,), -7, **i32), "rank_counts": torch.full((w.R,), -7, **i32),
            "dst_pos": torch.full((w.T, w.k), -7, **i32), "src_idx": torch.full((w.rows,), -7, **i32)}


def _ptrs(o):
    return [o[f].data_ptr() for f in FIELDS]


@pytest.mark.gpu
@pytest.mark.parametrize("w", [
    WORKLOADS["prefill"],
    WORKLOADS["finegrained"],
    WORKLOADS["decode"],
    Workload("skewed_capacity_8k", T=8192, H=128, E=256, R=32, k=8, zipf_s=1.2,
             capacity_factor=1.2),
    Workload("aligned", T=3000, H=64, E=64, R=8, k=4, align=128),
], ids=lambda w: w.name)
def test_noalloc_matches_workspace_layout_twice(w):
    import combine_moe_route_07_b200 as m
    lib = _binding.lib()
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    shape_py = m.MoeShape(tokens=w.T, hidden=w.H, experts=w.E, k=w.k, ranks=w.R,
                          capacity=w.capacity, align=w.align, renorm=w.renorm, fp8=w.fp8)
    inp = make_inputs(w)
    ws = m.Workspace(shape_py, dev)
    logits = inp.logits.to(dev)
    bias = None if inp.bias is None else inp.bias.to(dev)
    ids, _ = m.moe_route(shape_py, logits, bias, ws=ws)
    ref = m.moe_layout(shape_py, ids, ws=ws)
    m.moe_check(ws)
    want = {f: getattr(ref, f).cpu().numpy() for f in FIELDS}
    orc = oracle.layout(ids.cpu().numpy(), w.E, w.R, capacity=w.capacity, align=w.align)

    shape = _shape_c(w)
    for call in range(2):
        out = _outputs(w, dev)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info(dev)[0]
        st = lib.moe_layout_noalloc(ctypes.byref(shape), ids.data_ptr(), *_ptrs(out), stream)
        assert st == _binding.MOE_OK, _binding.status_string(st)
        torch.cuda.synchronize()
        if call == 1:  # set-up is done; the call itself reserves no device memory
            assert torch.cuda.mem_get_info(dev)[0] == free_before
        for f in FIELDS:
            got = out[f].cpu().numpy()
            assert np.array_equal(got, want[f]), (call, f)
            assert np.array_equal(got, orc[f]), (call, f, "oracle")


def test_noalloc_rejects_shapes_beyond_its_limit():
    lib = _binding.lib()
    fake = ctypes.c_void_p(0x1000)
    # two tables of 65 tiles x 1024 experts x 4 bytes > 512 KiB (E = 1024 allows T <= 1024)
    too_big = Workload("too_big", T=1025, H=128, E=1024, R=8, k=2)
    st = lib.moe_layout_noalloc(ctypes.byref(_shape_c(too_big)), fake, fake, fake, fake, fake,
                                fake, fake, None)
    assert st == _binding.MOE_ERR_UNSUPPORTED
    bad = Workload("bad", T=16, H=128, E=8, R=3, k=2)  # E % R != 0
    st = lib.moe_layout_noalloc(ctypes.byref(_shape_c(bad)), fake, fake, fake, fake, fake,
                                fake, fake, None)
    assert st == _binding.MOE_ERR_INVALID_ARG
