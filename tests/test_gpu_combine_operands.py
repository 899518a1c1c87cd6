"""The combine's two extra operands, told apart.

The combine adds two rows besides the gate-weighted expert outputs: the
always-on shared expert's output ("19. All-to-all", section "Why Qwen3.8's
512 experts is a systems statement": 10 routed experts plus one shared one)
and the residual, the layer input x ("MoE All-to-All Dispatch and Ragged
Routing", section "Returning Tokens to the Original GPU": x + dx).  Here the
shared expert's output is a seeded draw of its own, so the two operands
differ element by element, and every combine variant is checked with both,
with each one alone and with neither:

  bulk-fed combine, k = 8  (dense Prefill shape; 16 or 24 warps per SM
                            depending on how many extra rows a stage holds)
  bulk-fed combine, k = 10 (Fine-grained shape, FP8 experts)
  register combine, all slots in flight (Decode, and a dense batch below
                            the bulk variant's size threshold)
  register combine, kept slots only (capacity layouts: wide rows of a
                            skewed batch, and narrow rows)
  staged combine (dense layouts with rows wider than 8 KiB and at least 8
                            row slices per SM: a ring of stages per CTA; rows
                            cut into slices, k = 16, whole rows)

The sum is commutative up to fp32 rounding, so an exchange of the two
operands' order cannot be seen at bf16 precision; what these tests catch is
an operand read twice, dropped, or taken from the wrong token or slice.
`test_inputs_tell_the_operands_apart` shows, on the CPU, that each of those
mistakes moves most outputs by more than the 1-ulp tolerance.

Tolerance (as in every combine test, pipeline.assert_combine): bit for bit
against the oracle's fixed-order binary32 accumulation, and within one bf16
quantum plus the binary32 error bound of the exact sum.  With a shared row
and a residual that are independent draws, the sum sometimes nearly cancels;
there the bound, not one ulp, is what any binary32 accumulation can promise.
"""
import numpy as np
import pytest
import torch

from combine_moe_route_07_b200.workloads import WORKLOADS, Workload, make_inputs
from pipeline import (assert_combine, bf16_ulp_diff, gate_rows_equal, run_gpu, run_oracle,
                      shape_of, to_np)

BOTH = dict(shared=True, residual=True)
CASES = [
    WORKLOADS["prefill"].with_(name="prefill_shared_residual", **BOTH),
    WORKLOADS["prefill"].with_(name="prefill_shared_only", shared=True),
    WORKLOADS["prefill"].with_(name="prefill_residual_only", residual=True),
    WORKLOADS["finegrained"].with_(name="finegrained_8k", T=8192),
    WORKLOADS["finegrained"].with_(name="finegrained_8k_shared_only", T=8192, residual=False),
    WORKLOADS["finegrained"].with_(name="finegrained_8k_residual_only", T=8192, shared=False),
    WORKLOADS["decode"].with_(name="decode_shared_residual", **BOTH),
    Workload("dense_1k_shared_residual", T=1024, H=4096, E=128, R=16, k=8, expert="scale",
             **BOTH),
    WORKLOADS["skewed_capacity"].with_(name="skewed_capacity_4k_shared_residual", T=4096,
                                       **BOTH),
    WORKLOADS["skewed_capacity"].with_(name="skewed_capacity_4k_residual_only", T=4096,
                                       residual=True),
    Workload("capacity_narrow_shared_residual", T=3000, H=512, E=32, R=4, k=4,
             capacity_factor=1.0, zipf_s=1.2, **BOTH),
    # staged combine (rows wider than 8 KiB): rows cut into three 4784-byte
    # slices, the last 4768
    Workload("ragged_slices_shared_residual", T=1200, H=7168, E=64, R=8, k=8, **BOTH),
    # staged combine: k = 16 plus both extra rows, 18 slots of 3424 bytes a stage
    Workload("k16_wide_shared_residual", T=600, H=5120, E=64, R=8, k=16, **BOTH),
    # staged combine: whole 9 KiB rows, exactly 8 units per CTA
    Workload("eight_units_per_cta_residual", T=148 * 8, H=4608, E=32, R=4, k=4, residual=True),
    # bulk combine with k = 16 plus both extra rows
    Workload("k16_narrow_shared_residual", T=5000, H=1024, E=64, R=8, k=16, **BOTH),
]


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.gpu
@pytest.mark.parametrize("fused", [False, "dispatch"], ids=["separate", "fused3"])
@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_whole_path_with_distinct_shared_and_residual(w, fused):
    import combine_moe_route_07_b200 as m
    inp = make_inputs(w)
    o = run_oracle(w, inp)
    g = run_gpu(w, inp, fused=fused)
    assert m.moe_get_device_error(g["ws"]) == (0, 0)
    d = assert_combine(to_np(g["out"]), o, w.k, w.name,
                       exact_rows=gate_rows_equal(to_np(g["gates"]), o["gates"]))
    assert (d <= 1).mean() > 0.999


@pytest.mark.gpu
@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_combine_on_oracle_operands(w):
    """moe_combine alone on the oracle's expert outputs, gates and layout,
    with the shared and residual rows passed as separate device tensors."""
    import combine_moe_route_07_b200 as m
    inp = make_inputs(w)
    o = run_oracle(w, inp)
    shape = shape_of(w)
    ws = m.Workspace(shape, torch.device("cuda:0"))
    y = _dev_bf16(o["y"])
    dst = torch.from_numpy(o["layout"]["dst_pos"]).cuda()
    gates = torch.from_numpy(o["gates"]).cuda()
    sh = _dev_bf16(o["shared"]) if w.shared else None
    rs = _dev_bf16(o["x"]) if w.residual else None
    out = m.moe_combine(shape, y, dst, gates, ws=ws, shared=sh, residual=rs)
    torch.cuda.synchronize()
    assert m.moe_get_device_error(ws) == (0, 0)
    d = assert_combine(to_np(out), o, w.k, w.name)
    assert (d <= 1).mean() > 0.999


def test_inputs_tell_the_operands_apart():
    """CPU only: with the shared output drawn on its own, reading one operand
    twice, dropping one, or taking a neighbouring token's row changes most
    outputs by more than the tolerance, so the GPU tests above would fail on
    any of those mistakes."""
    import oracle
    w = Workload("operands", T=512, H=256, E=16, R=4, k=4, **BOTH)
    inp = make_inputs(w)
    o = run_oracle(w, inp)
    x, sh = o["x"], o["shared"]
    assert (x != sh).mean() > 0.99
    args = (o["y"], o["layout"]["dst_pos"], o["gates"], w.T)
    right = o["out"]
    wrong = {
        "shared twice": oracle.combine(*args, shared_bits=sh, residual_bits=sh),
        "residual twice": oracle.combine(*args, shared_bits=x, residual_bits=x),
        "no shared": oracle.combine(*args, residual_bits=x),
        "no residual": oracle.combine(*args, shared_bits=sh),
        "next token's shared": oracle.combine(*args, shared_bits=np.roll(sh, 1, axis=0),
                                              residual_bits=x),
    }
    for what, out in wrong.items():
        assert (bf16_ulp_diff(out, right) > 1).mean() > 0.9, what
    # the order of the two additions is invisible at bf16 precision
    swapped = oracle.combine(*args, shared_bits=x, residual_bits=sh)
    assert (bf16_ulp_diff(swapped, right) > 1).sum() == 0
