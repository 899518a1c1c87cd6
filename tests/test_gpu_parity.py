"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

Tolerances (from the arithmetic, stated once here):
  ids, counts, offsets, dst_pos, src_idx, dispatched bf16 rows, e4m3 codes and
  fp32 scales: bit-exact (integer work, copies, and fp32 decisions taken in the
  same precision on both sides);
  gates: 1e-6 relative (GPU fp64 softmax with a reciprocal-multiply, rounded to
  fp32 once, vs the oracle's fp64 division: at most one fp32 ulp apart);
  combine: bit for bit against the oracle's fixed-order binary32 accumulation
  (slot FMAs, then shared, then residual, one bf16 rounding: the arithmetic
  the kernels are specified with), and within one bf16 quantum plus the
  binary32 bound (k+2) * 2^-24 * sum|terms| of the exact sum (one bf16 ulp
  wherever the terms do not cancel); see pipeline.assert_combine.
"""
import numpy as np
import pytest
import torch

from combine_moe_route_07_b200.workloads import WORKLOADS, bf16_bits
from pipeline import (assert_combine, assert_gates_close, bf16_quantum, bf16_value,
                      gate_rows_equal, inputs_for, oracle_chunk, run_gpu, run_oracle, to_np)

pytestmark = pytest.mark.gpu

SMALL = ["tiny", "prefill", "decode"]
BIG = ["skewed_capacity", "skewed_dropless", "finegrained"]
LAYOUT_KEYS = ("counts", "expert_off", "rank_off", "rank_counts", "dst_pos", "src_idx")


def _compare_layout(g_lay, L, what):
    for key in LAYOUT_KEYS:
        got = to_np(getattr(g_lay, key))
        assert np.array_equal(got, L[key]), f"{what}: layout.{key} differs"


@pytest.mark.parametrize("fused", [False, True, "dispatch"], ids=["separate", "fused", "fused3"])
@pytest.mark.parametrize("name", SMALL)
def test_full_path_small_configs(name, fused):
    w = WORKLOADS[name]
    inp = inputs_for(w)
    o = run_oracle(w, inp)
    g = run_gpu(w, inp, fused=fused)
    import combine_moe_route_07_b200 as m
    assert m.moe_get_device_error(g["ws"]) == (0, 0)
    assert np.array_equal(to_np(g["ids"]), o["ids"])
    assert_gates_close(to_np(g["gates"]), o["gates"])
    _compare_layout(g["layout"], o["layout"], name)
    assert np.array_equal(to_np(g["dispatch"]), o["dispatch"])
    assert_combine(to_np(g["out"]), o, w.k, name,
                   exact_rows=gate_rows_equal(to_np(g["gates"]), o["gates"]))


@pytest.mark.parametrize("name", SMALL)
def test_each_kernel_on_oracle_inputs(name):
    """Feed the oracle's intermediates to the GPU path so each kernel is
    checked on its own (layout on the oracle's ids, combine on the oracle's
    expert outputs and gates)."""
    import combine_moe_route_07_b200 as m
    from pipeline import shape_of
    w = WORKLOADS[name]
    inp = inputs_for(w)
    o = run_oracle(w, inp)
    g = run_gpu(w, inp, ids=o["ids"], gates=o["gates"])
    _compare_layout(g["layout"], o["layout"], name)
    shape = shape_of(w)
    dev = g["x"].device
    y = torch.from_numpy(o["y"].view(np.int16)).view(torch.bfloat16).to(dev)
    dst = torch.from_numpy(o["layout"]["dst_pos"]).to(dev)
    gates = torch.from_numpy(o["gates"]).to(dev)
    out = m.moe_combine(shape, y, dst, gates, ws=g["ws"], shared=g["shared"],
                        residual=g["x"] if w.residual else None)
    assert_combine(to_np(out), o, w.k, name)


def _payload_every_token(w, g, o, name):
    """Dispatch and combine of every token against the oracle, a chunk of
    tokens at a time: the dispatched rows (bf16, or e4m3 codes and fp32
    scales) bit for bit, the combine as assert_combine states (and >= 99.9 %
    of it within one bf16 ulp of the exact sum).  With FP8 rows, also the
    combine against the unquantised rows: within 16/448 of each 128-channel
    block's max (the largest rounding of the e4m3 recipe) plus a bf16
    quantum of each side."""
    dst = o["layout"]["dst_pos"]  # equal to the GPU's (checked before)
    dev = g["x"].device
    chunk = max(256, (8 << 20) // w.H)  # tokens per oracle call
    same_gates = gate_rows_equal(to_np(g["gates"]), o["gates"])
    near = total = 0
    for t0 in range(0, w.T, chunk):
        t1 = min(w.T, t0 + chunk)
        tok = np.arange(t0, t1, dtype=np.int32)
        want = oracle_chunk(w, o["x"], o["ids"], o["gates"], dst, tok, o.get("shared"))
        keep = want["keep"].reshape(-1)
        idx = torch.from_numpy(np.where(want["keep"], dst[tok], 0).reshape(-1)).long().to(dev)
        if w.fp8:
            q_got = to_np(g["dispatch"][0].index_select(0, idx))
            s_got = to_np(g["dispatch"][1].index_select(0, idx))
            assert np.array_equal(q_got[keep], want["dispatch"][0][keep]), (name, t0, "codes")
            assert np.array_equal(s_got[keep], want["dispatch"][1][keep]), (name, t0, "scales")
        else:
            got = to_np(g["dispatch"].index_select(0, idx))
            assert np.array_equal(got[keep], want["dispatch"][keep]), (name, t0, "rows")
        got = to_np(g["out"][t0:t1])
        d = assert_combine(got, want, w.k, f"{name} tokens {t0}..", exact_rows=same_gates[t0:t1])
        if w.fp8:  # against the unquantised rows: within the e4m3 recipe's rounding
            ref = bf16_value(want["out_unquantised"])
            err = np.abs(bf16_value(got) - ref)
            slack = bf16_quantum(ref) + bf16_quantum(bf16_value(got))
            assert np.all(err <= want["fp8_bound"] + slack), (name, t0, "fp8 recipe bound")
        near += int((d <= 1).sum())
        total += d.size
    assert near / total > 0.999, (name, near, total)


@pytest.mark.slow
@pytest.mark.parametrize("fused", [False, True, "dispatch"], ids=["separate", "fused", "fused3"])
@pytest.mark.parametrize("name", BIG)
def test_full_size_every_token(name, fused):
    """The full-size batches: route and layout exact, and the dispatched
    payload and the combine of every token against the oracle.  The fused
    route + layout call feeds the same dispatch and combine launches as the
    separate calls, so its payload pass is left to those two."""
    import combine_moe_route_07_b200 as m
    w = WORKLOADS[name]
    inp = inputs_for(w)
    o = run_oracle(w, inp, through="layout")
    o["shared"] = bf16_bits(inp.shared) if w.shared else None
    g = run_gpu(w, inp, fused=fused)
    assert m.moe_get_device_error(g["ws"]) == (0, 0)
    assert np.array_equal(to_np(g["ids"]), o["ids"])
    assert_gates_close(to_np(g["gates"]), o["gates"])
    _compare_layout(g["layout"], o["layout"], name)
    if fused is not True:
        _payload_every_token(w, g, o, name)


def test_layout_is_deterministic_under_contention():
    import combine_moe_route_07_b200 as m
    from pipeline import shape_of
    w = WORKLOADS["skewed_dropless"].with_(T=8192)
    inp = inputs_for(WORKLOADS["skewed_dropless"])
    dev = torch.device("cuda:0")
    shape = shape_of(w)
    ws = m.Workspace(shape, dev)
    logits = inp.logits[: w.T].contiguous().to(dev)
    ids, _ = m.moe_route(shape, logits, None, ws=ws)
    a = m.moe_layout(shape, ids, ws=ws)
    outs = [[to_np(getattr(a, key)) for key in LAYOUT_KEYS]]
    for _ in range(3):
        b = m.moe_layout(shape, ids, ws=ws)
        outs.append([to_np(getattr(b, key)) for key in LAYOUT_KEYS])
    for other in outs[1:]:
        for u, v in zip(outs[0], other):
            assert np.array_equal(u, v)
    assert m.moe_get_device_error(ws) == (0, 0)
