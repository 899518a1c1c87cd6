"""Each workload's full path as the FIRST call of a fresh process.

A kernel whose dynamic shared memory is near or above the default 48 KiB
limit needs that limit raised before its first launch; inside one test
process an earlier, larger launch can hide a missing raise, so each case
runs in a process of its own."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

SCRIPT = r"""
import sys
sys.path[:0] = [{root!r}, {here!r}]
import numpy as np
from combine_moe_route_07_b200.workloads import WORKLOADS
from pipeline import inputs_for, run_gpu, to_np
import combine_moe_route_07_b200 as m
w = WORKLOADS[{name!r}]
inp = inputs_for(w)
g = run_gpu(w, inp, fused={fused!r})
assert m.moe_get_device_error(g["ws"]) == (0, 0)
print("ok", int(np.asarray(to_np(g["layout"].rank_counts)).sum()))
"""


@pytest.mark.parametrize("fused", [False, "dispatch"], ids=["separate", "fused3"])
@pytest.mark.parametrize("name", ["tiny", "decode", "prefill"])
def test_first_call_in_a_fresh_process(name, fused):
    code = SCRIPT.format(root=ROOT, here=HERE, name=name, fused=fused)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert r.stdout.startswith("ok")
