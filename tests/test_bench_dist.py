"""Host-side logic of the multi-GPU bench (replicas, weak scaling), run as two
gloo ranks on the CPU: the max over ranks and the whole-job throughput."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        m = bench.max_over_ranks(times[rank], dist, "cpu")
        v = bench.whole_job_tokens_per_s(world, 4096, 10, m)
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    times = [12.5, 17.25]
    procs = [ctx.Process(target=_rank, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in got:
        assert m == 17.25  # every rank sees the slowest rank's time
        assert v == pytest.approx(2 * 4096 * 10 / 17.25e-3)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.whole_job_tokens_per_s(1, 100, 4, 2.0) == pytest.approx(100 * 4 / 2e-3)


def test_reference_arm_prints_one_line_and_other_ranks_stay_silent(capsys, monkeypatch):
    sys.path.insert(0, ROOT)
    import json
    import bench
    from combine_moe_route_07_b200.workloads import WORKLOADS
    args = bench.parse(["--gpus", "2", "--steps", "2", "--warmup", "1"])
    monkeypatch.setenv("RANK", "1")
    assert bench.run_reference(args, WORKLOADS["tiny"]) == 0
    assert capsys.readouterr().out == ""
    monkeypatch.setenv("RANK", "0")
    assert bench.run_reference(args, WORKLOADS["tiny"]) == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 1
    assert cb["host_cores"] == os.cpu_count() and cb["usable_cores"] >= 1
    assert "cpu_model" in cb and set(cb["stage_ms_per_step"]) == set(bench.STAGES)
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    w = WORKLOADS["tiny"]
    cfg = line["config"]
    assert (cfg["tokens"], cfg["hidden"], cfg["experts"], cfg["k"], cfg["ranks"]) == \
        (w.T, w.H, w.E, w.k, w.R)
    assert cfg["rows"] == w.rows and cfg["capacity"] == w.capacity
    assert line["metric"] == bench.METRIC and line["higher_is_better"] is True
    # the kernel arm prints the same config object for the same arguments
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert cfg == bench.bench_config(w, args, 2)


def test_step_plan_names_every_call_and_the_bias_update():
    """The calls a step makes, for every bench variant; the bias update sits
    before the combine whenever it is asked for."""
    import bench
    from combine_moe_route_07_b200.workloads import WORKLOADS
    w = WORKLOADS["prefill"]
    plan = lambda *a: bench.step_plan(w, bench.parse(list(a)))  # noqa: E731
    assert plan() == (("route_layout_dispatch", "combine"), False)
    assert plan("--path", "fused") == (("route_layout", "dispatch", "combine"), False)
    assert plan("--path", "separate")[0] == ("route", "layout", "dispatch", "combine")
    assert plan("--layout", "src") == (("route", "layout_src", "dispatch", "combine"), True)
    assert plan("--max-ranks", "2")[0][0] == "route_limited"
    assert plan("--router", "round_robin")[0][0] == "route_round_robin"
    assert plan("--home", "3")[0][1] == "layout_remote_first"
    for extra in ([], ["--path", "fused"], ["--path", "separate"], ["--layout", "src"]):
        names = plan("--bias-gamma", "0.01", *extra)[0]
        assert names[-2:] == ("bias_update", "combine")


def test_algorithmic_bytes_cover_every_step_name():
    """Every kernel name a bench path can report has a byte count."""
    import bench
    from combine_moe_route_07_b200.workloads import WORKLOADS
    names = {"route", "route_limited", "route_round_robin", "layout", "layout_src",
             "layout_remote_first", "dispatch", "combine", "bias_update", "route_layout",
             "route_layout_dispatch"}
    for w in WORKLOADS.values():
        for ww in (w, w.with_(align=128) if not w.capacity else w):
            b = bench.algorithmic_bytes(ww, ww.rows)
            assert names <= set(b), names - set(b)
            assert all(v > 0 for v in b.values())


def test_small_route_layout_rule_matches_the_library_constants():
    """The bench's launch count follows the library's choice of the one-launch
    route+layout; its limits are read from the kernel header."""
    import re
    import bench
    hdr = open(os.path.join(ROOT, "combine_moe_route_07_b200", "csrc", "kernels.h")).read()
    assign = int(re.search(r"kSmallMaxAssign = (\d+);", hdr).group(1))
    experts = int(re.search(r"kSmallMaxExperts = (\d+);", hdr).group(1))
    assert bench.small_route_layout(assign // 8, experts, 8)
    assert not bench.small_route_layout(assign // 8 + 1, experts, 8)
    assert not bench.small_route_layout(4, experts + 1, 2)
    assert not bench.small_route_layout(0, 8, 2)
    assert bench.kernels_per_step("fused3", False, False, True, False) == 3
    assert bench.kernels_per_step("fused3", False, False, False, False) == 4
    assert bench.kernels_per_step("fused3", False, False, False, True) == 5
    assert bench.kernels_per_step("separate", False, False, True, False) == 5
    assert bench.kernels_per_step("fused3", True, True, False, False) == 7
    assert bench.kernels_per_step("fused3", False, False, False, False, True) == 3
    assert bench.kernels_per_step("fused", False, False, False, False, True) == 4


def test_place_dispatch_rule_matches_the_library_constants():
    """The bench's copy of the place-and-dispatch kernel's limits equals the
    library's constants, and the rule picks the workloads it should."""
    import re
    import bench
    from combine_moe_route_07_b200.workloads import WORKLOADS
    hdr = open(os.path.join(ROOT, "combine_moe_route_07_b200", "csrc", "kernels.h")).read()
    src = open(os.path.join(ROOT, "combine_moe_route_07_b200", "csrc", "place_dispatch.cu")).read()
    const = lambda text, name: int(re.search(name + r" = (\d+)", text).group(1))  # noqa: E731
    assert bench.PD_MIN_TOKENS == const(hdr, "kPdMinTokens")
    assert bench.PD_PIPES == const(src, "kPdPipes")
    assert bench.PD_MAX_STAGES == const(src, "kPdMaxStages")
    assert bench.PD_WARPS * 32 == const(src, "kPdThreads")
    assert bench.PD_SMEM == const(src, "kPdSmemBudget") * 1024
    assert bench.PD_MAX_ASSIGN == const(src, "kPdMaxAssign")
    fits = {n: bench.place_dispatch_one_kernel(w.T, w.E, w.k, w.H, w.fp8, w.capacity, 148)
            for n, w in WORKLOADS.items()}
    assert fits == {"tiny": False, "prefill": True, "decode": False, "skewed_capacity": False,
                    "skewed_dropless": False, "finegrained": False}
