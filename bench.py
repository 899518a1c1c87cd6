"""Benchmark: MoE route + layout + dispatch + combine on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill]
    python bench.py --impl reference ...        # the CPU oracle, timed as is

One step is one pass of the whole path over one batch: moe_route, moe_layout
(count + place kernels), moe_dispatch, moe_combine.  The expert FFN between
dispatch and combine is not part of the path; its output y (the workload's
stand-in expert applied to a warm-up dispatch of the same batch) is prepared
before the timed region, like the inputs.  L2 (126 MB): when the bytes one
step touches exceed twice the L2 the steps run back to back (no step can find
another's data in L2, and each step's dirty lines are written back during the
next, which is the steady state); otherwise a 256 MiB buffer is written and
then read between steps, outside the per-step CUDA events, so each step starts
from an L2 holding only clean, unrelated lines.  The step time is the sum of
the event intervals.

Prints ONE JSON line (rank 0).  With N > 1 (torchrun, one process per GPU)
every rank runs its own batch (weak scaling, no collective on the data path);
the reported time is the max over ranks.  On one GPU the line also carries a
`per_workload` block: the other workloads (tiny, decode, skewed with capacity
and dropless, fine-grained) each measured the same way with fewer steps, and
a `cpu_baseline` (the oracle on this host, with its core count, CPU model and
per-stage times).  Both arms print the same `config` object.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FALLBACK_HBM_GBS = 6650.0
METRIC = "dispatch+combine tokens/s at 1 B200; achieved HBM GB/s vs peak"


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=3000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["native", "reference"], default="native")
    p.add_argument("--workload", default="prefill")
    p.add_argument("--e2e-steps", type=int, default=200)
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--layout", choices=["expert", "src"], default="expert",
                   help="expert: rows by expert; src: the per-source-rank layout (rows by "
                        "destination rank, source shard, expert), route + layout_src + dispatch "
                        "+ combine as separate calls")
    p.add_argument("--max-ranks", type=int, default=0,
                   help="> 0: rank-limited routing (moe_route_limited), each token's experts from "
                        "at most this many ranks; route, layout, dispatch, combine as separate calls")
    p.add_argument("--bias-gamma", type=float, default=0.0,
                   help="> 0: each step also runs the aux-loss-free bias update "
                        "(moe_bias_update) with this step size; the bias feeds the next step's "
                        "route")
    p.add_argument("--router", choices=["learned", "round_robin"], default="learned",
                   help="round_robin: the diagnostic router (ids (t*k+j) mod E, gates 1/k) in "
                        "place of the learned one")
    p.add_argument("--home", type=int, default=-1,
                   help=">= 0: remote-first layout seen from this rank (moe_layout_remote_first)")
    p.add_argument("--align", type=int, default=0,
                   help="> 0: override the workload's segment alignment (e.g. 128-row tiles)")
    p.add_argument("--tokens", type=int, default=0,
                   help="override the workload's token count (smaller cases for profiler "
                        "captures; a changed workload, not a bench line)")
    p.add_argument("--path", choices=["fused3", "fused", "separate"], default="fused3",
                   help="steps 1-4 in one moe_route_layout_dispatch call; route+layout in one "
                        "moe_route_layout call; or one call per step")
    p.add_argument("--per-workload", default="tiny,decode,skewed_capacity,skewed_dropless,"
                                             "finegrained",
                   help="comma-separated workloads also measured (one GPU only) and reported "
                        "in the line's per_workload block; 'none' for none")
    p.add_argument("--per-workload-steps", type=int, default=50)
    return p.parse_args(argv)


# ------------------------------------------------------------ byte counts --

def algorithmic_bytes(w, kept_rows):
    """Bytes each step must move (the per-token figures of each step, summed over the
    rows actually kept)."""
    T, H, E, k = w.T, w.H, w.E, w.k
    row = 2 * H
    disp_row_out = (H + 4 * (H // 128)) if w.fp8 else row
    b = {}
    b["route"] = T * E * 4 + (4 * E if w.bias else 0) + T * k * 8
    b["route_limited"] = b["route"]
    b["bias_update"] = 12 * E  # counts in, bias in and out
    b["route_round_robin"] = T * k * 8  # ids and gates out
    b["layout"] = T * k * 4 * 2 + w.rows * 4 + (3 * E + 2 * w.R) * 4  # ids in, dst_pos/src_idx out
    b["layout_remote_first"] = b["layout"] + (w.rows // w.align) * 4  # + the tile map
    b["dispatch"] = T * row + kept_rows * disp_row_out + T * k * 4
    b["combine"] = kept_rows * row + T * k * 8 + T * row \
        + (T * row if w.shared else 0) + (T * row if w.residual else 0)
    # per-source-rank layout: ids in, dst_pos and src_idx out, the [R,E]
    # counts, the R*E+1 segment offsets and the [R,R] message sizes out
    b["layout_src"] = T * k * 4 * 2 + w.rows_src * 4 + (2 * w.R * E + 1 + w.R * w.R) * 4
    # fused route + layout: the ids stay in the CTA between the two steps
    b["route_layout"] = b["route"] + b["layout"] - T * k * 4
    b["route_layout_dispatch"] = b["route_layout"] + b["dispatch"] - T * k * 4
    return b


# ----------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi samples during the timed region (clocks, throttle reasons)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        self.sel = sel

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", *self.sel, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for name, val in zip(self.REASONS, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------ peaks --

def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def small_route_layout(T, E, k):
    """Whether moe_route_layout runs as one cluster launch instead of the route
    and place kernels (kSmallMaxAssign = 1024 assignments and kSmallMaxExperts
    = 512 experts in the library's kernels.h)."""
    return T > 0 and E <= 512 and T * k <= 1024


# the library's limits for placing and dispatching in one kernel behind the
# route kernel (kernels.h: kPdMinTokens; place_dispatch.cu: the pipelines, the
# stages and the shared-memory budget)
PD_MIN_TOKENS, PD_WARPS, PD_PIPES, PD_MAX_STAGES, PD_SMEM = 2048, 16, 4, 8, 200 * 1024
PD_MAX_ASSIGN = 512


def place_dispatch_one_kernel(T, E, k, H, fp8, capacity, num_sms):
    """Whether moe_route_layout_dispatch places and dispatches in one kernel
    (bf16 rows of 1-32 KiB, dropless, at least PD_MIN_TOKENS tokens, at most
    PD_MAX_ASSIGN assignments a CTA, within the shared-memory budget)."""
    row = 2 * H
    if fp8 or capacity > 0 or T < PD_MIN_TOKENS or row < 1024 or row > 32768:
        return False
    TB = -(-T // num_sms)
    if TB * k > PD_MAX_ASSIGN:
        return False
    ints = (PD_WARPS * E + 4 * E + 1 + 2 * TB * k) * 4
    if ints >= PD_SMEM:
        return False
    return min(PD_MAX_STAGES, (PD_SMEM - ints) // (PD_PIPES * row)) >= 2


def kernels_per_step(path, separate, src, small, bias_update, place_dispatch=False):
    """Kernels one step launches: route (1) + layout (count and place: 2; the
    per-source-rank layout 4) + dispatch + combine on the separate calls; the
    fused paths route and lay out in 2 kernels, or 1 for a small batch; the
    fused steps 1-4 place and dispatch in one kernel when the batch fits."""
    if separate:
        n = 1 + (4 if src else 2) + 2
    elif path == "separate":
        n = 5
    elif path == "fused3" and place_dispatch:
        n = 3
    else:
        n = (1 if small else 2) + 2
    return n + (1 if bias_update else 0)


def ncu_traffic(kernel, workload):
    """Per-launch DRAM bytes from the committed ncu summary, if one exists for
    this kernel and workload (profiles/ncu_traffic.txt: `kernel workload bytes`)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    try:
        with open(path) as f:
            for line in f:
                parts = line.split("#", 1)[0].split()
                if len(parts) >= 3 and parts[0] == kernel and parts[1] == workload:
                    return float(parts[2])
    except OSError:
        pass
    return None


# ------------------------------------------------------------ multi-rank --

def max_over_ranks(x: float, dist=None, device=None) -> float:
    """The max of a per-rank scalar (a device time) over all ranks."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(world: int, tokens_per_rank: int, steps: int, max_ms: float) -> float:
    """Weak scaling: every rank processes its own batch each step; the job's
    throughput is all ranks' tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (max_ms * 1e-3)


# ----------------------------------------------------------------- oracle --

def host_facts():
    """The host the oracle runs on: logical CPUs, the ones this process may
    use, and the CPU model string."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        usable = os.cpu_count()
    return {"host_cores": os.cpu_count(), "usable_cores": usable, "cpu_model": model}


STAGES = ("route", "layout", "dispatch", "combine")


def oracle_step_fn(w, inp, tokens):
    """One oracle pass of the path over the first `tokens` tokens (the expert
    output is prepared outside the returned closure, which returns the seconds
    each stage took)."""
    import numpy as np
    import oracle
    from combine_moe_route_07_b200.workloads import bf16_bits
    x = np.ascontiguousarray(bf16_bits(inp.x)[:tokens])
    sh = np.ascontiguousarray(bf16_bits(inp.shared)[:tokens]) if w.shared else None
    logits = np.ascontiguousarray(inp.logits.numpy()[:tokens])
    bias = None if inp.bias is None else inp.bias.numpy()
    cap = w.capacity if w.capacity == 0 else max(1, -(-w.capacity * tokens // w.T))
    ids, gates = oracle.route(logits, w.k, bias, renorm=w.renorm)
    L = oracle.layout(ids, w.E, w.R, capacity=cap, align=w.align)
    N = L["src_idx"].shape[0]
    if w.fp8:
        q, s = oracle.dispatch_fp8(x, L["dst_pos"], N)
        y = oracle.dequant_fp8(q, s)
    else:
        d = oracle.dispatch_bf16(x, L["dst_pos"], N)
        y = oracle.expert_scale(d, L["expert_off"], L["counts"], cap) \
            if w.expert == "scale" else d

    def step():
        t = [time.perf_counter()]
        i2, g2 = oracle.route(logits, w.k, bias, renorm=w.renorm)
        t.append(time.perf_counter())
        L2 = oracle.layout(i2, w.E, w.R, capacity=cap, align=w.align)
        t.append(time.perf_counter())
        if w.fp8:
            oracle.dispatch_fp8(x, L2["dst_pos"], N)
        else:
            oracle.dispatch_bf16(x, L2["dst_pos"], N)
        t.append(time.perf_counter())
        oracle.combine(y, L2["dst_pos"], g2, tokens, shared_bits=sh,
                       residual_bits=x if w.residual else None)
        t.append(time.perf_counter())
        return [b - a for a, b in zip(t, t[1:])]
    return step


def time_oracle(w, inp, budget_s, max_steps=None):
    """Time the oracle on a bounded sample: the whole batch if one pass fits
    the budget, else a prefix of tokens.  Returns (tokens/s, tokens, passes,
    seconds, per-stage milliseconds of one pass)."""
    tokens = w.T
    step = oracle_step_fn(w, inp, tokens)
    one = sum(step())
    if one > budget_s and tokens > 1:
        tokens = max(1, int(tokens * budget_s / one / 2))
        step = oracle_step_fn(w, inp, tokens)
    reps, elapsed = 0, 0.0
    stage = [0.0] * len(STAGES)
    while elapsed < budget_s and (max_steps is None or reps < max_steps):
        st = step()
        stage = [a + b for a, b in zip(stage, st)]
        elapsed += sum(st)
        reps += 1
    stage_ms = {n: round(v / reps * 1e3, 3) for n, v in zip(STAGES, stage)}
    return tokens * reps / elapsed, tokens, reps, elapsed, stage_ms


# ------------------------------------------------------------ the step plan --

def step_plan(w, args):
    """The calls one step makes, in order, and whether route and layout are
    separate calls because a variant asks for them (no device work here)."""
    src = args.layout == "src"
    M, RR, HOME, G = args.max_ranks, args.router == "round_robin", args.home, args.bias_gamma
    separate = src or M > 0 or RR or HOME >= 0
    if separate:
        names = ["route_round_robin" if RR else ("route_limited" if M > 0 else "route"),
                 "layout_src" if src else ("layout_remote_first" if HOME >= 0 else "layout"),
                 "dispatch", "combine"]
    elif args.path == "fused3":
        names = ["route_layout_dispatch", "combine"]
    elif args.path == "fused":
        names = ["route_layout", "dispatch", "combine"]
    else:
        names = ["route", "layout", "dispatch", "combine"]
    if G > 0:
        names.insert(names.index("combine"), "bias_update")
    return tuple(names), separate


L2_BYTES = 126 * 10**6


def touched_bytes(w, args, kept_rows):
    b = algorithmic_bytes(w, kept_rows)
    lay = "layout_src" if args.layout == "src" else "layout"
    return b["route"] + b[lay] + b["dispatch"] + b["combine"]


def flushes_between_steps(w, args):
    """Whether the steps are separated by an L2 flush: when a step touches
    less than twice the L2 (counted at the layout's static row count)."""
    return touched_bytes(w, args, w.rows) < 2 * L2_BYTES


def bench_config(w, args, world):
    """The `config` object of the JSON line; both arms print this same object."""
    names, _ = step_plan(w, args)
    src = args.layout == "src"
    touched = touched_bytes(w, args, w.rows)
    return {
        "workload": w.describe(), "tokens": w.T, "hidden": w.H, "experts": w.E, "k": w.k,
        "ranks": w.R, "capacity": w.capacity_src if src else w.capacity,
        "rows": w.rows_src if src else w.rows, "parallelism": f"replicas x{world}",
        "l2": ("256 MiB write + read between timed steps, outside the step events"
               if flushes_between_steps(w, args) else
               f"no flush: inputs larger than L2 ({touched / 1e6:.0f} MB touched per step vs "
               f"126 MB L2), steps back to back"),
        "layout": ("per-source-rank: rows by destination rank, source shard (R shards of "
                   "ceil(T/R) tokens), expert, token") if src else "rows by expert, token",
        "max_ranks": args.max_ranks if args.max_ranks > 0 else None,
        "bias_gamma": args.bias_gamma if args.bias_gamma > 0 else None,
        "router": args.router,
        "home_rank": args.home if args.home >= 0 else None,
        "step": " + ".join(names) + ", one CUDA graph",
    }


def run_reference(args, w):
    """The reference arm: the CPU oracle, as it stands, on this machine's host."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from combine_moe_route_07_b200.workloads import make_inputs
    inp = make_inputs(w)
    # each step is a bounded sample of the workload: a prefix of the batch
    # sized so that the timed steps take about a minute in all
    probe_tokens = max(1, w.T // 16)
    step = oracle_step_fn(w, inp, probe_tokens)
    per_token = sum(step()) / probe_tokens
    budget = 60.0 / max(1, args.steps + args.warmup)
    tokens = int(min(w.T, max(8, budget / per_token)))
    step = oracle_step_fn(w, inp, tokens)
    for _ in range(args.warmup):
        step()
    stage = [0.0] * len(STAGES)
    for _ in range(args.steps):
        stage = [a + b for a, b in zip(stage, step())]
    el = sum(stage)
    value = tokens * args.steps / el
    sample = f"first {tokens} of {w.T} tokens of the {w.name} batch per step, single thread"
    world = int(os.environ.get("WORLD_SIZE", str(getattr(args, "gpus", 1))))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8-e4m3 dispatch, bf16 rows, fp32 accumulate" if w.fp8 else "bf16",
        "data": "synthetic",
        "config": bench_config(w, args, world),
        "tokens_per_step": tokens,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": sample, **host_facts(),
                         "stage_ms_per_step": {n: round(v / args.steps * 1e3, 3)
                                               for n, v in zip(STAGES, stage)}},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- native --

class Path:
    """Device buffers and the calls of one step of one workload (the library's
    public API, torch only for memory and streams)."""

    def __init__(self, args, w, dev, seed):
        import torch
        import combine_moe_route_07_b200 as m
        from combine_moe_route_07_b200.workloads import make_inputs
        self.m, self.args, self.w, self.dev = m, args, w, dev
        self.inp = inp = make_inputs(w, seed=seed)
        src = self.src = args.layout == "src"
        shape = self.shape = m.MoeShape(
            tokens=w.T, hidden=w.H, experts=w.E, k=w.k, ranks=w.R,
            capacity=w.capacity_src if src else w.capacity, align=w.align, renorm=w.renorm,
            fp8=w.fp8, src_layout=src)
        ws = self.ws = m.Workspace(shape, dev)
        self.x = inp.x.to(dev)
        self.logits = inp.logits.to(dev)
        bias = None if inp.bias is None else inp.bias.to(dev)
        G = args.bias_gamma
        if G > 0 and bias is None:
            bias = torch.zeros(w.E, dtype=torch.float32, device=dev)
        self.bias = bias
        # the shared expert's output: a tensor of its own (not x), read by the combine
        self.shared = inp.shared.to(dev) if w.shared else None
        T, k, N = w.T, w.k, shape.rows
        i32 = dict(dtype=torch.int32, device=dev)
        ids = self.ids = torch.empty((T, k), **i32)
        gates = self.gates = torch.empty((T, k), dtype=torch.float32, device=dev)
        if src:
            lay = m.LayoutSrc(torch.empty((w.R, w.E), **i32), torch.empty(w.R * w.E + 1, **i32),
                              torch.empty((w.R, w.R), **i32), torch.empty(w.R + 1, **i32),
                              torch.empty(w.R, **i32), torch.empty((T, k), **i32),
                              torch.empty(N, **i32))
        else:
            lay = m.Layout(torch.empty(w.E, **i32), torch.empty(w.E + 1, **i32),
                           torch.empty(w.R + 1, **i32), torch.empty(w.R, **i32),
                           torch.empty((T, k), **i32), torch.empty(N, **i32))
        self.lay = lay
        if w.fp8:
            xd = torch.empty((N, w.H), dtype=torch.float8_e4m3fn, device=dev)
            sc = torch.empty((N, w.H // 128), dtype=torch.float32, device=dev)
        else:
            xd = torch.empty((N, w.H), dtype=torch.bfloat16, device=dev)
            sc = None
        self.xd, self.sc = xd, sc
        self.out = torch.empty((T, w.H), dtype=torch.bfloat16, device=dev)
        M, RR, HOME = args.max_ranks, args.router == "round_robin", args.home
        tile_expert = (torch.empty(N // w.align, dtype=torch.int32, device=dev) if HOME >= 0
                       else None)

        def route():
            if RR:
                m.moe_route_round_robin(shape, ids=ids, gates=gates)
            elif M > 0:
                m.moe_route_limited(shape, self.logits, M, bias, ws=ws, ids=ids, gates=gates)
            else:
                m.moe_route(shape, self.logits, bias, ws=ws, ids=ids, gates=gates)

        def layout():
            if src:
                m.moe_layout_src(shape, ids, ws=ws, out=lay)
            elif HOME >= 0:
                m.moe_layout_remote_first(shape, ids, HOME, ws=ws, out=lay,
                                          tile_expert=tile_expert)
            else:
                m.moe_layout(shape, ids, ws=ws, out=lay)

        def dispatch():
            m.moe_dispatch(shape, self.x, lay.dst_pos, ws=ws, out=xd, scales=sc)

        def combine():
            m.moe_combine(shape, self.y, lay.dst_pos, gates, ws=ws, shared=self.shared,
                          residual=self.x if w.residual else None, out=self.out)

        calls = {
            "route": route, "route_limited": route, "route_round_robin": route,
            "layout": layout, "layout_src": layout, "layout_remote_first": layout,
            "route_layout": lambda: m.moe_route_layout(shape, self.logits, bias, ws=ws, ids=ids,
                                                       gates=gates, out=lay),
            "route_layout_dispatch": lambda: m.moe_route_layout_dispatch(
                shape, self.logits, self.x, bias, ws=ws, ids=ids, gates=gates, lay=lay, out=xd,
                scales=sc),
            "dispatch": dispatch, "combine": combine,
            "bias_update": lambda: m.moe_bias_update(shape, lay.counts, G, bias),
        }
        self.names, self.separate = step_plan(w, args)
        self.ops = [calls[n] for n in self.names]
        # the per-kernel probe splits the fused steps 1-4 at the dispatch
        if self.names[0] == "route_layout_dispatch":
            self.probe_names = ("route_layout", "dispatch") + self.names[1:]
        else:
            self.probe_names = self.names
        self.probe_ops = [calls[n] for n in self.probe_names]
        self.calls = calls

        # the expert stand-in's output for this batch, prepared once (outside the path)
        route()
        layout()
        dispatch()
        if w.fp8:
            y = (xd.float() * sc.repeat_interleave(128, dim=1)).to(torch.bfloat16)
        elif w.expert == "scale":
            # expert of every row from src_idx (any row order); empty rows read expert 0
            e = ids.flatten()[lay.src_idx.clamp(min=0).long()].long()
            s = (torch.arange(1, w.E + 1, dtype=torch.float32, device=dev)
                 / torch.tensor(float(w.E), device=dev))[e]
            y = (xd.float() * s[:, None]).to(torch.bfloat16)
        else:
            y = xd.clone()
        self.y = y
        torch.cuda.synchronize()
        self.kept_rows = int(lay.rank_counts.sum().item())
        m.moe_check(ws)

    def step(self):
        for op in self.ops:
            op()

    def m_check(self):
        """Raise if a kernel recorded a device-side error."""
        self.m.moe_check(self.ws)


def _flush_fn(buf):
    """An L2 flush (a 256 MiB write, then a read that leaves L2 clean), or a
    no-op when buf is None."""
    import torch

    def flush():
        if buf is not None:
            buf.fill_(1)
            buf.view(torch.int64).sum()
    return flush


def capture_step(path, warmup, stream, flush):
    """Warm up eagerly, then capture the step as one CUDA graph: the step is
    launch-bound at its small kernels, and a graph replay is how the path is
    meant to be driven."""
    import torch
    dev = path.dev
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for _ in range(max(3, warmup)):
            flush()
            path.step()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        path.step()
    for _ in range(3):
        flush()
        g.replay()
    torch.cuda.synchronize()
    path.m_check()
    return g


def time_steps(g, K, stream, flush):
    """Per-step CUDA-event times (ms) of K graph replays, the L2 flush (when
    used) outside the events."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    for i in range(K):
        flush()
        ev[i][0].record(stream)
        g.replay()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def probe_kernels(path, K_ops, flush):
    """Per-call device time inside the step: a probe graph of the same step
    with event-record nodes between the calls, replayed after an L2 flush and
    read back one replay at a time; the mean over K_ops replays."""
    import torch
    dev = path.dev
    n = len(path.probe_ops)
    pev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n + 1)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cap = torch.cuda.current_stream(dev)
        pev[0].record(cap)
        for j, op in enumerate(path.probe_ops):
            op()
            pev[j + 1].record(cap)
    sums = [0.0] * n
    for _ in range(K_ops):
        flush()
        g.replay()
        torch.cuda.synchronize()
        for j in range(n):
            sums[j] += pev[j].elapsed_time(pev[j + 1])
    del g
    return [v / K_ops for v in sums]


def time_isolated(path, K_ops, iso_buf, stream):
    """Dispatch and combine each on its own: a 256 MiB L2 write + read-back
    before every launch (outside the events, so the dirty lines of the
    previous op are written back there); the median over K_ops launches."""
    import torch
    iso = {}
    for name in ("dispatch", "combine"):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            path.calls[name]()
        times = []
        for _ in range(K_ops):
            iso_buf.fill_(1)
            iso_buf.view(torch.int64).sum()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        del g
        iso[name] = sorted(times)[len(times) // 2]
    return iso


def dc_summary(w, kept_rows, t_disp, t_comb, peak):
    """Dispatch + combine: µs, GB/s and the fractions of the measured copy
    peak and of 8 TB/s, from the two ops' times in ms."""
    b = algorithmic_bytes(w, kept_rows)
    ms = t_disp + t_comb
    gbs = (b["dispatch"] + b["combine"]) / (ms * 1e-3) / 1e9
    return {"us": round(ms * 1e3, 2), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
            "frac_of_8tbs": round(gbs / 8000.0, 4)}


def measure_workload(args, w, dev, stream, peak, K, warmup):
    """A compact measurement of one more workload (one GPU): the step as one
    graph replayed K times, per-call times inside the step, and dispatch and
    combine each alone after an L2 flush."""
    import torch
    path = Path(args, w, dev, seed=w.seed)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush = _flush_fn(flush_buf if flushes_between_steps(w, args) else None)
    g = capture_step(path, warmup, stream, flush)
    times = time_steps(g, K, stream, flush)
    del g
    K_ops = 20
    mean = probe_kernels(path, K_ops, flush)
    iso = time_isolated(path, K_ops, flush_buf, stream)
    path.m_check()
    byts = algorithmic_bytes(w, path.kept_rows)
    ms = sum(times) / K
    t_disp = mean[path.probe_names.index("dispatch")]
    t_comb = mean[path.probe_names.index("combine")]
    kern = {}
    for s, name in enumerate(path.probe_names):
        gbs = byts[name] / (mean[s] * 1e-3) / 1e9
        kern[name] = {"us": round(mean[s] * 1e3, 2), "frac": round(gbs / peak, 4)}
    res = {
        "workload": w.describe(), "steps": K, "us_per_step": round(ms * 1e3, 2),
        "tokens_per_s": w.T / (ms * 1e-3), "rows": path.shape.rows,
        "kept_rows": path.kept_rows,
        "l2": "flushed between steps" if flushes_between_steps(w, args) else "steps back to back",
        "dispatch_combine_in_step": dc_summary(w, path.kept_rows, t_disp, t_comb, peak),
        "dispatch_combine_isolated": dc_summary(w, path.kept_rows, iso["dispatch"],
                                                iso["combine"], peak),
        "kernels_in_step": kern,
    }
    del path, flush_buf
    torch.cuda.empty_cache()
    return res


def main():
    args = parse()
    from combine_moe_route_07_b200.workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.tokens > 0:
        w = w.with_(name=f"{w.name}_t{args.tokens}", T=args.tokens)
    if args.align > 0:
        w = w.with_(name=f"{w.name}_a{args.align}", align=args.align)
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    import combine_moe_route_07_b200 as m

    path = Path(args, w, dev, seed=w.seed + rank)
    T, k, N = w.T, w.k, path.shape.rows
    kept_rows = path.kept_rows
    flush_between = flushes_between_steps(w, args)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush = _flush_fn(flush_buf if flush_between else None)

    g_step = capture_step(path, args.warmup, stream, flush)
    K = args.steps
    sampler = ClockSampler(local) if rank == 0 else None
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    times = time_steps(g_step, K, stream, flush)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    m.moe_check(path.ws)
    total_ms = max_over_ranks(sum(times), dist, dev)
    del g_step

    K_ops = max(20, min(400, K // 10))
    mean = probe_kernels(path, K_ops, flush)
    iso = time_isolated(path, K_ops, flush_buf, stream)

    # the achievable floor for the same bytes: a plain device-to-device copy
    # moving as many bytes (read + write) as dispatch and combine together,
    # timed the same way (flushed L2, median)
    _ab = algorithmic_bytes(w, kept_rows)
    copy_bytes = (_ab["dispatch"] + _ab["combine"]) // 2 // 16 * 16
    csrc = torch.empty(copy_bytes, dtype=torch.uint8, device=dev)
    cdst = torch.empty_like(csrc)
    csrc.fill_(3)
    ctimes = []
    for _ in range(K_ops):
        flush_buf.fill_(1)
        flush_buf.view(torch.int64).sum()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        cdst.copy_(csrc)
        b.record(stream)
        torch.cuda.synchronize()
        ctimes.append(a.elapsed_time(b))
    copy_ms = sorted(ctimes)[len(ctimes) // 2]
    del csrc, cdst

    # end to end through the public API: every step copies its inputs in from
    # pinned host memory and its result back out.  Pipelined the way a server
    # would run it: two device buffer sets, the next step's upload and the
    # previous step's download on their own streams, overlapping this step's
    # kernels (which stay strictly one step at a time).  64 such steps are
    # captured as one CUDA graph (copies, event edges and kernels) and
    # replayed, so host launch overhead does not stand in for the copies.
    e2e = None
    if args.e2e_steps > 0:
        inp = path.inp
        x_h = inp.x.pin_memory()
        lg_h = inp.logits.pin_memory()
        out_h = [torch.empty((T, w.H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        set_a = (path.x, path.logits, path.out)
        set_b = (torch.empty_like(path.x), torch.empty_like(path.logits),
                 torch.empty_like(path.out))
        sets = (set_a, set_b)
        U = 64
        cin, cout = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        path.x, path.logits, path.out = set_b
        set_b[0].copy_(path.inp.x)
        set_b[1].copy_(path.inp.logits)
        path.step()  # the second set's first pass, outside capture
        torch.cuda.synchronize()
        g_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_e2e):
            cap = torch.cuda.current_stream()
            evs = []
            for u in range(U):
                bset = u % 2
                xs, ls, os_ = sets[bset]
                h2d_e, done_e, d2h_e = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()
                with torch.cuda.stream(cin):
                    if u >= 2:
                        cin.wait_event(evs[u - 2][1])  # step u-2 has finished reading this set
                    else:
                        cin.wait_stream(cap)
                    xs.copy_(x_h, non_blocking=True)
                    ls.copy_(lg_h, non_blocking=True)
                    h2d_e.record(cin)
                cap.wait_event(h2d_e)
                if u >= 2:
                    cap.wait_event(evs[u - 2][2])  # step u-2's result has left this set
                path.x, path.logits, path.out = xs, ls, os_
                path.step()
                done_e.record(cap)
                with torch.cuda.stream(cout):
                    cout.wait_event(done_e)
                    out_h[bset].copy_(os_, non_blocking=True)
                    d2h_e.record(cout)
                evs.append((h2d_e, done_e, d2h_e))
            cap.wait_stream(cin)
            cap.wait_stream(cout)
        path.x, path.logits, path.out = set_a
        reps = max(1, -(-args.e2e_steps // U))
        for _ in range(2):
            g_e2e.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g_e2e.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / (reps * U), dist, dev)
        del g_e2e
        e2e = {"value": world * T / (e2e_ms * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": x_h.numel() * 2 + lg_h.numel() * 4,
               "d2h_bytes_per_step": out_h[0].numel() * 2, "ms_per_step": e2e_ms,
               "steps": reps * U,
               "mode": ("pipelined over two buffer sets: step i's kernels overlap step i+1's "
                        "upload and step i-1's download (pinned host memory, own streams); "
                        "64 steps per captured CUDA graph")}
    m.moe_check(path.ws)

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return 0

    byts = algorithmic_bytes(w, kept_rows)
    peak, peak_kind = hbm_peak()
    kern = {}
    for s, name in enumerate(path.probe_names):
        us = mean[s] * 1e3
        gbs = byts[name] / (mean[s] * 1e-3) / 1e9
        kern[name] = {"us": round(us, 2), "bytes": byts[name], "gbs": round(gbs, 1),
                      "frac": round(gbs / peak, 4)}
    t_disp = mean[path.probe_names.index("dispatch")]
    t_comb = mean[path.probe_names.index("combine")]
    dom = "dispatch" if t_disp >= t_comb else "combine"
    dom_gbs = byts[dom] / (max(t_disp, t_comb) * 1e-3) / 1e9
    dc = dc_summary(w, kept_rows, t_disp, t_comb, peak)
    dci = dc_summary(w, kept_rows, iso["dispatch"], iso["combine"], peak)
    ms_step = total_ms / K
    line = {
        "metric": METRIC,
        "value": whole_job_tokens_per_s(world, T, K, total_ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8-e4m3 dispatch, bf16 rows, fp32 accumulate" if w.fp8 else "bf16",
        "data": "synthetic",
        "config": bench_config(w, args, world),
        "kept_rows": kept_rows,
        "dispatch_combine": {"tokens_per_s": world * T / ((t_disp + t_comb) * 1e-3), **dc,
                             "method": (f"in the step: a replay of the step with event records "
                                        f"between its kernels (no launch overlap across them), "
                                        f"mean of {K_ops}; a fused steps 1-4 call is timed as "
                                        f"moe_route_layout then moe_dispatch")},
        "copy_anchor": {
            "bytes_moved": 2 * copy_bytes, "us": round(copy_ms * 1e3, 2),
            "gbs": round(2 * copy_bytes / (copy_ms * 1e-3) / 1e9, 1),
            "dispatch_combine_over_copy": round((iso["dispatch"] + iso["combine"]) / copy_ms, 3),
            "method": ("torch device-to-device copy of the same bytes as dispatch + combine "
                       "(half read, half written), flushed L2, median")},
        "dispatch_combine_isolated": {
            "tokens_per_s": world * T / ((iso["dispatch"] + iso["combine"]) * 1e-3), **dci,
            "dispatch_us": round(iso["dispatch"] * 1e3, 2),
            "combine_us": round(iso["combine"] * 1e3, 2),
            "method": (f"each op alone as a one-kernel CUDA graph, median of {K_ops}, "
                       "256 MiB L2 write + read-back before each launch outside the events")},
        "kernels": kern,
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(dom_gbs, 1),
                     "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs (copy)",
                     "unit": "GB/s", "frac": round(dom_gbs / peak, 4),
                     "traffic": ncu_traffic(dom, w.name)},
        "gpu_launches": kernels_per_step(
            args.path, path.separate, path.src, small_route_layout(T, w.E, k),
            args.bias_gamma > 0,
            place_dispatch_one_kernel(T, w.E, k, w.H, w.fp8, path.shape.capacity,
                                      torch.cuda.get_device_properties(dev).multi_processor_count)
        ) * K,
        "clocks": clocks,
        "e2e": e2e,
    }
    if not args.no_cpu_baseline and world == 1:
        v, tokens, reps, el, stage_ms = time_oracle(w, path.inp, args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{reps} single-threaded oracle passes over the first {tokens} of "
                      f"{T} tokens of the same batch ({el:.1f} s)",
            **host_facts(), "stage_ms_per_pass": stage_ms}
    del path, flush_buf
    torch.cuda.empty_cache()
    others = [n for n in args.per_workload.split(",") if n and n != "none" and n != w.name]
    if world == 1 and others:
        per = {}
        for name in others:
            per[name] = measure_workload(args, WORKLOADS[name], dev, stream, peak,
                                         args.per_workload_steps, args.warmup)
        line["per_workload"] = per
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
