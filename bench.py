#!/usr/bin/env python
"""Benchmark of the fused MoE FFN layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one call of the whole layer (route -> permute -> fc1 + SwiGLU -> fc2 ->
combine) on one batch of synthetic tokens with the inputs resident in HBM.  The
default workload is decode_bf16 (T=4, H=2816, E=128, k=8, I=704), the configuration
the layer's headline metric is quoted on; --workload picks another row of
synth.WORKLOADS.  Steps are replayed from CUDA graphs of S steps each; between
reuses of a weight set, `--sets` - 1 other copies of the weights are streamed, so
the touched weights never sit in L2 when a step starts.

Prints ONE JSON line (rank 0).  Multi-GPU (torchrun, one rank per GPU) runs
independent replicas: the layer has no exchange step on one GPU's batch, so there
is no data-path collective; the barrier and the max-over-ranks timing are the only
communication.  `--impl reference` times the CPU oracle (the reference arm of this
build) on the host cores instead.
"""
import argparse
import datetime
import json
import math
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s + TFLOP/s or HBM GB/s as fraction of roofline, 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DEFAULT_STEPS = {"tiny_fp32": 2000, "decode_bf16": 6000, "batched_decode_bf16": 2000,
                 "prefill_bf16": 400, "long_prefill_bf16": 100}
GRAPH_STEPS = {"tiny_fp32": 20, "decode_bf16": 20, "batched_decode_bf16": 20,
               "prefill_bf16": 4, "long_prefill_bf16": 2}
HBM_BOUND = {"decode_bf16", "batched_decode_bf16", "tiny_fp32"}
SWIGLU_PRESETS = {"standard": (1.0, 0.0, float("inf")), "gpt_oss": (1.702, 1.0, 7.0)}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode_bf16")
    ap.add_argument("--sets", type=int, default=None, help="rotating weight copies (L2)")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--swiglu", choices=list(SWIGLU_PRESETS), default="standard",
                    help="SwiGLU attributes (alpha, beta, limit) of the op")
    ap.add_argument("--expert-bias", action="store_true", help="with fc1/fc2 expert biases")
    ap.add_argument("--pre-norm", action="store_true",
                    help="the layer's input is a residual activation normalised by the pre-FFN "
                         "RMSNorm inside the call")
    ap.add_argument("--q8", action="store_true",
                    help="weight-only int8 experts (one float32 scale per weight row); "
                         "decode workloads only")
    ap.add_argument("--fc1-convert", action="store_true",
                    help="convert chunked fc1 to the interleaved layout at set-up instead of "
                         "reading it in place")
    return ap.parse_args(argv)


# --------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def job_throughput(tokens_per_rank, world, ms_per_step):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's step time."""
    return tokens_per_rank * world / ms_per_step * 1e3


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def max_over_ranks(x, world, device=None):
    """Max of a float over all ranks (identity for one rank)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms in the background."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.file = None
        self.t0 = self.t1 = None

    def start(self):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"], stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(1.0)

    def mark(self, begin):
        if begin:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.file.flush()
        rows = []
        with open(self.file.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        # the rows of the timed region: the busiest (highest power) contiguous half
        def num(s):
            try:
                return float(s)
            except ValueError:
                return float("nan")
        power = [num(r[3]) for r in rows]
        thr = sorted(power)[len(power) // 2] if len(power) > 2 else -1
        load = [r for r, p in zip(rows, power) if p >= thr] or rows
        sm = sorted(num(r[1]) for r in load)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": num(load[0][2]), "reasons": reasons,
                "samples": len(load), "power_w_max": max(num(r[3]) for r in load)}


NORM_EPS = 1e-6


def algorithmic(wl, counts, pre_norm=False, q8=False):
    """Algorithmic bytes and FLOPs of one step (only the routed work, used experts once;
    with the pre-FFN norm, its read of the residual and the weight and its write)."""
    T, H, E, k, I = wl.T, wl.H, wl.E, wl.k, wl.I
    es = 2 if wl.dtype == "bf16" else 4
    rows = T * k
    used = int(sum(1 for c in counts if c > 0))
    fc1 = {"bytes": used * 2 * I * H * es + rows * H * es + rows * I * es,
           "flops": 2.0 * rows * H * 2 * I}
    fc2 = {"bytes": used * H * I * es + rows * I * es + rows * H * es,
           "flops": 2.0 * rows * I * H}
    layer = {"bytes": used * 3 * H * I * es + E * H * es + 2 * T * H * es
             + 2 * rows * H * es + 2 * rows * I * es + 2 * rows * H * es,
             "flops": float(T) * (6.0 * k * H * I + 2.0 * H * E)}
    if pre_norm:
        layer["bytes"] += 2 * T * H * es + H * es
    if q8:
        # int8 weights (1 byte each) and a float32 scale per weight row
        for d, n_rows, n_cols in ((fc1, 2 * I, H), (fc2, H, I)):
            d["bytes"] -= used * n_rows * n_cols * (es - 1)
            d["bytes"] += used * n_rows * 4
        layer["bytes"] -= used * 3 * H * I * (es - 1)
        layer["bytes"] += used * (2 * I + H) * 4
    return used, fc1, fc2, layer


def kernel_source(one_launch_or_decode):
    """Source file of the dominant kernel: the decode FFN (gemm_tc.cu) or the CTA-pair
    grouped GEMM (gemm_pair.cu)."""
    name = "gemm_tc.cu" if one_launch_or_decode else "gemm_pair.cu"
    return os.path.join(ROOT, "mixture_experts_ffn_15_b200", "csrc", name)


def source_sha(path):
    import hashlib
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def kernel_traffic(workload, src):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary
    (profiles/traffic.json), if that summary was taken on the current source of the
    kernel; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    e = table.get(workload)
    if not e or e.get("source_sha") != source_sha(src):
        return None
    return e.get("bytes_per_launch")


def device_tensor(a, dev):
    """numpy storage array (uint16 bf16 bits or float32) -> torch tensor on `dev`."""
    import numpy as np
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


# --------------------------------------------------------------------------- CPU oracle

def q8_getters(q8_host):
    """Oracle weight getters of int8 experts: q * scale of each row, float64."""
    from oracle import moe_oracle as O
    q1, s1, q2, s2 = q8_host
    return (lambda e: O.dequantize_rows(q1[e], s1[e]), lambda e: O.dequantize_rows(q2[e], s2[e]))


def oracle_cost(wl, inp, seconds, pre=None, q8_host=None):
    """The CPU oracle, as it stands, on whole tokens of `wl` for about `seconds` (with
    pre = (residual values, norm weight values), each token through the pre-FFN norm
    first).

    Returns (tokens/s, threads, description of the sample)."""
    import numpy as np
    from threadpoolctl import threadpool_info

    from oracle import moe_oracle as O
    cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    x = inp.values("hidden")
    rw = inp.values("router_w")
    bias = inp["router_bias"]
    fc1 = lambda e: inp.expert_values("fc1", e)
    fc2 = lambda e: inp.expert_values("fc2", e)
    if q8_host is not None:
        fc1, fc2 = q8_getters(q8_host)
    t0 = time.perf_counter()
    n = 0
    while True:
        t = n % wl.T
        xt = x[t:t + 1] if pre is None else O.pre_ffn_norm(pre[0][t:t + 1], pre[1], NORM_EPS,
                                                           wl.dtype)
        r = O.moe_forward(xt, rw, bias, fc1, fc2, wl.k, wl.normalize, wl.fc1_layout)
        assert np.isfinite(r["out"]).all()
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    el = time.perf_counter() - t0
    return n / el, cores, (f"{n} whole tokens of the workload, one at a time (router logits, "
                           f"top-k, {wl.k} expert FFNs, combine in float64), {el:.1f} s")


def oracle_pair_step(wl, inp, state, act=(1.0, 0.0, float("inf")), biases=(None, None), pre=None,
                     getters=None):
    """One bounded reference step: routing of one token and one of its expert FFNs (with
    pre, the token's pre-FFN norm first)."""
    import numpy as np

    from oracle import moe_oracle as O
    t = state["t"]
    xt = inp.values("hidden")[t:t + 1] if pre is None else \
        O.pre_ffn_norm(pre[0][t:t + 1], pre[1], NORM_EPS, wl.dtype)
    L = O.router_logits(xt, inp.values("router_w"), inp["router_bias"])
    idx = O.select_topk(L, wl.k)
    w = O.routing_weights(L, idx, wl.normalize)
    j = state["j"]
    e = int(idx[0, j])
    b1, b2 = biases
    g1, g2 = getters if getters is not None else (lambda i: inp.expert_values("fc1", i),
                                                   lambda i: inp.expert_values("fc2", i))
    y = O.expert_ffn(xt, g1(e), g2(e), wl.fc1_layout, act,
                     None if b1 is None else b1[e], None if b2 is None else b2[e])
    assert np.isfinite(w[0, j] * y).all()
    state["j"] += 1
    if state["j"] == wl.k:
        state["j"] = 0
        state["t"] = (t + 1) % wl.T


def run_reference(args):
    from synth import WORKLOADS, bf16_bits_to_f32, make_inputs
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    wl = WORKLOADS[args.workload]
    steps = args.steps if args.steps is not None else DEFAULT_STEPS.get(wl.name, 100)
    from threadpoolctl import threadpool_info
    cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    inp = make_inputs(wl, weights=not args.q8)
    act = SWIGLU_PRESETS[args.swiglu]
    biases = (None, None)
    pre = None
    getters = None
    if args.q8:
        from synth import make_q8_experts
        getters = q8_getters(make_q8_experts(wl))
    if args.pre_norm:
        from synth import make_pre_norm_inputs
        px, pw = make_pre_norm_inputs(wl)
        wide = lambda a: bf16_bits_to_f32(a) if a.dtype.name == "uint16" else a
        pre = (wide(px), wide(pw))
    if args.expert_bias:
        from synth import make_expert_biases
        nb1, nb2 = make_expert_biases(wl)
        wide = lambda a: bf16_bits_to_f32(a) if a.dtype.name == "uint16" else a
        biases = (wide(nb1), wide(nb2))
    state = {"t": 0, "j": 0}
    for _ in range(args.warmup):
        oracle_pair_step(wl, inp, state, act, biases, pre, getters)
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle_pair_step(wl, inp, state, act, biases, pre, getters)
    el = time.perf_counter() - t0
    value = (steps / wl.k) / el
    sample = (f"each step: router logits + top-k of one token and one of its {wl.k} expert "
              f"FFNs (1/{wl.k} token); {steps} steps in {el:.1f} s")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(wl, sets=4 if wl.name in HBM_BOUND else 1),
                       parallelism=f"replicas x{args.gpus}",
                       graph_steps=GRAPH_STEPS.get(wl.name, 4), swiglu=list(act),
                       expert_bias=bool(args.expert_bias), pre_norm=bool(args.pre_norm),
                       q8=bool(args.q8),
                       fc1_layout_read="interleaved" if args.fc1_convert else wl.fc1_layout),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl, sets):
    cfg = {"workload": wl.name, "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k, "I": wl.I,
           "normalize": wl.normalize, "seed": wl.seed, "fc1_layout_given": wl.fc1_layout}
    if wl.router_bias_std is not None:
        cfg["router_bias_std"] = wl.router_bias_std
    if wl.outlier_frac:
        cfg["outliers"] = f"{wl.outlier_frac:g} of rows x{wl.outlier_scale:g}"
    cfg["l2"] = (f"{sets} rotating weight copies: {sets - 1} other copies stream between "
                 "reuses of one (inputs larger than L2)" if sets > 1 else
                 "per-step traffic larger than L2")
    return cfg


# --------------------------------------------------------------------------- our arm

def run_ours(args):
    import numpy as np
    import torch

    import mixture_experts_ffn_15_b200 as moe
    from synth import WORKLOADS, make_inputs

    rank, world, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=dev)
    wl = WORKLOADS[args.workload]
    S = GRAPH_STEPS.get(wl.name, 4)
    steps = args.steps if args.steps is not None else DEFAULT_STEPS.get(wl.name, 100)
    reps = max(1, math.ceil(steps / S))
    steps = reps * S
    warm_reps = max(1, math.ceil(args.warmup / S))
    sets = args.sets if args.sets is not None else (4 if wl.name in HBM_BOUND else 1)

    if args.q8 and wl.name not in HBM_BOUND:
        raise SystemExit("--q8: the int8 experts run in the decode FFN only (decode workloads)")
    inp = make_inputs(wl, weights=not args.q8)
    hidden = device_tensor(inp["hidden"], dev)
    norm_kw, pre = {}, None
    if args.pre_norm:
        # the input is a residual activation; the layer normalises it itself
        from synth import bf16_bits_to_f32, make_pre_norm_inputs
        px, pw = make_pre_norm_inputs(wl)
        hidden = device_tensor(px, dev)
        norm_kw = dict(norm_weight=device_tensor(pw, dev), norm_eps=NORM_EPS)
        wide = lambda a: bf16_bits_to_f32(a) if a.dtype.name == "uint16" else a
        pre = (wide(px), wide(pw))
    router_w = device_tensor(inp["router_w"], dev)
    bias = None if inp["router_bias"] is None else torch.from_numpy(inp["router_bias"]).to(dev)
    layout = wl.fc1_layout
    q8_host = None
    if args.q8:
        from synth import make_q8_experts
        q8_host = make_q8_experts(wl)
        q8 = [torch.from_numpy(a).to(dev) for a in q8_host]
        weight_sets = [q8] + [[t.clone() for t in q8] for _ in range(sets - 1)]
    else:
        fc1 = device_tensor(inp["fc1"], dev)
        if layout == "chunked" and args.fc1_convert:
            fc1 = moe.convert_chunked_to_interleaved(fc1)      # set-up, as at session load
            layout = "interleaved"
        fc2 = device_tensor(inp["fc2"], dev)
        weight_sets = [[fc1, fc2]] + [[fc1.clone(), fc2.clone()] for _ in range(sets - 1)]

    def run_layer(x, i, **kw):
        """One call of the layer on input x with the i-th rotating copy of the weights."""
        w = weight_sets[i % sets]
        if args.q8:
            return moe.forward_q8(x, router_w, w[0], w[1], w[2], w[3], wl.k, **kw)
        return moe.forward(x, router_w, w[0], w[1], wl.k, **kw)
    act = SWIGLU_PRESETS[args.swiglu]
    b1 = b2 = None
    if args.expert_bias:
        from synth import make_expert_biases
        nb1, nb2 = make_expert_biases(wl)
        b1, b2 = device_tensor(nb1, dev), device_tensor(nb2, dev)
    ffn_kw = dict(swiglu=act, fc1_bias=b1, fc2_bias=b2, fc1_layout=layout, **norm_kw)
    out = torch.empty_like(hidden)
    ws = moe.alloc_workspace(moe.workspace_size(wl.T, wl.H, wl.E, wl.k, wl.I, hidden.dtype), dev)

    # routing outside the timed region, for the byte accounting only
    x_in = moe.rmsnorm(hidden, norm_kw["norm_weight"], NORM_EPS) if args.pre_norm else hidden
    r = moe.route(x_in, router_w, wl.k, normalize=bool(wl.normalize), router_bias=bias)
    p = moe.permute(r["idx"], wl.E)
    counts = p["counts"].cpu().numpy()
    used, fc1_work, fc2_work, layer_work = algorithmic(wl, counts, args.pre_norm, args.q8)

    stream = torch.cuda.Stream(device=dev)
    call = lambda i: run_layer(hidden, i,
                                 normalize=bool(wl.normalize), router_bias=bias, out=out,
                                 workspace=ws, **ffn_kw)
    with torch.cuda.stream(stream):
        for i in range(sets):
            call(i)
    torch.cuda.synchronize(dev)

    # Two graphs of S steps each.  The timed region for `value` replays the plain
    # graph: consecutive kernels overlap their launch through programmatic
    # dependencies, which an event node between them would cut.  The stage times
    # (and the dominant kernel's duration for the roofline) come from a second timed
    # region that replays the same steps with the 6 stage events of every step.
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(S)]
    for row in events:
        for ev in row:
            ev.record(stream)
    torch.cuda.synchronize(dev)
    lib = moe.load_library()
    n0 = lib.moe_kernel_launches()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(S):
            call(i)
    launches_per_step = (lib.moe_kernel_launches() - n0) / S
    graph_ev = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_ev, stream=stream):
        for i in range(S):
            moe.set_stage_events([ev.cuda_event for ev in events[i]])
            call(i)
        moe.set_stage_events(None)

    with torch.cuda.stream(stream):
        for _ in range(warm_reps):
            graph.replay()
            graph_ev.replay()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    clocks.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks.mark(True)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for _ in range(reps):
            graph.replay()
        t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark(False)
    if world > 1:
        torch.distributed.barrier()
    # second timed region: the same steps with stage events
    with torch.cuda.stream(stream):
        for _ in range(max(1, reps // 4)):
            graph_ev.replay()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    ms_total = t_start.elapsed_time(t_end)
    ms_total = max_over_ranks(ms_total, world, dev)
    ms_step = ms_total / steps

    # stage durations of the last replay (inside the timed region)
    stage_names = ["route", "permute", "ffn1", "ffn2", "combine"]
    st = {n: 0.0 for n in stage_names}
    for i in range(S):
        for a, n in enumerate(stage_names):
            st[n] += events[i][a].elapsed_time(events[i][a + 1]) / S
    path = lib.moe_forward_path(wl.T, wl.H, wl.E, wl.k, wl.I, 1 if wl.dtype == "bf16" else 0)
    if args.q8:
        path &= ~32   # int8 experts: the decode FFN after the staged routing kernels
    fused = bool(path & 2)
    # the dominant kernel: the fused decode FFN (fc1 + SwiGLU and fc2 in one launch),
    # else the fc1 + SwiGLU grouped GEMM
    dom_ms = max_over_ranks(st["ffn1"], world, dev)
    # the fused decode kernel also does the combine: reads y_perm, writes out
    es = 2 if wl.dtype == "bf16" else 4
    comb_bytes = wl.T * wl.k * wl.H * es + wl.T * wl.H * es
    dom = {"bytes": fc1_work["bytes"] + fc2_work["bytes"] + comb_bytes,
           "flops": fc1_work["flops"] + fc2_work["flops"]} if fused else fc1_work
    one_launch = bool(path & 32)
    if one_launch:
        # ... and the routing: router weights and the token rows, the logits
        dom = {"bytes": dom["bytes"] + wl.E * wl.H * es + wl.T * wl.H * es + wl.T * wl.E * 4,
               "flops": dom["flops"] + 2.0 * wl.T * wl.H * wl.E}

    peaks, peak_kind = load_peaks()
    hbm = wl.name in HBM_BOUND
    if hbm:
        achieved = dom["bytes"] / (dom_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        achieved = dom["flops"] / (dom_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = ("tc_ffn_decode_kernel<ROUTE> (routing, fc1 + SwiGLU, fc2 and combine, weight rows on M)"
                      if one_launch else
                      "tc_ffn_decode_kernel (fc1 + SwiGLU, fc2 and combine, weight rows on M)" if fused else
                      "tc_pair_kernel<SWIGLU> (fc1 + SwiGLU on CTA pairs, weight rows on M)")
    roof["peak_source"] = f"{peak_kind} ({'hbm_gbs' if hbm else 'bf16_tflops, burst'})"
    roof["algorithmic_per_launch"] = dom["bytes"] if hbm else dom["flops"]
    roof["kernel_us"] = round(dom_ms * 1e3, 2)
    roof["traffic"] = kernel_traffic(wl.name, kernel_source(fused))
    if args.q8:
        roof["kernel"] = ("tc_ffn_decode_kernel<Q8> (int8 weights converted to bf16 in shared "
                          "memory, fc1 + SwiGLU, fc2 and combine, weight rows on M)")
        roof["traffic"] = None   # the committed counters are the bf16 kernel's

    layer_s = ms_step * 1e-3
    layer = {"GB/s": layer_work["bytes"] / layer_s / 1e9, "TFLOP/s": layer_work["flops"] / layer_s / 1e12,
             "hbm_frac": layer_work["bytes"] / layer_s / 1e9 / peaks["hbm_gbs"],
             "tensor_frac": layer_work["flops"] / layer_s / 1e12 / peaks["bf16_tflops"],
             "experts_used": used, "algorithmic_bytes": layer_work["bytes"],
             "algorithmic_flops": layer_work["flops"]}

    # end to end through the public API: pinned host input -> device -> layer -> host
    h_host = torch.empty(hidden.shape, dtype=hidden.dtype, pin_memory=True)
    h_host.copy_(hidden)
    o_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    d_in = torch.empty_like(hidden)
    n_e2e = args.e2e_steps
    with torch.cuda.stream(stream):
        for i in range(3):
            d_in.copy_(h_host, non_blocking=True)
            run_layer(d_in, i,
                        normalize=bool(wl.normalize), router_bias=bias, out=out, workspace=ws,
                        **ffn_kw)
            o_host.copy_(out, non_blocking=True)
            stream.synchronize()
        if world > 1:
            torch.distributed.barrier()
        t0 = time.perf_counter()
        for i in range(n_e2e):
            d_in.copy_(h_host, non_blocking=True)
            run_layer(d_in, i,
                        normalize=bool(wl.normalize), router_bias=bias, out=out, workspace=ws,
                        **ffn_kw)
            o_host.copy_(out, non_blocking=True)
            stream.synchronize()
        e2e_s = max_over_ranks(time.perf_counter() - t0, world, dev)
    e2e = {"value": wl.T * world * n_e2e / e2e_s, "unit": "tokens/s",
           "h2d_bytes_per_step": h_host.numel() * h_host.element_size(),
           "d2h_bytes_per_step": o_host.numel() * o_host.element_size(), "steps": n_e2e}

    st_err, bits = moe.get_error(moe.workspace_error_word(ws), stream)
    if st_err != 0:
        raise SystemExit(f"device error word {bits} after the bench")

    line = {
        "metric": METRIC, "value": job_throughput(wl.T, world, ms_step), "unit": "tokens/s",
        "n_gpus": world, "steps": steps, "warmup": warm_reps * S, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic",
        "config": dict(workload_config(wl, sets), parallelism=f"replicas x{world}",
                       graph_steps=S, swiglu=list(act), expert_bias=bool(args.expert_bias),
                       pre_norm=bool(args.pre_norm), q8=bool(args.q8), fc1_layout_read=layout),
        "roofline": roof, "layer": layer,
        "stages_us": {n: round(v * 1e3, 2) for n, v in st.items()},
        "stages_note": "second timed region, same steps with stage events between kernels",
        "e2e": e2e, "clocks": clk,
        "gpu_launches": int(round(launches_per_step * steps)),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample = oracle_cost(wl, inp, args.cpu_seconds, pre, q8_host)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph, graph_ev
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
