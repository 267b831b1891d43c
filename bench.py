#!/usr/bin/env python
"""Benchmark of the fused MoE FFN layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one call of the whole layer (route -> permute -> fc1 + SwiGLU -> fc2 ->
combine) on one batch of synthetic tokens with the inputs resident in HBM.  The
line's workload is long_prefill_bf16 (T=32768, H=4096, E=64, k=4, I=1536, 1% of the
rows x8), the largest of the five single-GPU workloads of synth.WORKLOADS;
--workload picks another.  It runs W warm-up steps (eager calls through the public
API) and then times exactly K steps, replayed from a CUDA graph of S steps (S
divides K), between two CUDA events on the launching stream.  Each of the other
four workloads is then measured the same way with its own step counts and reported
under `per_config` (value, roofline of its dominant kernel, e2e, CPU baseline,
clocks).  For the weight-streaming workloads `--sets` copies of the weights rotate,
so that the weights of a step never sit in L2 when it starts; the prefill workloads
move more than L2 per step.

Prints ONE JSON line (rank 0).  Multi-GPU (torchrun, one rank per GPU) runs
independent replicas: the layer has no exchange step on one GPU's batch, so there
is no data-path collective; the barrier and the max-over-ranks timing are the only
communication.  `--impl reference` times the CPU oracle (the reference arm) on the
host instead.
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
ORDER = ["tiny_fp32", "decode_bf16", "batched_decode_bf16", "prefill_bf16", "long_prefill_bf16"]
DEFAULT_WORKLOAD = "long_prefill_bf16"
# steps and warm-up steps of a workload when the command line does not set them
DEFAULT_STEPS = {"tiny_fp32": 10000, "decode_bf16": 4000, "batched_decode_bf16": 1000,
                 "prefill_bf16": 300, "long_prefill_bf16": 100}
DEFAULT_WARMUP = {"tiny_fp32": 40, "decode_bf16": 40, "batched_decode_bf16": 20,
                  "prefill_bf16": 5, "long_prefill_bf16": 3}
# steps per CUDA graph (at most; the graph size divides the step count)
GRAPH_STEPS = {"tiny_fp32": 20, "decode_bf16": 20, "batched_decode_bf16": 20,
               "prefill_bf16": 1, "long_prefill_bf16": 1}
HBM_BOUND = {"decode_bf16", "batched_decode_bf16", "tiny_fp32"}
SWIGLU_PRESETS = {"standard": (1.0, 0.0, float("inf")), "gpt_oss": (1.702, 1.0, 7.0)}
NORM_EPS = 1e-6
CPU_WORKERS_MAX = 32


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--sets", type=int, default=None, help="rotating weight copies (L2)")
    ap.add_argument("--e2e-seconds", type=float, default=1.0,
                    help="about how long the end-to-end measurement of a workload runs")
    ap.add_argument("--cpu-seconds", type=float, default=6.0,
                    help="CPU baseline of the line's workload: seconds per timing")
    ap.add_argument("--per-config-cpu-seconds", type=float, default=2.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="measure the line's workload only")
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


def variant_flags(args):
    """True when a flag changes the layer (then only the line's workload is measured)."""
    return bool(args.q8 or args.pre_norm or args.expert_bias or args.swiglu != "standard"
                or args.fc1_convert)


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


def graph_steps(limit, steps):
    """Steps per CUDA graph: the largest divisor of `steps` not above `limit`."""
    for s in range(max(1, min(limit, steps)), 0, -1):
        if steps % s == 0:
            return s
    return 1


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 50 ms in the background
    with their timestamps, so that each timed region takes the samples inside it."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.file = None
        self.rows = []

    def start(self):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "50"], stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.5)

    def stop(self):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.file.flush()
        with open(self.file.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except ValueError:
                    ts = None
                self.rows.append((ts, parts[1:]))
        os.unlink(self.file.name)

    @staticmethod
    def _num(s):
        try:
            return float(s)
        except ValueError:
            return float("nan")

    def summary(self, t0, t1):
        """Median SM clock and the throttle reasons seen during [t0, t1] (host times)."""
        inside = [r for ts, r in self.rows if ts is not None and t0 - 0.06 <= ts <= t1 + 0.06]
        note = "samples inside the timed region"
        if not inside:
            after = [(ts, r) for ts, r in self.rows if ts is not None and ts >= t0]
            inside = [after[0][1]] if after else [r for _, r in self.rows[-1:]]
            note = "timed region shorter than the sampling period: the next sample"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = sorted(self._num(r[0]) for r in inside)
        reasons = sorted({self.NAMES[i] for r in inside for i in range(4)
                          if r[4 + i].lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": self._num(inside[0][1]),
                "reasons": reasons, "samples": len(inside), "note": note,
                "power_w_max": max(self._num(r[2]) for r in inside)}


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


def kernel_source(decode_kernel):
    """Source file of the dominant kernel: the decode FFN (gemm_tc.cu) or the CTA-pair
    grouped GEMM (gemm_pair.cu)."""
    name = "gemm_tc.cu" if decode_kernel else "gemm_pair.cu"
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


def wide(a):
    from synth import bf16_bits_to_f32
    return None if a is None else (bf16_bits_to_f32(a) if a.dtype.name == "uint16" else a)


# --------------------------------------------------------------------------- host inputs

def host_inputs(names, q8=False):
    """The synthetic inputs of each workload (CPU arrays).  Expert weights depend only
    on (seed, E, H, I, dtype), so workloads that share those share one draw."""
    from synth import WORKLOADS, make_inputs
    drawn = {}
    out = {}
    for n in names:
        wl = WORKLOADS[n]
        inp = make_inputs(wl, weights=False)
        if not q8:
            key = (wl.seed, wl.E, wl.H, wl.I, wl.dtype)
            if key not in drawn:
                full = make_inputs(wl)
                drawn[key] = (full["fc1"], full["fc2"])
            inp.arrays["fc1"], inp.arrays["fc2"] = drawn[key]
        out[n] = inp
    return out


class LayerOptions:
    """The layer's optional inputs, as host arrays, for the oracle and the device."""

    def __init__(self, args, wl):
        from synth import make_expert_biases, make_pre_norm_inputs, make_q8_experts
        self.act = SWIGLU_PRESETS[args.swiglu]
        self.biases = make_expert_biases(wl) if args.expert_bias else (None, None)
        self.pre = make_pre_norm_inputs(wl) if args.pre_norm else None
        self.q8 = make_q8_experts(wl) if args.q8 else None

    def oracle_getters(self, inp):
        from oracle import moe_oracle as O
        if self.q8 is not None:
            q1, s1, q2, s2 = self.q8
            return (lambda e: O.dequantize_rows(q1[e], s1[e]),
                    lambda e: O.dequantize_rows(q2[e], s2[e]))
        return (lambda e: inp.expert_values("fc1", e), lambda e: inp.expert_values("fc2", e))


# --------------------------------------------------------------------------- CPU oracle

def oracle_tokens(wl, inp, opts, seconds, start=0, stride=1):
    """The CPU oracle, as it stands, on whole tokens start, start + stride, ... of `wl`
    for about `seconds` (each token routed over all E experts and run through its k
    experts in float64; with the pre-FFN norm, normalised first).  Returns (tokens, s)."""
    import numpy as np

    from oracle import moe_oracle as O
    x = inp.values("hidden")
    rw = inp.values("router_w")
    fc1, fc2 = opts.oracle_getters(inp)
    b1, b2 = (wide(b) for b in opts.biases)
    t0 = time.perf_counter()
    n = 0
    t = start % wl.T
    while True:
        xt = x[t:t + 1] if opts.pre is None else O.pre_ffn_norm(
            wide(opts.pre[0])[t:t + 1], wide(opts.pre[1]), NORM_EPS, wl.dtype)
        r = O.moe_forward(xt, rw, inp["router_bias"], fc1, fc2, wl.k, wl.normalize,
                          wl.fc1_layout, act=opts.act, fc1_bias=b1, fc2_bias=b2)
        assert np.isfinite(r["out"]).all()
        n += 1
        t = (t + stride) % wl.T
        if time.perf_counter() - t0 >= seconds:
            break
    return n, time.perf_counter() - t0


_POOL_STATE = {}


def _pool_job(job):
    """One worker of the all-core CPU baseline: its own token stride, one BLAS thread."""
    from threadpoolctl import threadpool_limits
    name, start, stride, seconds = job
    wl, inp, opts = _POOL_STATE[name]
    with threadpool_limits(1):
        return oracle_tokens(wl, inp, opts, seconds, start, stride)


class CpuBaseline:
    """The oracle timed on the host: one thread, and one process per core (up to
    CPU_WORKERS_MAX) on interleaved tokens.  The worker processes are forked before
    the first CUDA call, so that they hold the inputs already drawn."""

    def __init__(self, workloads):
        import multiprocessing as mp
        _POOL_STATE.update(workloads)
        self.workers = max(1, min(os.cpu_count() or 1, CPU_WORKERS_MAX))
        self.pool = mp.get_context("fork").Pool(self.workers) if self.workers > 1 else None

    def measure(self, name, seconds):
        from threadpoolctl import threadpool_limits
        wl, inp, opts = _POOL_STATE[name]
        with threadpool_limits(1):
            n1, s1 = oracle_tokens(wl, inp, opts, seconds)
        single = n1 / s1
        res = {"value": single, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": (f"{n1} whole tokens of the workload, one thread (router logits over "
                          f"all {wl.E} experts, top-k, {wl.k} expert FFNs, combine in float64), "
                          f"{s1:.1f} s")}
        if self.pool is not None:
            jobs = [(name, i, self.workers, seconds) for i in range(self.workers)]
            try:
                got = self.pool.map_async(_pool_job, jobs).get(timeout=seconds * 4 + 60)
                n = sum(g[0] for g in got)
                el = max(g[1] for g in got)
                res = {"value": n / el, "unit": "tokens/s", "cores": self.workers,
                       "kind": "oracle",
                       "sample": (f"{n} whole tokens in {el:.1f} s on {self.workers} processes "
                                  f"(one BLAS thread each, interleaved tokens)"),
                       "single_thread": res}
            except Exception as ex:   # a stuck worker: keep the one-thread figure
                res["all_cores"] = f"unavailable: {type(ex).__name__}"
        return res

    def close(self):
        if self.pool is not None:
            self.pool.terminate()
            self.pool.join()


def oracle_pair_step(wl, inp, opts, state):
    """One bounded reference step: routing of one token and one of its expert FFNs (with
    the pre-FFN norm, the token's norm first)."""
    import numpy as np

    from oracle import moe_oracle as O
    t = state["t"]
    xt = inp.values("hidden")[t:t + 1] if opts.pre is None else \
        O.pre_ffn_norm(wide(opts.pre[0])[t:t + 1], wide(opts.pre[1]), NORM_EPS, wl.dtype)
    L = O.router_logits(xt, inp.values("router_w"), inp["router_bias"])
    idx = O.select_topk(L, wl.k)
    w = O.routing_weights(L, idx, wl.normalize)
    j = state["j"]
    e = int(idx[0, j])
    b1, b2 = (wide(b) for b in opts.biases)
    g1, g2 = opts.oracle_getters(inp)
    y = O.expert_ffn(xt, g1(e), g2(e), wl.fc1_layout, opts.act,
                     None if b1 is None else b1[e], None if b2 is None else b2[e])
    assert np.isfinite(w[0, j] * y).all()
    state["j"] += 1
    if state["j"] == wl.k:
        state["j"] = 0
        state["t"] = (t + 1) % wl.T


def run_reference(args):
    from threadpoolctl import threadpool_limits

    from synth import WORKLOADS, make_inputs
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    wl = WORKLOADS[args.workload]
    steps = args.steps if args.steps is not None else DEFAULT_STEPS.get(wl.name, 100)
    warmup = args.warmup if args.warmup is not None else DEFAULT_WARMUP.get(wl.name, 3)
    inp = make_inputs(wl, weights=not args.q8)
    opts = LayerOptions(args, wl)
    state = {"t": 0, "j": 0}
    with threadpool_limits(1):
        for _ in range(warmup):
            oracle_pair_step(wl, inp, opts, state)
        t0 = time.perf_counter()
        for _ in range(steps):
            oracle_pair_step(wl, inp, opts, state)
        el = time.perf_counter() - t0
    value = (steps / wl.k) / el
    sample = (f"each step: router logits + top-k of one token and one of its {wl.k} expert "
              f"FFNs (1/{wl.k} token), one thread; {steps} steps in {el:.1f} s")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": warmup,
        "ms_per_step": 1e3 * el / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(wl, sets=default_sets(wl, args)),
                       parallelism=f"replicas x{args.gpus}", swiglu=list(opts.act),
                       expert_bias=bool(args.expert_bias), pre_norm=bool(args.pre_norm),
                       q8=bool(args.q8),
                       fc1_layout_read="interleaved" if args.fc1_convert else wl.fc1_layout),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def default_sets(wl, args):
    if args.sets is not None:
        return args.sets
    return 4 if wl.name in HBM_BOUND else 1


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

def measure(wl, inp, opts, args, steps, warmup, world, dev, clocks):
    """The layer on workload `wl`: W eager warm-up calls, then K steps replayed from a
    CUDA graph between two events, a second region with stage events, and the end-to-end
    figure through the public API.  Returns the workload's result row."""
    import numpy as np
    import torch

    import mixture_experts_ffn_15_b200 as moe

    sets = default_sets(wl, args)
    S = graph_steps(GRAPH_STEPS.get(wl.name, 1), steps)
    reps = steps // S
    hidden = device_tensor(inp["hidden"], dev)
    norm_kw = {}
    if opts.pre is not None:
        # the input is a residual activation; the layer normalises it itself
        hidden = device_tensor(opts.pre[0], dev)
        norm_kw = dict(norm_weight=device_tensor(opts.pre[1], dev), norm_eps=NORM_EPS)
    router_w = device_tensor(inp["router_w"], dev)
    bias = None if inp["router_bias"] is None else torch.from_numpy(inp["router_bias"]).to(dev)
    layout = wl.fc1_layout
    if opts.q8 is not None:
        q8 = [torch.from_numpy(a).to(dev) for a in opts.q8]
        weight_sets = [q8] + [[t.clone() for t in q8] for _ in range(sets - 1)]
    else:
        fc1 = device_tensor(inp["fc1"], dev)
        if layout == "chunked" and args.fc1_convert:
            fc1 = moe.convert_chunked_to_interleaved(fc1)      # set-up, as at session load
            layout = "interleaved"
        fc2 = device_tensor(inp["fc2"], dev)
        weight_sets = [[fc1, fc2]] + [[fc1.clone(), fc2.clone()] for _ in range(sets - 1)]
    b1 = b2 = None
    if opts.biases[0] is not None:
        b1, b2 = (device_tensor(b, dev) for b in opts.biases)
    ffn_kw = dict(swiglu=opts.act, fc1_bias=b1, fc2_bias=b2, fc1_layout=layout, **norm_kw)
    out = torch.empty_like(hidden)
    ws = moe.alloc_workspace(moe.workspace_size(wl.T, wl.H, wl.E, wl.k, wl.I, hidden.dtype), dev)

    def run_layer(x, i, **kw):
        """One call of the layer on input x with the i-th rotating copy of the weights."""
        w = weight_sets[i % sets]
        if opts.q8 is not None:
            return moe.forward_q8(x, router_w, w[0], w[1], w[2], w[3], wl.k, **kw)
        return moe.forward(x, router_w, w[0], w[1], wl.k, **kw)

    # routing outside the timed region, for the byte accounting only
    x_in = moe.rmsnorm(hidden, norm_kw["norm_weight"], NORM_EPS) if norm_kw else hidden
    r = moe.route(x_in, router_w, wl.k, normalize=bool(wl.normalize), router_bias=bias)
    counts = moe.permute(r["idx"], wl.E)["counts"].cpu().numpy()
    del r, x_in
    used, fc1_work, fc2_work, layer_work = algorithmic(wl, counts, opts.pre is not None,
                                                       opts.q8 is not None)

    stream = torch.cuda.Stream(device=dev)
    call = lambda x, i: run_layer(x, i, normalize=bool(wl.normalize), router_bias=bias, out=out,
                                  workspace=ws, **ffn_kw)
    # warm-up: W eager steps through the public API (the first call of each weight set
    # also does the library's once-per-device set-up, which must precede a capture)
    with torch.cuda.stream(stream):
        for i in range(max(warmup, sets)):
            call(hidden, i)
    torch.cuda.synchronize(dev)

    # The timed graph (S steps): consecutive kernels overlap their launch through
    # programmatic dependencies, which an event between them would cut.  The stage
    # times (and the dominant kernel's duration) come from a second graph of the same
    # steps with the 6 stage events of every step, replayed after the timed region.
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
            call(hidden, i)
    launches_per_step = (lib.moe_kernel_launches() - n0) / S
    graph_ev = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_ev, stream=stream):
        for i in range(S):
            moe.set_stage_events([ev.cuda_event for ev in events[i]])
            call(hidden, i)
        moe.set_stage_events(None)

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    h0 = time.time()
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for _ in range(reps):
            graph.replay()
        t_end.record(stream)
    torch.cuda.synchronize(dev)
    h1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    ms_step = max_over_ranks(t_start.elapsed_time(t_end), world, dev) / steps

    # second region: the same steps with stage events (stage times of the last replay)
    with torch.cuda.stream(stream):
        for _ in range(max(1, min(reps // 4, 8))):
            graph_ev.replay()
    torch.cuda.synchronize(dev)
    stage_names = ["route", "permute", "ffn1", "ffn2", "combine"]
    st = {n: 0.0 for n in stage_names}
    for i in range(S):
        for a, n in enumerate(stage_names):
            st[n] += events[i][a].elapsed_time(events[i][a + 1]) / S
    path = lib.moe_forward_path(wl.T, wl.H, wl.E, wl.k, wl.I, 1 if wl.dtype == "bf16" else 0)
    fused = bool(path & 2)
    one_launch = bool(path & 32)
    es = 2 if wl.dtype == "bf16" else 4
    # the dominant kernel: the fused decode FFN (fc1 + SwiGLU, fc2 and the combine in one
    # launch; one-launch decode: also the routing), else fc1 + SwiGLU
    dom = fc1_work
    if fused:
        comb_bytes = wl.T * wl.k * wl.H * es + wl.T * wl.H * es
        dom = {"bytes": fc1_work["bytes"] + fc2_work["bytes"] + comb_bytes,
               "flops": fc1_work["flops"] + fc2_work["flops"]}
    if one_launch:
        dom = {"bytes": dom["bytes"] + wl.E * wl.H * es + wl.T * wl.H * es + wl.T * wl.E * 4,
               "flops": dom["flops"] + 2.0 * wl.T * wl.H * wl.E}
    dom_ms_events = max_over_ranks(st["ffn1"], world, dev)
    # an event on each side cuts the launch overlap with the neighbouring kernels, so the
    # bracketed time can exceed the step's share; the kernel never takes longer than the
    # step it is part of
    dom_ms = min(dom_ms_events, ms_step)

    peaks, peak_kind = load_peaks()
    hbm = wl.name in HBM_BOUND
    if hbm:
        achieved = dom["bytes"] / (dom_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        achieved = dom["flops"] / (dom_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    if not hbm:
        roof["peak_sustained"] = peaks["bf16_tflops_sustained"]
        roof["frac_sustained"] = roof["achieved"] / peaks["bf16_tflops_sustained"]
    if wl.dtype != "bf16":
        roof["note"] = ("float32 on the FMA pipes, launch-latency bound at this size: neither "
                        "roofline is reachable; HBM fraction reported for reference")
    roof["kernel"] = ("tc_ffn_decode_kernel<ROUTE> (routing, fc1 + SwiGLU, fc2 and combine, weight rows on M)"
                      if one_launch else
                      "tc_ffn_decode_kernel (fc1 + SwiGLU, fc2 and combine, weight rows on M)" if fused else
                      "tc_pair_kernel<SWIGLU> (fc1 + SwiGLU on CTA pairs, weight rows on M)"
                      if wl.dtype == "bf16" else "ffn_simt fc1 + SwiGLU (float32 FMA)")
    if opts.q8 is not None:
        roof["kernel"] = ("tc_ffn_decode_kernel<Q8> (" + ("routing, " if one_launch else "") +
                          "int8 weights converted to bf16 in tensor memory, fc1 + SwiGLU, fc2 "
                          "and combine, weight rows on M)")
    roof["peak_source"] = f"{peak_kind} ({'hbm_gbs' if hbm else 'bf16_tflops, burst'})"
    roof["algorithmic_per_launch"] = dom["bytes"] if hbm else dom["flops"]
    roof["kernel_us"] = round(dom_ms * 1e3, 2)
    roof["kernel_us_events"] = round(dom_ms_events * 1e3, 2)
    roof["traffic"] = None if opts.q8 is not None or wl.dtype != "bf16" else \
        kernel_traffic(wl.name, kernel_source(fused))
    if not fused and wl.dtype == "bf16":
        # the second grouped GEMM of the prefill path, for reference
        fc2_ms = max_over_ranks(st["ffn2"], world, dev)
        roof["fc2"] = {"kernel": "tc_pair_kernel<plain> (fc2 on CTA pairs)",
                       "achieved": fc2_work["flops"] / (fc2_ms * 1e-3) / 1e12,
                       "frac": fc2_work["flops"] / (fc2_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                       "kernel_us": round(fc2_ms * 1e3, 2)}

    layer_s = ms_step * 1e-3
    layer = {"GB/s": layer_work["bytes"] / layer_s / 1e9, "TFLOP/s": layer_work["flops"] / layer_s / 1e12,
             "hbm_frac": layer_work["bytes"] / layer_s / 1e9 / peaks["hbm_gbs"],
             "tensor_frac": layer_work["flops"] / layer_s / 1e12 / peaks["bf16_tflops"],
             "experts_used": used, "algorithmic_bytes": layer_work["bytes"],
             "algorithmic_flops": layer_work["flops"]}

    # end to end through the public API: pinned host input -> device -> layer -> host,
    # streamed as a serving loop would run it: the copy-in of step i+1 and the copy-out
    # of step i-1 run on streams of their own while the layer of step i runs (device
    # input and output double-buffered).  Every step still moves its whole input in and
    # its whole output out; the clock stops once the last output is in host memory.
    h_host = torch.empty(hidden.shape, dtype=hidden.dtype, pin_memory=True)
    h_host.copy_(hidden)
    o_host = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    d_in = [torch.empty_like(hidden) for _ in range(2)]
    d_out = [out, torch.empty_like(out)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    io_bytes = 2 * h_host.numel() * h_host.element_size()
    est_s = max(layer_s, io_bytes / 2 / 25e9)
    n_e2e = int(max(3, min(200, args.e2e_seconds / est_s)))

    def e2e_steps(n):
        in_done, done, out_done = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(done[b])          # step i-2's layer has read d_in[b]
                d_in[b].copy_(h_host, non_blocking=True)
                in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            if i >= 2:
                stream.wait_event(out_done[b])        # step i-2's output has left d_out[b]
            run_layer(d_in[b], i, normalize=bool(wl.normalize), router_bias=bias,
                      out=d_out[b], workspace=ws, stream=stream, **ffn_kw)
            done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[b])
                o_host[b].copy_(d_out[b], non_blocking=True)
                out_done[b].record(s_out)
        for st_ in (s_in, stream, s_out):
            st_.synchronize()

    e2e_steps(2)
    if world > 1:
        torch.distributed.barrier()
    t0 = time.perf_counter()
    e2e_steps(n_e2e)
    e2e_s = max_over_ranks(time.perf_counter() - t0, world, dev)
    # the streamed outputs are the layer's: the last one against a call on the device
    with torch.cuda.stream(stream):
        call(hidden, 0)
    stream.synchronize()
    if not torch.equal(o_host[(n_e2e - 1) % 2], out.cpu()):
        raise SystemExit(f"{wl.name}: streamed output differs from the device result")
    e2e = {"value": wl.T * world * n_e2e / e2e_s, "unit": "tokens/s",
           "h2d_bytes_per_step": h_host.numel() * h_host.element_size(),
           "d2h_bytes_per_step": o_host[0].numel() * o_host[0].element_size(), "steps": n_e2e,
           "pipeline": "copy-in of step i+1 and copy-out of step i-1 overlap the layer of "
                       "step i (three streams, double-buffered device input and output)"}

    st_err, bits = moe.get_error(moe.workspace_error_word(ws), stream)
    if st_err != 0:
        raise SystemExit(f"{wl.name}: device error word {bits} after the bench")

    row = {
        "value": job_throughput(wl.T, world, ms_step), "unit": "tokens/s",
        "steps": steps, "warmup": max(warmup, sets), "ms_per_step": ms_step,
        "config": dict(workload_config(wl, sets), parallelism=f"replicas x{world}",
                       graph_steps=S),
        "roofline": roof, "layer": layer,
        "stages_us": {n: round(v * 1e3, 2) for n, v in st.items()},
        "e2e": e2e,
        "gpu_launches": int(round(launches_per_step * steps)),
        "_timed_host": (h0, h1),
    }
    del graph, graph_ev, weight_sets, ws, out, hidden, d_in, h_host, o_host
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return row


def run_ours(args):
    from synth import WORKLOADS

    rank, world, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    head = WORKLOADS[args.workload]
    if args.q8 and head.name not in HBM_BOUND:
        raise SystemExit("--q8: the int8 experts run in the decode FFN only (decode workloads)")
    names = [head.name]
    if not args.no_per_config and not variant_flags(args):
        names += [n for n in ORDER if n != head.name]

    # host inputs and the CPU baseline's worker processes, before the first CUDA call
    inputs = host_inputs(names, q8=args.q8)
    opts = {n: LayerOptions(args, WORKLOADS[n]) for n in names}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = CpuBaseline({n: (WORKLOADS[n], inputs[n], opts[n]) for n in names})

    import torch
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=dev)
    clocks = ClockSampler(local)
    clocks.start()
    rows = {}
    try:
        for n in names:
            wl = WORKLOADS[n]
            is_head = n == head.name
            steps = DEFAULT_STEPS.get(n, 100)
            warmup = DEFAULT_WARMUP.get(n, 3)
            if is_head:
                steps = args.steps if args.steps is not None else steps
                warmup = args.warmup if args.warmup is not None else warmup
            rows[n] = measure(wl, inputs[n], opts[n], args, steps, warmup, world, dev, clocks)
    finally:
        clocks.stop()
    for n in names:
        rows[n]["clocks"] = clocks.summary(*rows[n].pop("_timed_host"))
    if cpu is not None:
        try:
            for n in names:
                secs = args.cpu_seconds if n == head.name else args.per_config_cpu_seconds
                rows[n]["cpu_baseline"] = cpu.measure(n, secs)
        finally:
            cpu.close()

    h = rows[head.name]
    line = {
        "metric": METRIC, "value": h["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": h["steps"], "warmup": h["warmup"], "ms_per_step": h["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if head.dtype == "bf16" else "f32", "data": "synthetic",
        "config": dict(h["config"], swiglu=list(opts[head.name].act),
                       expert_bias=bool(args.expert_bias), pre_norm=bool(args.pre_norm),
                       q8=bool(args.q8), fc1_layout_read=(
                           "interleaved" if args.fc1_convert else head.fc1_layout)),
        "roofline": h["roofline"], "layer": h["layer"], "stages_us": h["stages_us"],
        "stages_note": "second timed region, same steps with stage events between kernels",
        "e2e": h["e2e"], "clocks": h["clocks"], "gpu_launches": h["gpu_launches"],
    }
    if "cpu_baseline" in h:
        line["cpu_baseline"] = h["cpu_baseline"]
    if len(names) > 1:
        line["per_config"] = {
            n: {k: rows[n][k] for k in ("value", "unit", "ms_per_step", "steps", "warmup",
                                        "config", "roofline", "layer", "stages_us", "e2e",
                                        "clocks", "gpu_launches", "cpu_baseline") if k in rows[n]}
            for n in names[1:]}
    if rank == 0:
        print(json.dumps(line), flush=True)
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
