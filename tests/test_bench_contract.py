"""bench.py on the CPU: the reference arm's JSON line and the byte accounting of the
layer variants (no GPU needed)."""
import contextlib
import io
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _reference_line(monkeypatch, *extra):
    import bench
    for v in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(v, raising=False)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--steps", "2", "--warmup", "1",
                         "--workload", "tiny_fp32", *extra])
    assert rc == 0
    return json.loads(buf.getvalue().strip().splitlines()[-1])


def test_reference_arm_line(monkeypatch):
    line = _reference_line(monkeypatch)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["config"]["workload"] == "tiny_fp32"


@pytest.mark.parametrize("flags", [["--swiglu", "gpt_oss", "--expert-bias"], ["--pre-norm"]])
def test_reference_arm_records_the_layer_options(monkeypatch, flags):
    line = _reference_line(monkeypatch, *flags)
    cfg = line["config"]
    if "--pre-norm" in flags:
        assert cfg["pre_norm"] is True
    else:
        assert cfg["swiglu"] == [1.702, 1.0, 7.0] and cfg["expert_bias"] is True


def test_algorithmic_bytes_of_the_variants():
    import bench
    from synth import WORKLOADS
    wl = WORKLOADS["decode_bf16"]
    counts = [1] * 28 + [0] * (wl.E - 28)
    T, H, E, k, I = wl.T, wl.H, wl.E, wl.k, wl.I
    used, fc1, fc2, layer = bench.algorithmic(wl, counts)
    assert used == 28
    assert fc1["bytes"] == 28 * 2 * I * H * 2 + T * k * H * 2 + T * k * I * 2
    assert fc2["bytes"] == 28 * H * I * 2 + T * k * I * 2 + T * k * H * 2
    _, _, _, normed = bench.algorithmic(wl, counts, pre_norm=True)
    assert normed["bytes"] - layer["bytes"] == 2 * T * H * 2 + H * 2
    _, q1, q2, q8 = bench.algorithmic(wl, counts, q8=True)
    # int8 weights: one byte each instead of two, plus a float32 scale per weight row
    assert fc1["bytes"] - q1["bytes"] == 28 * 2 * I * H - 28 * 2 * I * 4
    assert fc2["bytes"] - q2["bytes"] == 28 * H * I - 28 * H * 4
    assert layer["bytes"] - q8["bytes"] == 28 * 3 * H * I - 28 * (2 * I + H) * 4
    assert q8["flops"] == layer["flops"]


def test_graph_steps_divide_the_step_count():
    import bench
    for limit in (1, 2, 20):
        for steps in (1, 5, 20, 37, 100, 4000):
            s = bench.graph_steps(limit, steps)
            assert 1 <= s <= limit and steps % s == 0


def test_workloads_with_the_same_expert_shapes_share_one_weight_draw():
    import numpy as np

    import bench
    from synth import WORKLOADS, Workload, make_inputs
    a = Workload("wa", T=8, H=64, E=4, k=2, I=32, dtype="bf16")
    b = Workload("wb", T=16, H=64, E=4, k=2, I=32, dtype="bf16", fc1_layout="chunked")
    WORKLOADS.update(wa=a, wb=b)
    try:
        got = bench.host_inputs(["wa", "wb"])
    finally:
        del WORKLOADS["wa"], WORKLOADS["wb"]
    assert got["wa"]["fc1"] is got["wb"]["fc1"]
    np.testing.assert_array_equal(got["wb"]["fc1"], make_inputs(b)["fc1"])
    np.testing.assert_array_equal(got["wb"]["hidden"], make_inputs(b)["hidden"])


def test_cpu_baseline_one_thread_and_all_cores():
    import argparse

    import bench
    from synth import WORKLOADS
    wl = WORKLOADS["tiny_fp32"]
    args = bench.parse_args([])
    inputs = bench.host_inputs([wl.name])
    cpu = bench.CpuBaseline({wl.name: (wl, inputs[wl.name], bench.LayerOptions(args, wl))})
    try:
        r = cpu.measure(wl.name, 0.3)
    finally:
        cpu.close()
    assert r["kind"] == "oracle" and r["value"] > 0 and r["cores"] >= 1
    if r["cores"] > 1:
        assert r["single_thread"]["cores"] == 1 and r["single_thread"]["value"] > 0
    del argparse
