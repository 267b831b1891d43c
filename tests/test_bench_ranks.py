"""bench.py across ranks on the CPU (gloo, world size 2).

The layer has no exchange step on one GPU's batch, so N GPUs run N independent
replicas; the only communication is the barrier and the max over ranks of the
device time.  These tests run that plumbing with two gloo ranks on the host: the
max over ranks, the whole-job throughput from it, and the reference arm, which only
rank 0 runs and prints.
"""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import contextlib
    import io
    import sys
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # each rank's device time differs; every rank must see the slowest one
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        value = bench.job_throughput(tokens_per_rank=4, world=world, ms_per_step=ms)
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            rc = bench.main(["--impl", "reference", "--gpus", str(world), "--steps", "2",
                             "--warmup", "1", "--workload", "tiny_fp32"])
        dist.barrier()
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"ms": ms, "value": value, "rc": rc, "stdout": buf.getvalue()}, f)


def test_two_gloo_ranks_max_time_and_reference_arm(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(2)]
    assert r[0]["ms"] == r[1]["ms"] == 15.0                     # max over ranks
    assert r[0]["value"] == pytest.approx(2 * 4 / 15.0e-3)       # all ranks' tokens / slowest time
    assert r[0]["rc"] == 0 and r[1]["rc"] == 0
    assert r[1]["stdout"] == ""                                  # only rank 0 prints
    line = json.loads(r[0]["stdout"].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["unit"] == "tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
