"""Expert parallelism on a GPU: ep_forward with the library's kernels under NCCL.

One rank on cuda:0 (a process group of world size 1, backend nccl), in a spawned
child process so that the process group lives and dies with it.  The all-to-all
exchanges are then self-exchanges through NCCL, but every computing step runs on the
device through KernelOps: the routing, the permutation, the k = 1 regrouping of the
received rows by local expert, the expert FFN, the k = 1 copy back to arrival order
and the weighted combine.  The output is compared with the oracle's layer on the
routing the GPU chose, within the stated bf16 tolerance.
"""
import datetime
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = [
    dict(name="spread", T=64, H=256, E=16, k=4, I=128, bias=None),
    # a skewed router: most rows go to a few experts, some experts get none
    dict(name="skewed", T=200, H=256, E=64, k=4, I=128, bias=1.0),
]


def _child(rank, port, out_dir, case):
    import sys

    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import mixture_experts_ffn_15_b200 as moe
    from mixture_experts_ffn_15_b200.expert_parallel import ep_forward
    from oracle import moe_oracle as O
    from parity_util import assert_close, device_inputs, from_dev, match_routing, tol
    from synth import Workload, make_inputs

    torch.cuda.set_device(0)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), NCCL_NVLS_ENABLE="0")
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0),
                            timeout=datetime.timedelta(seconds=60))
    res = {"ok": False}
    try:
        wl = Workload("ep_" + case["name"], T=case["T"], H=case["H"], E=case["E"], k=case["k"],
                      I=case["I"], dtype="bf16", seed=21, router_bias_std=case["bias"])
        inp = make_inputs(wl)
        dev = device_inputs(inp)
        out = ep_forward(dev["hidden"], dev["router_w"], dev["fc1"], dev["fc2"], wl.k,
                         router_bias=dev["router_bias"])
        r = moe.route(dev["hidden"], dev["router_w"], wl.k, router_bias=dev["router_bias"])
        torch.cuda.synchronize()
        L = O.router_logits(inp.values("hidden"), inp.values("router_w"), inp["router_bias"])
        idx, _ = match_routing(L, from_dev(r["idx"]).astype(np.int64), wl.k)
        ref = O.moe_forward(inp.values("hidden"), inp.values("router_w"), inp["router_bias"],
                            lambda e: inp.expert_values("fc1", e),
                            lambda e: inp.expert_values("fc2", e), wl.k, 1, idx=idx)["out"]
        atol, rtol = tol("bf16", ref)
        assert_close(from_dev(out), ref, atol, rtol, f"{wl.name} expert-parallel output")
        counts = np.bincount(idx.ravel(), minlength=wl.E)
        res = {"ok": True, "idle_experts": int(np.sum(counts == 0)),
               "max_rows": int(counts.max())}
    except AssertionError as ex:
        res = {"ok": False, "error": str(ex)}
    finally:
        dist.destroy_process_group()
        with open(os.path.join(out_dir, "result.json"), "w") as f:
            json.dump(res, f)


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_one_rank_nccl_expert_parallel_on_the_gpu(tmp_path, case):
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    mp.start_processes(_child, args=(port, str(tmp_path), case), nprocs=1, join=True,
                       start_method="spawn")
    r = json.load(open(tmp_path / "result.json"))
    assert r["ok"], r.get("error")
    if case["bias"] is not None:
        assert r["idle_experts"] > 0, "the skewed case should leave some experts without rows"
