"""Expert parallelism across ranks on the CPU (gloo, world size 2).

Each rank routes its own tokens and owns half of the experts; the rows travel to the
owning rank and back with all-to-all exchanges.  Here the computing steps run on host
tensors through the oracle (the GPU runs the library's kernels through the same
interface), so the exchange plan, the regrouping and the return path are checked
against the oracle's layer on each rank's tokens with all experts.
"""
import datetime
import json
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_exchange_plan():
    from mixture_experts_ffn_15_b200.expert_parallel import exchange_plan, owned_experts
    assert owned_experts(8, 2, 0) == (0, 4) and owned_experts(8, 2, 1) == (4, 8)
    with pytest.raises(ValueError):
        owned_experts(6, 4, 0)
    send, recv, ids = exchange_plan([[1, 0, 2], [3, 0, 0]], [[2, 1, 0], [0, 0, 3]])
    assert send == [3, 3] and recv == [3, 3]
    assert ids == [0, 0, 1, 2, 2, 2]          # source-major, then expert
    send, recv, ids = exchange_plan([[0, 0], [0, 0]], [[0, 0], [0, 0]])
    assert send == [0, 0] and recv == [0, 0] and ids == []


class OracleOps:
    """The four computing steps of the layer on host tensors, by the oracle."""

    def route(self, hidden, router_w, k, normalize, router_bias):
        import torch
        from oracle import moe_oracle as O
        L = O.router_logits(hidden.numpy(), router_w.numpy(),
                            None if router_bias is None else router_bias.numpy())
        idx = O.select_topk(L, k)
        w = O.routing_weights(L, idx, int(normalize))
        return torch.from_numpy(idx.astype(np.int32)), torch.from_numpy(np.asarray(w, dtype=np.float64))

    def permute(self, topk_idx, E, hidden):
        import torch
        from oracle import moe_oracle as O
        counts, offsets, src, dst = O.stable_permutation(topk_idx.numpy().astype(np.int64), E)
        x_perm = O.gather_rows(hidden.numpy(), src)
        return (torch.from_numpy(np.asarray(counts, dtype=np.int32)), np.asarray(offsets),
                torch.from_numpy(np.asarray(dst, dtype=np.int64)),
                torch.from_numpy(np.ascontiguousarray(x_perm, dtype=np.float64)))

    def expert_ffn(self, x_perm, offsets, fc1, fc2):
        import torch
        from oracle import moe_oracle as O
        x = x_perm.numpy()
        y = np.zeros_like(x)
        for e in range(len(offsets) - 1):
            a, b = int(offsets[e]), int(offsets[e + 1])
            if b > a:
                y[a:b] = O.expert_ffn(x[a:b], fc1[e].numpy(), fc2[e].numpy())
        return torch.from_numpy(y)

    def combine(self, y_perm, perm_dst, topk_w, T, k):
        import torch
        from oracle import moe_oracle as O
        return torch.from_numpy(O.combine(y_perm.numpy(), perm_dst.numpy(), topk_w.numpy(), T, k))


def _rank_main(rank, world, port, out_dir, skew):
    import sys

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from mixture_experts_ffn_15_b200.expert_parallel import ep_forward, owned_experts
    from oracle import moe_oracle as O
    from synth import Workload, make_inputs
    from test_expert_parallel import OracleOps

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = Workload("ep", T=24 + 7 * rank, H=32, E=8, k=2, I=16, dtype="f32", seed=1)
        weights = make_inputs(wl.with_(T=1))                  # experts and router, shared
        hidden = make_inputs(wl, seed=10 + rank, weights=False).values("hidden")
        rw = weights.values("router_w")
        bias = None
        if skew:   # every token picks experts 0-3: rank 1 receives nothing
            bias = np.array([10.0] * 4 + [0.0] * 4, dtype=np.float32)
        fc1, fc2 = weights.values("fc1"), weights.values("fc2")
        lo, hi = owned_experts(wl.E, world, rank)
        out = ep_forward(torch.from_numpy(hidden.astype(np.float64)),
                         torch.from_numpy(rw.astype(np.float64)),
                         torch.from_numpy(fc1[lo:hi].astype(np.float64)),
                         torch.from_numpy(fc2[lo:hi].astype(np.float64)), wl.k,
                         router_bias=None if bias is None else torch.from_numpy(bias),
                         ops=OracleOps())
        ref = O.moe_forward(hidden, rw, bias, fc1, fc2, wl.k, 1)["out"]
        err = float(np.max(np.abs(out.numpy() - ref)) / max(1e-30, np.max(np.abs(ref))))
        dist.barrier()
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"err": err, "shape": list(out.shape)}, f)


@pytest.mark.parametrize("skew", [False, True], ids=["spread", "one_rank_idle"])
def test_two_gloo_ranks_expert_parallel_equals_the_layer(tmp_path, skew):
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path), skew), nprocs=2, join=True,
                       start_method="spawn")
    for rank in range(2):
        r = json.load(open(tmp_path / f"rank{rank}.json"))
        assert r["shape"] == [24 + 7 * rank, 32]
        assert r["err"] < 1e-12, (rank, r["err"])
