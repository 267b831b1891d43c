"""Expert parallelism: the MoE layer with its experts split over the ranks of a process
group (one process per GPU), every rank routing its own tokens.

Rank r owns the experts [r E/N, (r+1) E/N) (E divisible by the world size N) and holds
only their fc1 / fc2.  One call on every rank, in the same order:

1. route and permute the rank's own tokens (the library's kernels): the permuted rows
   are grouped by expert, hence by the rank that owns the expert;
2. exchange the per-expert row counts (all-to-all of an [N, E/N] matrix), then the rows
   themselves (all-to-all-v);
3. the received rows, ordered by (source rank, expert, token), are regrouped by local
   expert with the permutation kernel (k = 1: expert ids are the rows' owners' local
   indices, the order inside an expert stays source-major), and the expert FFN runs on
   them;
4. the combine kernel with k = 1 and weight 1 puts the outputs back in received order
   (an exact copy: 1.0 * y in float32, rounded back to the input dtype), they travel
   back by the inverse all-to-all-v, and each rank's combine applies its own routing
   weights.

The exchange uses torch.distributed (NCCL over NVLink on GPUs); the row-count matrix
crosses to the host once per call to size the all-to-all-v.  Every computing step is
one of the library's kernels through `KernelOps`; `ops` may be any object with the
same four methods (the CPU tests pass one that runs on host tensors, so that the
exchange logic runs with gloo ranks).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import ops as _ops


class KernelOps:
    """The library's kernels (CUDA tensors)."""

    def route(self, hidden, router_w, k, normalize, router_bias):
        r = _ops.route(hidden, router_w, k, normalize=normalize, router_bias=router_bias)
        return r["idx"], r["w"]

    def permute(self, topk_idx, E, hidden):
        p = _ops.permute(topk_idx, E, hidden=hidden)
        return p["counts"], p["offsets"], p["perm_dst"], p["x_perm"]

    def expert_ffn(self, x_perm, offsets, fc1, fc2, **kw):
        return _ops.expert_ffn(x_perm, offsets, fc1, fc2, **kw)

    def combine(self, y_perm, perm_dst, topk_w, T, k):
        return _ops.combine(y_perm, perm_dst, topk_w, T, k)


def owned_experts(E: int, world: int, rank: int):
    """[lo, hi): the experts rank `rank` owns."""
    if E % world:
        raise ValueError(f"E = {E} experts do not split evenly over {world} ranks")
    n = E // world
    return rank * n, (rank + 1) * n


def exchange_plan(counts_by_dst, recv_counts):
    """Host arithmetic of one exchange.

    counts_by_dst [N, E/N]: rows this rank sends to each rank, per destination expert
    (this rank's per-expert counts, grouped by owner); recv_counts [N, E/N]: rows this
    rank receives from each source, per local expert.  Returns (send_splits,
    recv_splits, local_ids): rows per destination, rows per source, and the local expert
    id of every received row in arrival order (source-major, then expert)."""
    send_splits = [int(sum(row)) for row in counts_by_dst]
    recv_splits = [int(sum(row)) for row in recv_counts]
    local_ids = []
    for row in recv_counts:
        for e, c in enumerate(row):
            local_ids.extend([e] * int(c))
    return send_splits, recv_splits, local_ids


def ep_forward(hidden, router_w, fc1_local, fc2_local, k, group=None, normalize=True,
               router_bias=None, ops=None, **ffn_kw):
    """The layer on this rank's tokens with experts split over `group` (see the module
    docstring).  fc1_local [E/N, 2I, H], fc2_local [E/N, H, I]: this rank's experts;
    router_w [E, H] and router_bias [E]: all experts (replicated).  Returns out [T, H]."""
    ops = ops if ops is not None else KernelOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    T, H = hidden.shape
    E = router_w.shape[0]
    lo, hi = owned_experts(E, world, rank)
    n_local = hi - lo
    if fc1_local.shape[0] != n_local or fc2_local.shape[0] != n_local:
        raise ValueError(f"rank {rank} owns {n_local} experts; got fc1 {tuple(fc1_local.shape)}, "
                         f"fc2 {tuple(fc2_local.shape)}")

    # 1. this rank's routing; rows grouped by expert, hence by owning rank
    topk_idx, topk_w = ops.route(hidden, router_w, k, normalize, router_bias)
    counts, _, perm_dst, x_perm = ops.permute(topk_idx, E, hidden)

    # 2. counts, then rows
    counts_i32 = counts.to(torch.int32).reshape(world, n_local).contiguous()
    recv_counts = torch.empty_like(counts_i32)
    dist.all_to_all_single(recv_counts, counts_i32, group=group)
    send_splits, recv_splits, local_ids = exchange_plan(counts_i32.cpu().tolist(),
                                                        recv_counts.cpu().tolist())
    n_recv = sum(recv_splits)
    x_recv = torch.empty((n_recv, H), dtype=x_perm.dtype, device=x_perm.device)
    dist.all_to_all_single(x_recv, x_perm[:sum(send_splits)].contiguous(), recv_splits,
                           send_splits, group=group)

    # 3. regroup by local expert (k = 1 permutation) and the expert FFN
    if n_recv > 0:
        ids = torch.tensor(local_ids, dtype=torch.int32).reshape(n_recv, 1).to(x_recv.device)
        _, offsets2, perm_dst2, x_local = ops.permute(ids, n_local, x_recv)
        y_local = ops.expert_ffn(x_local, offsets2, fc1_local, fc2_local, **ffn_kw)
        # 4. back to arrival order: k = 1, weight 1 (exact)
        ones = torch.ones((n_recv, 1), dtype=torch.float32, device=x_recv.device)
        y_recv = ops.combine(y_local, perm_dst2, ones, n_recv, 1)
    else:
        y_recv = torch.empty((0, H), dtype=x_perm.dtype, device=x_perm.device)
    y_back = torch.empty((sum(send_splits), H), dtype=x_perm.dtype, device=x_perm.device)
    dist.all_to_all_single(y_back, y_recv.contiguous(), send_splits, recv_splits, group=group)
    return ops.combine(y_back, perm_dst, topk_w, T, k)
