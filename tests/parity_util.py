"""Helpers shared by the GPU parity tests: device transfer, routing match, tolerances.

Routing match: where the oracle flags a near tie (float32 logits of two candidate
experts within 1e-5), more than one selection is correct.  The oracle enumerates
the valid selections (`valid_selections`) and valid slot orders; the test picks the
oracle-generated routing equal to the GPU's and checks every downstream value
(weights, counts, permutation, output) against the oracle run on that routing.
Tokens without a flag must match the oracle's own selection exactly.
"""
import numpy as np
import torch

from oracle import moe_oracle as O

# bf16 storage, float32 accumulation (stated for the layer): |d| <= 1e-2 + 2e-2 |ref|
BF16_ATOL, BF16_RTOL = 1e-2, 2e-2
# float32: 1e-4 relative, plus a floor for outputs near zero (cancellation) of
# 1e-5 x the RMS of the compared tensor.  Float32 accumulation of n <= 4096 terms
# leaves rounding of order sqrt(n) * 2^-24 ~ 4e-6 of the output scale, inside the
# floor; a TF32 product (2^-11 relative) would exceed it by two orders of magnitude.
F32_ATOL, F32_RTOL = 0.0, 1e-4
F32_RMS_FLOOR = 1e-5
# routing weights are float32 softmax values of float32 logits
W_ATOL = 1e-5


def tol(dtype, ref=None):
    """(atol, rtol) for outputs of the given storage dtype compared with `ref`."""
    if dtype == "bf16":
        return BF16_ATOL, BF16_RTOL
    floor = 0.0 if ref is None else F32_RMS_FLOOR * float(np.sqrt(np.mean(np.square(ref))))
    return F32_ATOL + floor, F32_RTOL


def assert_close(got, ref, atol, rtol, what, extra=None):
    """|got - ref| <= atol + rtol |ref| elementwise (atol a scalar or an array that
    broadcasts).  `extra` (same shape as ref, or None) is an additional per-element
    allowance; the elements that need it -- beyond the stated bound, within the
    stated bound plus `extra` -- are counted and printed.  Returns that count."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    d = np.abs(got - ref)
    stated = atol + rtol * np.abs(ref)
    lim = stated if extra is None else stated + extra
    bad = d > lim
    if bad.any():
        i = np.unravel_index(np.argmax(d - lim), d.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {d.size} elements out of tolerance; worst at {i}: "
            f"got {got[i]!r} ref {ref[i]!r} |d|={d[i]:.3e} limit={lim[i]:.3e}")
    n_extra = 0
    if extra is not None:
        n_extra = int(np.count_nonzero(d > stated))
        print(f"{what}: {n_extra} of {d.size} elements beyond the stated bound and within "
              f"the bf16 storage allowance; worst |d|/stated = {float(np.max(d / stated)):.3f}")
    return n_extra


def to_dev(a, dtype, device="cuda"):
    """numpy storage array (uint16 bf16 bits or float32) -> torch tensor on the device."""
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def from_dev(t):
    """torch tensor -> numpy float64 (bf16 widened exactly) or int array."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.float().numpy().astype(np.float64)
    if t.dtype in (torch.float32, torch.float64):
        return t.numpy().astype(np.float64)
    return t.numpy()


def device_inputs(inp):
    dt = inp.wl.dtype
    return dict(
        hidden=to_dev(inp["hidden"], dt),
        router_w=to_dev(inp["router_w"], dt),
        router_bias=to_dev(inp["router_bias"], dt),
        fc1=to_dev(inp["fc1"], dt),
        fc2=to_dev(inp["fc2"], dt),
    )


def _order_is_valid(L32_row, order, gap):
    vals = [float(L32_row[e]) for e in order]
    for a in range(len(vals)):
        for b in range(a + 1, len(vals)):
            if vals[a] < vals[b] - gap:
                return False
    return True


def match_routing(L64, gpu_idx, k, gap=O.NEAR_TIE_GAP):
    """The oracle-valid routing equal to the GPU's, token by token.

    Returns (idx [T, k] int32, n_changed).  Raises AssertionError where the GPU's
    selection is not one the oracle accepts.
    """
    L64 = np.asarray(L64)
    gpu_idx = np.asarray(gpu_idx)
    mine = O.select_topk(L64, k)
    flags = O.near_tie_flags(L64, k, gap)
    L32 = L64.astype(np.float32)
    out = mine.copy()
    changed = 0
    for t in np.nonzero(np.any(mine != gpu_idx, axis=1))[0]:
        g = [int(e) for e in gpu_idx[t]]
        assert flags[t] != 0, (
            f"token {t}: GPU chose {g}, oracle {list(mine[t])}, and the oracle sees no near tie")
        valid_sets = [set(s) for s in O.valid_selections(L64[t], k, gap)]
        assert set(g) in valid_sets, f"token {t}: GPU set {sorted(g)} is not a valid selection"
        assert _order_is_valid(L32[t], g, gap), f"token {t}: GPU slot order {g} is not valid"
        out[t] = g
        changed += 1
    return out, changed


def sample_tokens(T, idx, E, n=256, must=(), seed=123):
    """A seeded token sample that includes `must` and tokens of the least/most loaded experts."""
    rng = np.random.default_rng(seed)
    counts = np.bincount(np.asarray(idx).ravel(), minlength=E)
    used = np.nonzero(counts)[0]
    picks = set(int(t) for t in must)
    for e in (used[np.argmin(counts[used])], int(np.argmax(counts))):
        toks = np.nonzero(np.any(np.asarray(idx) == e, axis=1))[0]
        picks.update(int(t) for t in toks[:4])
    picks.update([0, T - 1])
    extra = rng.choice(T, size=min(T, n), replace=False)
    picks.update(int(t) for t in extra)
    return np.array(sorted(picks), dtype=np.int64)


def bf16_storage_bound(act, fc2_e, y):
    """First-order bound on what storing act and y in bf16 (round to nearest, relative
    error <= 2^-9 each) moves y = act fc2^T: 2^-9 (|act| |fc2|^T + |y|), per element.
    act [n, I], fc2_e [H, I], y [n, H], all exact (float64)."""
    u = 2.0 ** -9
    return u * (np.abs(act) @ np.abs(fc2_e).T + np.abs(y))


def scaled_row_storage_bound(inp, idx, tokens, scaled_rows):
    """The bf16 storage allowance of the layer's output on the rows the input generator
    scaled up (the long-prefill workload's x8 outlier rows), zero on every other row.

    For token t and its chosen experts e_j with routing weights w_j (the oracle's, from
    its float64 logits): sum_j w_j 2^-9 (|a_j| |fc2_e_j|^T + |y_j|), a_j = the oracle's
    SwiGLU of t under e_j and y_j = a_j fc2_e_j^T -- what bf16 storage of the
    intermediates act and y_perm may move the output by, to first order.  An x8 input
    row makes its gate and up values 8 times larger and its act ~64 times larger, so
    the absolute term of the stated tolerance, sized for ordinary rows, cannot hold
    there for any kernel that stores act in bf16.

    Returns [len(tokens), H] float64 (standard SwiGLU, no expert biases)."""
    wl = inp.wl
    tokens = np.asarray(tokens, dtype=np.int64)
    scaled = set(int(t) for t in np.asarray(scaled_rows).tolist())
    out = np.zeros((tokens.size, wl.H))
    pick = [i for i, t in enumerate(tokens.tolist()) if t in scaled]
    if not pick:
        return out
    x = inp.values("hidden")
    L = O.router_logits(x[tokens[pick]], inp.values("router_w"), inp["router_bias"])
    w = O.routing_weights(L, np.asarray(idx)[tokens[pick]], wl.normalize)
    sub_idx = np.asarray(idx)[tokens[pick]]
    for e in np.unique(sub_idx):
        rows, slots = np.nonzero(sub_idx == e)
        xe = x[tokens[pick][rows]].astype(np.float64)
        w_gate, w_up = O.fc1_gate_up(inp.expert_values("fc1", int(e)).astype(np.float64),
                                     wl.fc1_layout)
        a = O.swiglu(xe @ w_gate.T, xe @ w_up.T)
        fc2_e = inp.expert_values("fc2", int(e)).astype(np.float64)
        b = bf16_storage_bound(a, fc2_e, a @ fc2_e.T)
        np.add.at(out, np.asarray(pick)[rows], w[rows, slots][:, None] * b)
    return out
