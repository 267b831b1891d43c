"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Indices, counts and permutations are compared bit-exactly (near ties resolved
through oracle-generated alternatives, see parity_util); values within the stated
tolerances: bf16 |d| <= 1e-2 + 2e-2 |ref|, float32 |d| <= 1e-6 + 1e-4 |ref|.
"""
import numpy as np
import pytest
import torch

import mixture_experts_ffn_15_b200 as moe
from oracle import moe_oracle as O
from parity_util import (W_ATOL, assert_close, bf16_storage_bound, device_inputs, from_dev,
                         match_routing, sample_tokens, scaled_row_storage_bound, to_dev, tol)
from synth import Workload, bf16_bits_to_f32, make_inputs, round_to_bf16_bits

pytestmark = pytest.mark.gpu


def W(name, **kw):
    base = dict(T=64, H=128, E=8, k=2, I=64, dtype="bf16", seed=1)
    base.update(kw)
    return Workload(name, **base)


# Small cases: several tiles in every dimension with ragged tails, both orientations
# of the tensor-core GEMM, every column-tile width, the float32 path and edge cases.
CASES = [
    W("f32_tiles", T=300, H=256, E=16, k=4, I=192, dtype="f32"),
    W("f32_T1", T=1, H=64, E=4, k=2, I=32, dtype="f32"),
    W("f32_normalize_off", T=70, H=64, E=6, k=3, I=32, dtype="f32", normalize=0),
    W("bf16_tokenM_bn192", T=300, H=256, E=16, k=4, I=192),
    W("bf16_tokenM_bn176", T=300, H=128, E=8, k=2, I=704),
    W("bf16_tokenM_bias", T=520, H=192, E=8, k=2, I=64, router_bias_std=1.0),
    # CTA pairs with more units than pairs and an odd number of 64-K slices in both
    # GEMMs (23 and 3): the slot ring wraps after short last stages
    W("bf16_tokenM_odd_k_wrap", T=6144, H=1472, E=8, k=2, I=192),
    W("bf16_weightM", T=40, H=256, E=16, k=4, I=192),
    W("bf16_weightM_skew", T=100, H=256, E=8, k=2, I=128, router_bias_std=1.0),
    W("bf16_router_tc", T=600, H=256, E=64, k=4, I=128),
    W("bf16_router_tc_k16_E256", T=150, H=128, E=256, k=16, I=64),
    W("bf16_router_tc_norm0_bias", T=300, H=192, E=128, k=6, I=64, normalize=0,
      router_bias_std=0.5),
    W("bf16_router_tc_T17", T=17, H=64, E=64, k=8, I=64),
    # the whole layer in one launch (routing inside the decode FFN)
    W("bf16_onelaunch_T64_k8", T=64, H=256, E=64, k=8, I=128),
    W("bf16_onelaunch_bias_norm0", T=33, H=128, E=128, k=6, I=64, normalize=0,
      router_bias_std=0.5),
    W("bf16_onelaunch_E256_k16", T=8, H=128, E=256, k=16, I=64),
    W("bf16_k1", T=130, H=128, E=8, k=1, I=64),
    # k > 32: the float32-logit top-k, and the row-by-row gather into x_perm
    W("bf16_k40", T=40, H=128, E=64, k=40, I=64),
    W("bf16_k_eq_E", T=20, H=128, E=4, k=4, I=64),
    W("bf16_T1", T=1, H=128, E=8, k=2, I=64),
    W("bf16_normalize_off", T=90, H=128, E=8, k=3, I=64, normalize=0),
]
IDS = [c.name for c in CASES]


def oracle_forward(inp, idx, tokens=None):
    wl = inp.wl
    layout = wl.fc1_layout
    return O.moe_forward(inp.values("hidden"), inp.values("router_w"), inp["router_bias"],
                         lambda e: inp.expert_values("fc1", e),
                         lambda e: inp.expert_values("fc2", e), wl.k, wl.normalize, layout,
                         idx=idx, tokens=tokens)


def run_route(dev, wl):
    return moe.route(dev["hidden"], dev["router_w"], wl.k, normalize=bool(wl.normalize),
                     router_bias=dev["router_bias"])


def check_routing(inp, r):
    """GPU routing vs the oracle; returns (logits64, matched idx)."""
    wl = inp.wl
    L = O.router_logits(inp.values("hidden"), inp.values("router_w"), inp["router_bias"])
    gidx = from_dev(r["idx"]).astype(np.int64)
    idx, _ = match_routing(L, gidx, wl.k)
    np.testing.assert_array_equal(gidx, idx)
    # the logits: rigorous float32 summation bound gamma_H * sum_h |x w| (any order)
    H = wl.H
    xw = np.abs(inp.values("hidden")).astype(np.float64) @ np.abs(inp.values("router_w")).astype(np.float64).T
    u = 2.0 ** -24
    bound = (H * u / (1 - H * u)) * xw + 1e-7
    got = from_dev(r["logits"])
    dL = np.abs(got - L)
    assert np.all(dL <= bound), "router logits beyond the float32 summation bound"
    # the weights: softmax of the logits the GPU computed.  A logit error dL moves a
    # softmax weight by at most 2 w max|dL| (its Jacobian); on top of that float32
    # exp / sum / divide rounding (W_ATOL).
    w_ref = O.routing_weights(L, idx, wl.normalize)
    slack = 2.0 * w_ref * dL.max(axis=1, keepdims=True)
    got_w = from_dev(r["w"])
    assert np.all(np.abs(got_w - w_ref) <= W_ATOL + slack), (
        "routing weights beyond the float32 softmax of the GPU logits: max excess "
        f"{np.max(np.abs(got_w - w_ref) - W_ATOL - slack):.3e}")
    return L, idx


@pytest.mark.parametrize("wl", CASES, ids=IDS)
def test_route(wl):
    inp = make_inputs(wl)
    dev = device_inputs(inp)
    check_routing(inp, run_route(dev, wl))


@pytest.mark.parametrize("wl", CASES, ids=IDS)
def test_permute(wl):
    inp = make_inputs(wl)
    dev = device_inputs(inp)
    L = O.router_logits(inp.values("hidden"), inp.values("router_w"), inp["router_bias"])
    idx = O.select_topk(L, wl.k)
    p = moe.permute(torch.from_numpy(idx).cuda(), wl.E, hidden=dev["hidden"])
    counts, offsets, src, dst = O.stable_permutation(idx, wl.E)
    np.testing.assert_array_equal(from_dev(p["counts"]), counts)
    np.testing.assert_array_equal(from_dev(p["offsets"]), offsets)
    np.testing.assert_array_equal(from_dev(p["perm_src"]), src)
    np.testing.assert_array_equal(from_dev(p["perm_dst"]), dst)
    x_ref = O.gather_rows(inp["hidden"], src)
    got = p["x_perm"].detach().cpu()
    got = got.view(torch.int16).numpy().view(np.uint16) if got.dtype == torch.bfloat16 else got.numpy()
    np.testing.assert_array_equal(got, x_ref)
    st, bits = moe.get_error(p["err_word"])
    assert st == 0 and bits == 0


@pytest.mark.parametrize("wl", CASES, ids=IDS)
def test_expert_ffn(wl):
    inp = make_inputs(wl)
    dev = device_inputs(inp)
    L = O.router_logits(inp.values("hidden"), inp.values("router_w"), inp["router_bias"])
    idx = O.select_topk(L, wl.k)
    counts, offsets, src, dst = O.stable_permutation(idx, wl.E)
    x_perm = O.gather_rows(inp["hidden"], src)
    y = moe.expert_ffn(to_dev(x_perm, wl.dtype), torch.from_numpy(offsets).cuda(), dev["fc1"], dev["fc2"])
    torch.cuda.synchronize()
    xv = O.gather_rows(inp.values("hidden"), src)
    y_ref = np.zeros((x_perm.shape[0], wl.H))
    for e in range(wl.E):
        a, b = offsets[e], offsets[e + 1]
        if b > a:
            y_ref[a:b] = O.expert_ffn(xv[a:b], inp.expert_values("fc1", e), inp.expert_values("fc2", e))
    atol, rtol = tol(wl.dtype, y_ref)
    assert_close(from_dev(y), y_ref, atol, rtol, "y_perm")


# Expert row counts at every tile edge of the grouped GEMMs: empty, single rows, the
# 32-token rounding of a CTA-pair tile, the 64-token chunks of the decode FFN, the
# 256-token pair tile and one past each; fc1's 2I = 384 rows are a pair tile of 256
# plus a half tile, fc2's H = 256 rows one pair tile.
EDGE_COUNTS = [0, 1, 31, 32, 33, 63, 64, 65, 255, 256, 257, 300, 0, 2]


@pytest.mark.parametrize("scale", [1, 0], ids=["pair_tiles", "decode_chunks"])
def test_expert_ffn_at_tile_edges(scale):
    """moe_expert_ffn on offsets built from EDGE_COUNTS, against the oracle's expert
    FFN row block by row block.  scale=1 gives 1359 rows over 14 experts (> 64 per
    expert on average: the CTA-pair GEMMs); scale=0 keeps the counts <= 65 (the
    decode FFN, weight rows on M)."""
    counts = np.array(EDGE_COUNTS if scale else [min(c, 65) for c in EDGE_COUNTS], dtype=np.int64)
    E = len(counts)
    rows = int(counts.sum())
    wl = W("edges", T=rows, H=256, E=E, k=1, I=192)
    inp = make_inputs(wl)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    x = inp["hidden"]                      # the rows themselves stand for x_perm
    y = moe.expert_ffn(to_dev(x, wl.dtype), torch.from_numpy(offsets).cuda(), to_dev(inp["fc1"], wl.dtype),
                       to_dev(inp["fc2"], wl.dtype))
    torch.cuda.synchronize()
    xv = inp.values("hidden")
    y_ref = np.zeros((rows, wl.H))
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if b > a:
            y_ref[a:b] = O.expert_ffn(xv[a:b], inp.expert_values("fc1", e), inp.expert_values("fc2", e))
    atol, rtol = tol(wl.dtype, y_ref)
    assert_close(from_dev(y), y_ref, atol, rtol, f"y_perm at tile edges (scale {scale})")


@pytest.mark.parametrize("wl", CASES, ids=IDS)
def test_forward(wl):
    inp = make_inputs(wl)
    dev = device_inputs(inp)
    out = moe.forward(dev["hidden"], dev["router_w"], dev["fc1"], dev["fc2"], wl.k,
                      normalize=bool(wl.normalize), router_bias=dev["router_bias"])
    r = run_route(dev, wl)
    torch.cuda.synchronize()
    L, idx = check_routing(inp, r)
    ref = oracle_forward(inp, idx)["out"]
    atol, rtol = tol(wl.dtype, ref)
    assert_close(from_dev(out), ref, atol, rtol, f"{wl.name} output")


def test_token_gemm_layer_equals_the_staged_calls_bit_for_bit():
    """The layer's large-batch path (router, scatter, gather, fc1 and fc2 on CTA pairs,
    combine in one call) against the staged calls on the same inputs: same routing (the
    tensor-core router in both), same kernels, the same bits.  A skewed router gives
    experts of every size, so token tiles end at every offset."""
    from mixture_experts_ffn_15_b200 import _abi
    wl = W("token_gemm_skew", T=1500, H=256, E=64, k=4, I=192, router_bias_std=1.0)
    assert moe.load_library().moe_forward_path(wl.T, wl.H, wl.E, wl.k, wl.I, _abi.MOE_BF16) & 8
    inp = make_inputs(wl)
    dev = device_inputs(inp)
    out = moe.forward(dev["hidden"], dev["router_w"], dev["fc1"], dev["fc2"], wl.k,
                      router_bias=dev["router_bias"])
    r = run_route(dev, wl)
    p = moe.permute(r["idx"], wl.E, hidden=dev["hidden"])
    y = moe.expert_ffn(p["x_perm"], p["offsets"], dev["fc1"], dev["fc2"])
    staged = moe.combine(y, p["perm_dst"], r["w"], wl.T, wl.k)
    torch.cuda.synchronize()
    counts = from_dev(p["counts"])
    assert counts.min() < 32 and counts.max() > 256       # ragged tiles of every kind
    assert torch.equal(out.view(torch.int16), staged.view(torch.int16))
    L, idx = check_routing(inp, r)
    ref = oracle_forward(inp, idx)["out"]
    atol, rtol = tol(wl.dtype, ref)
    assert_close(from_dev(out), ref, atol, rtol, "token GEMM layer")


# ------------------------------------------- SwiGLU attributes and expert biases
# The op's activation_alpha / activation_beta / swiglu_limit ("Attribute set") and its
# optional fc1/fc2 expert biases, on every path of moe_forward.  limit 1.0 clips most
# gate and up values; the GPT-OSS values clip a few.
ATTR_CASES = [
    W("attr_one_launch", T=4, H=256, E=64, k=4, I=128),
    W("attr_router_decode", T=100, H=256, E=64, k=4, I=128, router_bias_std=0.5),
    W("attr_pairs", T=1100, H=256, E=64, k=4, I=192),
    W("attr_f32", T=70, H=64, E=6, k=3, I=32, dtype="f32"),
]
ATTRS = [("gpt_oss", (1.702, 1.0, 7.0)), ("clip_heavy", (0.5, -0.25, 1.0))]


@pytest.mark.parametrize("biased", [False, True], ids=["no_bias", "bias"])
@pytest.mark.parametrize("attr", ATTRS, ids=[a[0] for a in ATTRS])
@pytest.mark.parametrize("wl", ATTR_CASES, ids=[c.name for c in ATTR_CASES])
def test_forward_swiglu_attributes_and_biases(wl, attr, biased):
    from synth import make_expert_biases
    inp = make_inputs(wl)
    dev = device_inputs(inp)
    act = attr[1]
    b1 = b2 = None
    db1 = db2 = None
    if biased:
        b1, b2 = make_expert_biases(wl)
        db1, db2 = to_dev(b1, wl.dtype), to_dev(b2, wl.dtype)
    out = moe.forward(dev["hidden"], dev["router_w"], dev["fc1"], dev["fc2"], wl.k,
                      normalize=bool(wl.normalize), router_bias=dev["router_bias"], swiglu=act,
                      fc1_bias=db1, fc2_bias=db2)
    r = run_route(dev, wl)
    torch.cuda.synchronize()
    L, idx = check_routing(inp, r)
    f = lambda a: None if a is None else (bf16_bits_to_f32(a) if a.dtype == np.uint16 else a)
    ref = O.moe_forward(inp.values("hidden"), inp.values("router_w"), inp["router_bias"],
                        lambda e: inp.expert_values("fc1", e), lambda e: inp.expert_values("fc2", e),
                        wl.k, wl.normalize, wl.fc1_layout, idx=idx, act=act,
                        fc1_bias=f(b1), fc2_bias=f(b2))["out"]
    atol, rtol = tol(wl.dtype, ref)
    assert_close(from_dev(out), ref, atol, rtol, f"{wl.name} {attr[0]} biased={biased}")


def test_expert_ffn_attributes_and_biases_on_both_bf16_kernels():
    """moe_expert_ffn with the GPT-OSS attributes and biases: few rows per expert (the
    decode FFN) and many (the CTA pairs)."""
    from synth import make_expert_biases
    for rows_per_expert, name in ((6, "decode"), (300, "pairs")):
        wl = W("attr_ffn_" + name, T=rows_per_expert * 8, H=256, E=8, k=1, I=128)
        inp = make_inputs(wl)
        b1, b2 = make_expert_biases(wl, seed=5)
        offsets = (np.arange(wl.E + 1) * rows_per_expert).astype(np.int32)
        act = (1.702, 1.0, 7.0)
        y = moe.expert_ffn(to_dev(inp["hidden"], wl.dtype), torch.from_numpy(offsets).cuda(),
                           to_dev(inp["fc1"], wl.dtype), to_dev(inp["fc2"], wl.dtype), swiglu=act,
                           fc1_bias=to_dev(b1, wl.dtype), fc2_bias=to_dev(b2, wl.dtype))
        torch.cuda.synchronize()
        xv = inp.values("hidden")
        y_ref = np.zeros((wl.T, wl.H))
        bound = np.zeros((wl.T, wl.H))
        for e in range(wl.E):
            a, b = offsets[e], offsets[e + 1]
            fc1_e, fc2_e = inp.expert_values("fc1", e), inp.expert_values("fc2", e)
            b1_e, b2_e = bf16_bits_to_f32(b1[e]), bf16_bits_to_f32(b2[e])
            y_ref[a:b] = O.expert_ffn(xv[a:b], fc1_e, fc2_e, "interleaved", act, b1_e, b2_e)
            # the activations themselves, for the bound of their bf16 storage
            g = xv[a:b].astype(np.float64) @ fc1_e[0::2].T.astype(np.float64) + b1_e[0::2]
            u = xv[a:b].astype(np.float64) @ fc1_e[1::2].T.astype(np.float64) + b1_e[1::2]
            bound[a:b] = bf16_storage_bound(O.swiglu(g, u, *act), fc2_e.astype(np.float64), y_ref[a:b])
        # y_perm is an intermediate (each row before its routing weight): the beta on
        # the up branch and the biases roughly double |act|, and with it the error of
        # storing act in bf16.  The stated tolerance plus that storage bound; the
        # layer-level tests of the same attributes keep the stated tolerance alone.
        atol, rtol = tol(wl.dtype, y_ref)
        assert_close(from_dev(y), y_ref, atol, rtol, f"y_perm {name}", extra=bound)


# ------------------------------------------- fc1 in the chunked layout, read in place
# "Weight layout": Hugging Face stores gate_up_proj chunked (gate rows, then up rows);
# the op's CUDA kernel accepts either layout.  Every path reads the chunked weights
# (and a chunked fc1 bias) where they are: the result must be bit for bit the result
# on the same weights converted to the interleaved layout, and match the oracle's
# chunked reading.
LAYOUT_CASES = [
    W("chunked_one_launch", T=4, H=256, E=64, k=4, I=128, fc1_layout="chunked"),
    W("chunked_router_decode", T=100, H=256, E=64, k=4, I=192, fc1_layout="chunked"),
    W("chunked_small_decode", T=100, H=256, E=16, k=4, I=128, fc1_layout="chunked"),
    W("chunked_pairs", T=1100, H=256, E=64, k=4, I=192, fc1_layout="chunked"),
    # 2I = 1408 rows: the last 256-row tile of each expert is half padding
    W("chunked_pairs_half_tile", T=1100, H=128, E=8, k=2, I=704, fc1_layout="chunked"),
    W("chunked_f32", T=70, H=64, E=6, k=3, I=32, dtype="f32", fc1_layout="chunked"),
]


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


@pytest.mark.parametrize("biased", [False, True], ids=["standard", "gpt_oss_bias"])
@pytest.mark.parametrize("wl", LAYOUT_CASES, ids=[c.name for c in LAYOUT_CASES])
def test_forward_reads_chunked_fc1_in_place(wl, biased):
    from synth import make_expert_biases
    inp = make_inputs(wl)
    dev = device_inputs(inp)
    act = (1.702, 1.0, 7.0) if biased else (1.0, 0.0, float("inf"))
    b1 = b2 = None
    if biased:
        b1, b2 = make_expert_biases(wl, seed=3)      # b1 read in fc1's (chunked) layout
    d = lambda a: None if a is None else to_dev(a, wl.dtype)
    kw = dict(normalize=bool(wl.normalize), router_bias=dev["router_bias"], swiglu=act)
    out_c = moe.forward(dev["hidden"], dev["router_w"], dev["fc1"], dev["fc2"], wl.k,
                        fc1_bias=d(b1), fc2_bias=d(b2), fc1_layout="chunked", **kw)
    fc1_i = to_dev(O.chunked_to_interleaved(inp["fc1"]), wl.dtype)
    b1_i = None if b1 is None else O.chunked_to_interleaved(b1)
    out_i = moe.forward(dev["hidden"], dev["router_w"], fc1_i, dev["fc2"], wl.k,
                        fc1_bias=d(b1_i), fc2_bias=d(b2), **kw)
    torch.cuda.synchronize()
    assert torch.equal(_bits(out_c), _bits(out_i)), f"{wl.name}: chunked != interleaved"
    r = run_route(dev, wl)
    torch.cuda.synchronize()
    L, idx = check_routing(inp, r)
    f = lambda a: None if a is None else (bf16_bits_to_f32(a) if a.dtype == np.uint16 else a)
    ref = O.moe_forward(inp.values("hidden"), inp.values("router_w"), inp["router_bias"],
                        lambda e: inp.expert_values("fc1", e), lambda e: inp.expert_values("fc2", e),
                        wl.k, wl.normalize, "chunked", idx=idx, act=act,
                        fc1_bias=f(b1), fc2_bias=f(b2))["out"]
    atol, rtol = tol(wl.dtype, ref)
    assert_close(from_dev(out_c), ref, atol, rtol, f"{wl.name} chunked biased={biased}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_expert_ffn_reads_chunked_fc1_in_place(dtype):
    """moe_expert_ffn with chunked fc1 and fc1 bias: bit-equal to the interleaved call,
    for few rows per expert (the decode FFN) and many (the CTA pairs)."""
    from synth import make_expert_biases
    for rows_per_expert, name in ((6, "decode"), (300, "pairs")):
        wl = W("chunked_ffn_" + name, T=rows_per_expert * 8, H=256, E=8, k=1, I=192,
               dtype=dtype, fc1_layout="chunked")
        inp = make_inputs(wl)
        b1, b2 = make_expert_biases(wl, seed=6)
        offsets = torch.from_numpy((np.arange(wl.E + 1) * rows_per_expert).astype(np.int32)).cuda()
        x = to_dev(inp["hidden"], dtype)
        fc2, db2 = to_dev(inp["fc2"], dtype), to_dev(b2, dtype)
        act = (1.702, 1.0, 7.0)
        y_c = moe.expert_ffn(x, offsets, to_dev(inp["fc1"], dtype), fc2, swiglu=act,
                             fc1_bias=to_dev(b1, dtype), fc2_bias=db2, fc1_layout="chunked")
        y_i = moe.expert_ffn(x, offsets, to_dev(O.chunked_to_interleaved(inp["fc1"]), dtype), fc2,
                             swiglu=act, fc1_bias=to_dev(O.chunked_to_interleaved(b1), dtype),
                             fc2_bias=db2)
        torch.cuda.synchronize()
        assert torch.equal(_bits(y_c), _bits(y_i)), name


# ------------------------------------------------------------------ pre-FFN RMSNorm
# The Llama-style norm in front of the layer ("Contributing Gemma 4 support and ONNX
# export optimizations", "Key Technical Contributions").  Both sides evaluate it in
# float64 and round once to the storage dtype; the float64 values differ by a few
# float64 ulps at most (the order of the sums), which moves a bf16 or float32 rounding
# only for values within ~1e-15 relative of a rounding boundary: the results are
# compared bit for bit.
NORM_SHAPES = [(1, 64, "bf16", 4.0), (37, 2816, "bf16", 4.0), (300, 72, "bf16", 300.0),
               (64, 256, "bf16", 1e-3), (33, 136, "f32", 4.0), (5, 2816, "f32", 50.0)]


def _bits_np(a, dtype):
    return a.astype(np.float32).view(np.uint32) if dtype == "f32" else \
        round_to_bf16_bits(a.astype(np.float32))


@pytest.mark.parametrize("T,H,dtype,scale", NORM_SHAPES,
                         ids=[f"T{t}_H{h}_{d}_x{s:g}" for t, h, d, s in NORM_SHAPES])
def test_rmsnorm_bitexact(T, H, dtype, scale):
    from synth import make_pre_norm_inputs
    wl = W("norm", T=T, H=H, dtype=dtype)
    x, w = make_pre_norm_inputs(wl, scale=scale)
    eps = float(np.float32(1e-6))
    xv = bf16_bits_to_f32(x) if dtype == "bf16" else x
    wv = bf16_bits_to_f32(w) if dtype == "bf16" else w
    if T > 3:
        x = x.copy()
        x[3] = 0                              # an all-zero row: eps keeps it at zero
        x[2, :5] = 0x8000 if dtype == "bf16" else np.float32(-0.0)   # signed zeros stay signed
        xv = bf16_bits_to_f32(x) if dtype == "bf16" else x
    got = moe.rmsnorm(to_dev(x, dtype), to_dev(w, dtype), eps)
    ref = O.pre_ffn_norm(xv, wv, eps, dtype)
    got_bits = got.cpu().view(torch.int16).numpy().view(np.uint16) if dtype == "bf16" else \
        got.cpu().numpy().view(np.uint32)
    np.testing.assert_array_equal(got_bits, _bits_np(ref, dtype))


NORM_CASES = [
    W("norm_one_launch", T=4, H=256, E=64, k=4, I=128),
    W("norm_router_decode", T=100, H=256, E=64, k=4, I=128, router_bias_std=0.5),
    W("norm_small_decode", T=100, H=256, E=16, k=4, I=128),
    W("norm_pairs", T=1100, H=256, E=64, k=4, I=192),
    W("norm_f32", T=70, H=64, E=6, k=3, I=32, dtype="f32"),
]


@pytest.mark.parametrize("wl", NORM_CASES, ids=[c.name for c in NORM_CASES])
def test_forward_with_pre_norm(wl):
    """moe_forward(x, norm_weight) on every path: bit-equal to moe_rmsnorm followed by the
    plain layer, and the oracle's layer on the oracle's norm of x within tolerance."""
    from synth import make_pre_norm_inputs
    inp = make_inputs(wl)
    dev = device_inputs(inp)
    x, w = make_pre_norm_inputs(wl)
    dx, dw = to_dev(x, wl.dtype), to_dev(w, wl.dtype)
    eps = float(np.float32(1e-5))
    kw = dict(normalize=bool(wl.normalize), router_bias=dev["router_bias"])
    fused = moe.forward(dx, dev["router_w"], dev["fc1"], dev["fc2"], wl.k, norm_weight=dw,
                        norm_eps=eps, **kw)
    xn = moe.rmsnorm(dx, dw, eps)
    staged = moe.forward(xn, dev["router_w"], dev["fc1"], dev["fc2"], wl.k, **kw)
    torch.cuda.synchronize()
    assert torch.equal(_bits(fused), _bits(staged)), wl.name
    f = lambda a: bf16_bits_to_f32(a) if a.dtype == np.uint16 else a
    xn_ref = O.pre_ffn_norm(f(x), f(w), eps, wl.dtype)
    got_xn = xn.cpu().view(torch.int16).numpy().view(np.uint16) if wl.dtype == "bf16" else \
        xn.cpu().numpy().view(np.uint32)
    np.testing.assert_array_equal(got_xn, _bits_np(xn_ref, wl.dtype))
    # routing of the normalised input, then the layer, against the oracle
    r = moe.route(xn, dev["router_w"], wl.k, normalize=bool(wl.normalize),
                  router_bias=dev["router_bias"])
    torch.cuda.synchronize()
    L = O.router_logits(xn_ref, inp.values("router_w"), inp["router_bias"])
    gidx = from_dev(r["idx"]).astype(np.int64)
    idx, _ = match_routing(L, gidx, wl.k)
    np.testing.assert_array_equal(gidx, idx)
    ref = O.moe_forward(xn_ref, inp.values("router_w"), inp["router_bias"],
                        lambda e: inp.expert_values("fc1", e), lambda e: inp.expert_values("fc2", e),
                        wl.k, wl.normalize, wl.fc1_layout, idx=idx)["out"]
    atol, rtol = tol(wl.dtype, ref)
    assert_close(from_dev(fused), ref, atol, rtol, f"{wl.name} with pre-FFN norm")


@pytest.mark.parametrize("name", ["decode_bf16", "prefill_bf16"])
def test_full_workload_with_pre_norm(name):
    """The full-size layer with the pre-FFN norm: the norm bit-exact against the oracle
    on every element, and the fused call bit-equal to the norm followed by the layer
    (whose parity the full-workload tests establish)."""
    from synth import WORKLOADS, make_pre_norm_inputs
    wl = WORKLOADS[name]
    inp = make_inputs(wl)
    dev = device_inputs(inp)
    x, w = make_pre_norm_inputs(wl)
    dx, dw = to_dev(x, wl.dtype), to_dev(w, wl.dtype)
    eps = float(np.float32(1e-6))
    xn = moe.rmsnorm(dx, dw, eps)
    ref = O.pre_ffn_norm(bf16_bits_to_f32(x), bf16_bits_to_f32(w), eps, "bf16")
    np.testing.assert_array_equal(xn.cpu().view(torch.int16).numpy().view(np.uint16),
                                  _bits_np(ref, "bf16"))
    kw = dict(normalize=bool(wl.normalize), router_bias=dev["router_bias"],
              fc1_layout=wl.fc1_layout)
    fused = moe.forward(dx, dev["router_w"], dev["fc1"], dev["fc2"], wl.k, norm_weight=dw,
                        norm_eps=eps, **kw)
    staged = moe.forward(xn, dev["router_w"], dev["fc1"], dev["fc2"], wl.k, **kw)
    torch.cuda.synchronize()
    assert torch.equal(_bits(fused), _bits(staged))


# ------------------------------------------------------------------ int8 experts
# Weight-only int8 experts (one float32 scale per weight row) in the decode FFN.
# The routing inside the launch (T <= 64), after the tensor-core router, after the
# one-CTA router (an expert count the tensor-core router does not take).
Q8_CASES = [
    W("q8_decode", T=4, H=256, E=64, k=4, I=128),
    W("q8_router_tc", T=100, H=256, E=64, k=4, I=192, router_bias_std=0.5),
    W("q8_small_route", T=100, H=128, E=16, k=4, I=128),
    W("q8_chunked_norm0", T=20, H=256, E=32, k=6, I=128, normalize=0, fc1_layout="chunked"),
    W("q8_one_launch_bias", T=48, H=256, E=16, k=4, I=128, router_bias_std=0.5),
    # decode batches of 1 to 4 tokens: 1 to 4 rows per expert, wide H and I
    W("q8_one_token", T=1, H=512, E=64, k=8, I=192),
    W("q8_every_expert_all_rows", T=4, H=256, E=4, k=4, I=128),
    W("q8_shared_experts", T=4, H=384, E=8, k=4, I=128, router_bias_std=1.0),
    W("q8_three_tokens_chunked_norm0", T=3, H=384, E=32, k=6, I=192, normalize=0,
      fc1_layout="chunked"),
    W("q8_wide", T=2, H=4096, E=4, k=2, I=1536),
    W("q8_wider_h", T=4, H=4224, E=8, k=2, I=128),
]


def _q8_dev(wl, seed=None):
    from synth import make_q8_experts
    q1, s1, q2, s2 = make_q8_experts(wl, seed)
    dev = [torch.from_numpy(a).cuda() for a in (q1, s1, q2, s2)]
    return (q1, s1, q2, s2), dev


def _q8_oracle(inp, wl, host, idx, act=(1.0, 0.0, float("inf")), b1=None, b2=None):
    q1, s1, q2, s2 = host
    return O.moe_forward(inp.values("hidden"), inp.values("router_w"), inp["router_bias"],
                         lambda e: O.dequantize_rows(q1[e], s1[e]),
                         lambda e: O.dequantize_rows(q2[e], s2[e]), wl.k, wl.normalize,
                         wl.fc1_layout, idx=idx, act=act, fc1_bias=b1, fc2_bias=b2)["out"]


@pytest.mark.parametrize("wl", Q8_CASES, ids=[c.name for c in Q8_CASES])
def test_forward_q8(wl):
    lib = moe.load_library()
    one_launch = bool(lib.moe_forward_path(wl.T, wl.H, wl.E, wl.k, wl.I, 1) & 32)
    assert one_launch == (wl.T <= 64), wl.name
    inp = make_inputs(wl, weights=False)
    dev = device_inputs(inp)
    host, (q1, s1, q2, s2) = _q8_dev(wl)
    out = moe.forward_q8(dev["hidden"], dev["router_w"], q1, s1, q2, s2, wl.k,
                         normalize=bool(wl.normalize), router_bias=dev["router_bias"],
                         fc1_layout=wl.fc1_layout)
    r = run_route(dev, wl)
    torch.cuda.synchronize()
    L, idx = check_routing(inp, r)
    ref = _q8_oracle(inp, wl, host, idx)
    atol, rtol = tol(wl.dtype, ref)
    assert_close(from_dev(out), ref, atol, rtol, f"{wl.name} int8 experts")


@pytest.mark.parametrize("T", [8, 3])
def test_forward_q8_attributes_and_biases(T):
    """The op's SwiGLU attributes and both expert biases, at 8 and at 3 tokens."""
    from synth import make_expert_biases
    wl = W("q8_attr", T=T, H=256, E=32, k=4, I=128)
    inp = make_inputs(wl, weights=False)
    dev = device_inputs(inp)
    host, (q1, s1, q2, s2) = _q8_dev(wl)
    b1, b2 = make_expert_biases(wl, seed=9)
    act = (1.702, 1.0, 7.0)
    out = moe.forward_q8(dev["hidden"], dev["router_w"], q1, s1, q2, s2, wl.k, swiglu=act,
                         fc1_bias=to_dev(b1, "bf16"), fc2_bias=to_dev(b2, "bf16"))
    r = run_route(dev, wl)
    torch.cuda.synchronize()
    L, idx = check_routing(inp, r)
    ref = _q8_oracle(inp, wl, host, idx, act, bf16_bits_to_f32(b1), bf16_bits_to_f32(b2))
    atol, rtol = tol(wl.dtype, ref)
    assert_close(from_dev(out), ref, atol, rtol, "int8 experts, GPT-OSS + biases")


@pytest.mark.parametrize("layout", ["interleaved", "chunked"])
def test_expert_ffn_q8_unit_scales_equal_bf16_kernel(layout):
    """With every scale 1 the int8 experts are the bf16 experts bf16(q) (exact): the
    int8 decode FFN must give the bf16 decode FFN's bits, biases included; with real
    scales, the oracle on q * scale."""
    from synth import make_expert_biases
    rows_per_expert = 6
    wl = W("q8_ffn", T=rows_per_expert * 8, H=256, E=8, k=1, I=192, fc1_layout=layout)
    inp = make_inputs(wl, weights=False)
    host, (q1, s1, q2, s2) = _q8_dev(wl, seed=4)
    b1, b2 = make_expert_biases(wl, seed=7)
    db1, db2 = to_dev(b1, "bf16"), to_dev(b2, "bf16")
    x = to_dev(inp["hidden"], "bf16")
    offsets = torch.from_numpy((np.arange(wl.E + 1) * rows_per_expert).astype(np.int32)).cuda()
    one1, one2 = torch.ones_like(s1), torch.ones_like(s2)
    y_q = moe.expert_ffn_q8(x, offsets, q1, one1, q2, one2, fc1_bias=db1, fc2_bias=db2,
                            fc1_layout=layout)
    y_b = moe.expert_ffn(x, offsets, q1.to(torch.bfloat16), q2.to(torch.bfloat16), fc1_bias=db1,
                         fc2_bias=db2, fc1_layout=layout)
    torch.cuda.synchronize()
    assert torch.equal(_bits(y_q), _bits(y_b))
    y = moe.expert_ffn_q8(x, offsets, q1, s1, q2, s2, fc1_bias=db1, fc2_bias=db2, fc1_layout=layout)
    torch.cuda.synchronize()
    xv = inp.values("hidden")
    ref = np.zeros((wl.T, wl.H))
    for e in range(wl.E):
        a, b = rows_per_expert * e, rows_per_expert * (e + 1)
        ref[a:b] = O.expert_ffn(xv[a:b], O.dequantize_rows(host[0][e], host[1][e]),
                                O.dequantize_rows(host[2][e], host[3][e]), layout,
                                O.STANDARD_SWIGLU, bf16_bits_to_f32(b1[e]), bf16_bits_to_f32(b2[e]))
    atol, rtol = tol("bf16", ref)
    assert_close(from_dev(y), ref, atol, rtol, f"int8 expert FFN {layout}")


def test_full_decode_q8():
    """decode_bf16 (T=4, H=2816, E=128, k=8, I=704) with int8 experts: every output row
    against the oracle on the dequantized weights."""
    from synth import WORKLOADS
    wl = WORKLOADS["decode_bf16"]
    inp = make_inputs(wl, weights=False)
    dev = device_inputs(inp)
    host, (q1, s1, q2, s2) = _q8_dev(wl)
    out = moe.forward_q8(dev["hidden"], dev["router_w"], q1, s1, q2, s2, wl.k)
    r = run_route(dev, wl)
    torch.cuda.synchronize()
    L, idx = check_routing(inp, r)
    ref = _q8_oracle(inp, wl, host, idx)
    atol, rtol = tol(wl.dtype, ref)
    assert_close(from_dev(out), ref, atol, rtol, "decode_bf16 int8 experts")


@pytest.mark.parametrize("T", [4, 9])
def test_forward_q8_with_pre_norm(T):
    """forward_q8(x, norm_weight): bit-equal to rmsnorm then forward_q8 (the same
    kernels after the norm), and the oracle's layer on the oracle's norm of x."""
    from synth import make_pre_norm_inputs
    wl = W("q8_norm", T=T, H=512, E=16, k=4, I=128)
    inp = make_inputs(wl, weights=False)
    dev = device_inputs(inp)
    host, (q1, s1, q2, s2) = _q8_dev(wl)
    x, w = make_pre_norm_inputs(wl)
    dx, dw = to_dev(x, "bf16"), to_dev(w, "bf16")
    eps = float(np.float32(1e-5))
    fused = moe.forward_q8(dx, dev["router_w"], q1, s1, q2, s2, wl.k, norm_weight=dw, norm_eps=eps)
    xn = moe.rmsnorm(dx, dw, eps)
    staged = moe.forward_q8(xn, dev["router_w"], q1, s1, q2, s2, wl.k)
    r = moe.route(xn, dev["router_w"], wl.k)
    torch.cuda.synchronize()
    assert torch.equal(_bits(fused), _bits(staged))
    xn_ref = O.pre_ffn_norm(bf16_bits_to_f32(x), bf16_bits_to_f32(w), eps, "bf16")
    L = O.router_logits(xn_ref, inp.values("router_w"), inp["router_bias"])
    gidx = from_dev(r["idx"]).astype(np.int64)
    idx, _ = match_routing(L, gidx, wl.k)
    np.testing.assert_array_equal(gidx, idx)
    q1h, s1h, q2h, s2h = host
    ref = O.moe_forward(xn_ref, inp.values("router_w"), inp["router_bias"],
                        lambda e: O.dequantize_rows(q1h[e], s1h[e]),
                        lambda e: O.dequantize_rows(q2h[e], s2h[e]), wl.k, wl.normalize,
                        wl.fc1_layout, idx=idx)["out"]
    atol, rtol = tol("bf16", ref)
    assert_close(from_dev(fused), ref, atol, rtol, f"int8 experts with pre-FFN norm, T={T}")


def test_q8_refuses_sizes_outside_the_decode_ffn():
    wl = W("q8_big", T=2048, H=128, E=8, k=2, I=64)      # 512 rows per expert
    inp = make_inputs(wl, weights=False)
    dev = device_inputs(inp)
    _, (q1, s1, q2, s2) = _q8_dev(wl)
    with pytest.raises(moe.MoEError, match="UNSUPPORTED"):
        moe.forward_q8(dev["hidden"], dev["router_w"], q1, s1, q2, s2, wl.k)


def test_combine_matches_oracle():
    wl = W("comb", T=77, H=136, E=6, k=3, dtype="f32")
    inp = make_inputs(wl)
    L = O.router_logits(inp.values("hidden"), inp.values("router_w"))
    idx = O.select_topk(L, 3)
    w = O.routing_weights(L, idx, 1)
    _, _, _, dst = O.stable_permutation(idx, 6)
    y = np.random.default_rng(5).standard_normal((77 * 3, 136)).astype(np.float32)
    got = moe.combine(torch.from_numpy(y).cuda(), torch.from_numpy(dst).cuda(),
                      torch.from_numpy(w.astype(np.float32)).cuda(), 77, 3)
    ref = O.combine(y, dst, w.astype(np.float32), 77, 3)
    assert_close(from_dev(got), ref, 1e-6, 1e-5, "combine")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_convert_chunked_to_interleaved_bitexact(dtype):
    wl = W("conv", E=5, I=96, H=64, dtype=dtype)
    inp = make_inputs(wl)
    src = inp["fc1"]
    got = moe.convert_chunked_to_interleaved(to_dev(src, dtype)).cpu()
    got = got.view(torch.int16).numpy().view(np.uint16) if dtype == "bf16" else got.numpy()
    np.testing.assert_array_equal(got, O.chunked_to_interleaved(src))


def test_forward_with_device_converted_weights_is_bitwise_equal():
    wl = W("conv_fwd", T=200, H=128, E=8, k=2, I=128, fc1_layout="chunked")
    inp = make_inputs(wl)
    dev = device_inputs(inp)
    fc1_dev = moe.convert_chunked_to_interleaved(dev["fc1"])
    fc1_host = to_dev(O.chunked_to_interleaved(inp["fc1"]), "bf16")
    a = moe.forward(dev["hidden"], dev["router_w"], fc1_dev, dev["fc2"], 2)
    b = moe.forward(dev["hidden"], dev["router_w"], fc1_host, dev["fc2"], 2)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    # and the layer on chunked weights equals the oracle's chunked reading
    r = run_route(dev, wl)
    torch.cuda.synchronize()
    L, idx = check_routing(inp, r)
    ref = oracle_forward(inp, idx)["out"]
    assert_close(from_dev(a), ref, 1e-2, 2e-2, "converted forward")


def test_forward_is_deterministic():
    wl = W("det", T=300, H=256, E=16, k=4, I=192)
    dev = device_inputs(make_inputs(wl))
    a = moe.forward(dev["hidden"], dev["router_w"], dev["fc1"], dev["fc2"], 4)
    b = moe.forward(dev["hidden"], dev["router_w"], dev["fc1"], dev["fc2"], 4)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_shared_workspace_across_paths_and_repeated_calls():
    """One zero-filled workspace reused by calls of every bf16 path, in an order that
    makes each path start from what the others left behind (the one-launch decode
    relies on the counters being left at zero): every output equals the output of a
    call on a fresh workspace, bit for bit, and the error word stays clear."""
    cases = [W("ws_decode", T=4, H=256, E=64, k=4, I=128),      # one launch
             W("ws_batched", T=100, H=256, E=64, k=4, I=128),    # tensor-core router + decode FFN
             W("ws_small", T=100, H=256, E=16, k=4, I=128),      # one-CTA router + decode FFN
             W("ws_prefill", T=1100, H=256, E=64, k=4, I=128)]   # tensor-core router + CTA pairs
    devs = [device_inputs(make_inputs(wl)) for wl in cases]
    fresh = [moe.forward(d["hidden"], d["router_w"], d["fc1"], d["fc2"], wl.k)
             for wl, d in zip(cases, devs)]
    need = max(moe.workspace_size(wl.T, wl.H, wl.E, wl.k, wl.I, torch.bfloat16) for wl in cases)
    ws = moe.alloc_workspace(need, torch.device("cuda"))
    for i in [0, 0, 1, 0, 2, 0, 3, 0, 1, 3, 2, 0, 0]:
        wl, d = cases[i], devs[i]
        got = moe.forward(d["hidden"], d["router_w"], d["fc1"], d["fc2"], wl.k, workspace=ws)
        st, bits = moe.get_error(moe.workspace_error_word(ws))
        assert st == 0 and bits == 0, (wl.name, bits)
        assert torch.equal(got.view(torch.int16), fresh[i].view(torch.int16)), wl.name


def test_exact_tie_goes_to_lower_index():
    wl = W("tie", T=50, H=128, E=8, k=2)
    inp = make_inputs(wl)
    rw = inp["router_w"].copy()
    rw[6] = rw[1]                       # experts 1 and 6 tie exactly for every token
    r = moe.route(to_dev(inp["hidden"], "bf16"), to_dev(rw, "bf16"), 2)
    idx = from_dev(r["idx"])
    near = from_dev(r["near_tie"])
    for t in range(50):
        row = list(idx[t])
        if 6 in row:
            assert 1 in row and row.index(1) < row.index(6)
            assert near[t] & 2            # the two tied experts are adjacent chosen slots
        elif 1 in row:
            assert near[t] & 1            # expert 6 ties the k-th choice at the boundary


def test_zero_tokens_is_a_noop():
    wl = W("empty", T=0)
    H, E, I = 128, 8, 64
    hidden = torch.empty((0, H), dtype=torch.bfloat16, device="cuda")
    rw = torch.zeros((E, H), dtype=torch.bfloat16, device="cuda")
    fc1 = torch.zeros((E, 2 * I, H), dtype=torch.bfloat16, device="cuda")
    fc2 = torch.zeros((E, H, I), dtype=torch.bfloat16, device="cuda")
    out = moe.forward(hidden, rw, fc1, fc2, 2)
    assert out.shape == (0, H)
    del wl


def test_invalid_arguments_are_rejected():
    H, E, I = 128, 8, 64
    hidden = torch.zeros((4, H), dtype=torch.bfloat16, device="cuda")
    rw = torch.zeros((E, H), dtype=torch.bfloat16, device="cuda")
    fc1 = torch.zeros((E, 2 * I, H), dtype=torch.bfloat16, device="cuda")
    fc2 = torch.zeros((E, H, I), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError, match="INVALID_ARG"):
        moe.forward(hidden, rw, fc1, fc2, 9)                       # k > E
    with pytest.raises(moe.MoEError, match="INVALID_ARG"):
        moe.forward(hidden, rw, fc1, fc2, 2, swiglu=(float("nan"), 1.0, 7.0))   # alpha
    with pytest.raises(moe.MoEError, match="INVALID_ARG"):
        moe.forward(hidden, rw, fc1, fc2, 2, swiglu=(1.702, 1.0, -1.0))         # limit
    bad = torch.zeros((4 * H + 8,), dtype=torch.bfloat16, device="cuda")[1:1 + 4 * H].view(4, H)
    with pytest.raises(moe.MoEError, match="INVALID_ARG"):
        moe.forward(bad, rw, fc1, fc2, 2)                          # misaligned hidden
    # bf16 sizes without a tensor-core tiling are refused, not computed elsewhere
    h2 = torch.zeros((4, 72), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError, match="UNSUPPORTED"):
        moe.forward(h2, torch.zeros((E, 72), dtype=torch.bfloat16, device="cuda"),
                    torch.zeros((E, 2 * I, 72), dtype=torch.bfloat16, device="cuda"),
                    torch.zeros((E, 72, I), dtype=torch.bfloat16, device="cuda"), 2)


def test_routing_barrier_timeout_is_reported_and_the_next_call_is_clean():
    """Device-side failure detection without a fault: a test-only setting makes the
    one-launch path's routing grid barrier wait for an arrival that never comes, with a
    1 ms limit.  Every block gives up before any bulk copy or MMA, winds down and reports
    MOE_DEVERR_TIMEOUT; the context stays usable, and the next calls -- on the same
    workspace and on a fresh one -- are bit for bit the normal result."""
    from mixture_experts_ffn_15_b200 import _abi
    lib = _abi.load()
    wl = W("timeout", T=4, H=256, E=64, k=4, I=128)
    assert lib.moe_forward_path(wl.T, wl.H, wl.E, wl.k, wl.I, _abi.MOE_BF16) & 32
    dev = device_inputs(make_inputs(wl))
    args = (dev["hidden"], dev["router_w"], dev["fc1"], dev["fc2"], wl.k)
    ref = moe.forward(*args)
    need = moe.workspace_size(wl.T, wl.H, wl.E, wl.k, wl.I, torch.bfloat16)
    ws = moe.alloc_workspace(need, torch.device("cuda"))
    lib.moe_debug_arm_route_barrier_timeout()
    moe.forward(*args, workspace=ws)
    st, bits = moe.get_error(moe.workspace_error_word(ws))
    assert st == _abi.MOE_ERR_TIMEOUT and bits & _abi.MOE_DEVERR_TIMEOUT, (st, bits)
    again = moe.forward(*args, workspace=ws)          # the setting was one-shot
    st, bits = moe.get_error(moe.workspace_error_word(ws))
    assert st == _abi.MOE_OK and bits == 0
    assert torch.equal(again.view(torch.int16), ref.view(torch.int16))
    fresh = moe.forward(*args)
    torch.cuda.synchronize()
    assert torch.equal(fresh.view(torch.int16), ref.view(torch.int16))


def test_bad_expert_ids_are_reported_and_skipped():
    E, T, k = 8, 40, 2
    idx = np.stack([np.arange(T) % E, (np.arange(T) + 3) % E], axis=1).astype(np.int32)
    idx[5, 1] = E          # out of range
    idx[9, 0] = -2         # out of range
    p = moe.permute(torch.from_numpy(idx).cuda(), E)
    st, bits = moe.get_error(p["err_word"])
    assert st == moe._abi.MOE_ERR_DEVICE and bits & moe._abi.MOE_DEVERR_BAD_EXPERT
    good = idx.copy()
    mask = (good < 0) | (good >= E)
    counts = np.bincount(good[~mask], minlength=E)
    np.testing.assert_array_equal(from_dev(p["counts"]), counts)
    dst = from_dev(p["perm_dst"]).reshape(T, k)
    assert dst[5, 1] == -1 and dst[9, 0] == -1


# ------------------------------------------------------------------ full-size workloads

FULL = ["tiny_fp32", "decode_bf16", "batched_decode_bf16", "prefill_bf16", "long_prefill_bf16"]


@pytest.mark.parametrize("name", FULL)
def test_full_workload(name):
    from synth import WORKLOADS, outlier_rows
    wl = WORKLOADS[name]
    inp = make_inputs(wl)
    dev = device_inputs(inp)
    fc1 = dev["fc1"]
    out = moe.forward(dev["hidden"], dev["router_w"], fc1, dev["fc2"], wl.k,
                      normalize=bool(wl.normalize), router_bias=dev["router_bias"],
                      fc1_layout=wl.fc1_layout)
    if wl.fc1_layout == "chunked":
        # the chunked weights read in place equal the layer on converted weights
        conv = moe.forward(dev["hidden"], dev["router_w"], moe.convert_chunked_to_interleaved(fc1),
                           dev["fc2"], wl.k, normalize=bool(wl.normalize),
                           router_bias=dev["router_bias"])
        assert torch.equal(out.view(torch.int16), conv.view(torch.int16))
        del conv
    r = run_route(dev, wl)
    torch.cuda.synchronize()
    L, idx = check_routing(inp, r)
    # counts and permutation over all tokens, bit-exact
    p = moe.permute(r["idx"], wl.E)
    counts, offsets, src, dst = O.stable_permutation(idx, wl.E)
    np.testing.assert_array_equal(from_dev(p["offsets"]), offsets)
    np.testing.assert_array_equal(from_dev(p["perm_src"]), src)
    np.testing.assert_array_equal(from_dev(p["perm_dst"]), dst)
    # values: every token when the oracle is quick, else a seeded sample that holds
    # the outlier rows and tokens of the least and most loaded experts
    tokens = None
    scaled = outlier_rows(wl, wl.seed)
    if wl.T > 256:
        tokens = sample_tokens(wl.T, idx, wl.E, n=192, must=scaled[:64])
    ref = oracle_forward(inp, idx, tokens=tokens)["out"]
    got = from_dev(out) if tokens is None else from_dev(out[torch.from_numpy(tokens).cuda()])
    atol, rtol = tol(wl.dtype, ref)
    # the stated tolerance on every row; the rows the generator scaled x8 (long
    # prefill) also get the oracle's bound of storing act and y_perm in bf16
    extra = None
    if scaled.size and wl.dtype == "bf16":
        extra = scaled_row_storage_bound(inp, idx, np.arange(wl.T) if tokens is None else tokens,
                                         scaled)
    assert_close(got, ref, atol, rtol, f"{name} output", extra=extra)
