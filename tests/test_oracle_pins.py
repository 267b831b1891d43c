"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here compares the oracle with itself: each pin is a hand-derived value
(tests/golden/micro_cases.txt), a closed form, an invariant, or an independent
formulation through a different library routine (a stable sort, bincount,
reshape/transpose, scipy's softmax).  The mutation tests at the end plant a
plausible mistake in the oracle and check that some pin catches it.
"""
import math

import numpy as np
import pytest
from scipy.special import softmax as sp_softmax

from golden_io import load_cases, shaped
from oracle import moe_oracle as O
from synth import WORKLOADS, Workload, make_inputs, round_to_bf16_bits, bf16_bits_to_f32

CASES = load_cases()


def small(T=24, H=32, E=6, k=2, I=16, dtype="f32", seed=3, bias=None, layout="interleaved"):
    wl = Workload("pin", T=T, H=H, E=E, k=k, I=I, dtype=dtype, router_bias_std=bias,
                  fc1_layout=layout, seed=seed)
    return make_inputs(wl)


def fwd(inp, k=None, normalize=1, layout="interleaved", **kw):
    wl = inp.wl
    return O.moe_forward(inp.values("hidden"), inp.values("router_w"), inp["router_bias"],
                         inp.values("fc1"), inp.values("fc2"), wl.k if k is None else k,
                         normalize, layout, **kw)


# ------------------------------------------------------------------ golden cases

def check_golden_values():
    for name in ("single_expert", "normalize_off_two_experts", "chunked_gate_first"):
        c = CASES[name]
        s = shaped(c)
        r = O.moe_forward(s["hidden"], s["router_w"], None, s["fc1"], s["fc2"], c["k"],
                          c["normalize"], s["layout"])
        np.testing.assert_array_equal(r["idx"].ravel(), c["idx"].astype(np.int32))
        np.testing.assert_allclose(r["w"].ravel(), c["w"], rtol=1e-14, atol=0)
        np.testing.assert_allclose(r["out"].ravel(), c["out"], rtol=1e-14, atol=1e-15)


def check_golden_routing():
    c = CASES["routing_rational"]
    s = shaped(c)
    L = O.router_logits(s["hidden"], s["router_w"])
    idx = O.select_topk(L, c["k"])
    np.testing.assert_array_equal(idx.ravel(), c["idx"])
    np.testing.assert_allclose(O.routing_weights(L, idx, 1).ravel(), c["w"], rtol=1e-14)
    np.testing.assert_allclose(O.routing_weights(L, idx, 0).ravel(), c["w_normalize_off"],
                               rtol=1e-14)
    c = CASES["exact_tie"]
    s = shaped(c)
    L = O.router_logits(s["hidden"], s["router_w"])
    np.testing.assert_array_equal(O.select_topk(L, 1).ravel(), c["idx"])
    np.testing.assert_array_equal(O.select_topk(L, 3).ravel(), c["idx_k3"])


def test_golden_values():
    check_golden_values()


def test_golden_routing():
    check_golden_routing()


# --------------------------------------------------------------------- routing pins

def check_topk_brute_force(seed=5):
    inp = small(T=40, E=12, k=4, seed=seed)
    L = O.router_logits(inp.values("hidden"), inp.values("router_w"))
    L32 = L.astype(np.float32)
    idx = O.select_topk(L, 4)
    for t in range(L.shape[0]):
        ref = sorted(range(12), key=lambda e: (-float(L32[t, e]), e))[:4]
        assert list(idx[t]) == ref


def test_topk_matches_full_sort():
    check_topk_brute_force()


def test_topk_duplicate_router_rows_pick_lower_index():
    inp = small(T=16, E=8, k=3, seed=11)
    rw = inp.values("router_w").copy()
    rw[5] = rw[2]          # experts 2 and 5 now always tie exactly
    L = O.router_logits(inp.values("hidden"), rw)
    idx = O.select_topk(L, 3)
    for t in range(16):
        row = list(idx[t])
        if 5 in row:
            assert 2 in row and row.index(2) < row.index(5)


def test_k_equals_e_selects_all_in_sorted_order():
    inp = small(T=10, E=5, k=5)
    L = O.router_logits(inp.values("hidden"), inp.values("router_w"))
    idx = O.select_topk(L, 5)
    for t in range(10):
        assert sorted(idx[t]) == list(range(5))
        assert np.all(np.diff(L[t, idx[t]].astype(np.float32)) <= 0)


def check_weights_sum_to_one():
    inp = small(T=64, E=8, k=3, bias=0.5)
    L = O.router_logits(inp.values("hidden"), inp.values("router_w"), inp["router_bias"])
    w = O.routing_weights(L, O.select_topk(L, 3), 1)
    assert np.max(np.abs(w.sum(axis=1) - 1.0)) <= 1e-12


def test_weights_sum_to_one():
    check_weights_sum_to_one()


def test_normalized_weights_equal_softmax_over_chosen():
    # softmax over all, keep k, renormalise == softmax over the chosen logits alone
    inp = small(T=32, E=9, k=4)
    L = O.router_logits(inp.values("hidden"), inp.values("router_w"))
    idx = O.select_topk(L, 4)
    w = O.routing_weights(L, idx, 1)
    ref = sp_softmax(np.take_along_axis(L, idx.astype(np.int64), 1), axis=1)
    np.testing.assert_allclose(w, ref, rtol=1e-13)


def test_unnormalized_weights_are_full_softmax():
    inp = small(T=32, E=9, k=4)
    L = O.router_logits(inp.values("hidden"), inp.values("router_w"))
    idx = O.select_topk(L, 4)
    w = O.routing_weights(L, idx, 0)
    ref = np.take_along_axis(sp_softmax(L, axis=1), idx.astype(np.int64), 1)
    np.testing.assert_allclose(w, ref, rtol=1e-13)
    assert np.all(w.sum(axis=1) < 1.0)


def test_bias_is_added_before_selection():
    inp = small(T=8, E=6, k=1)
    bias = np.zeros(6, dtype=np.float32)
    bias[4] = 1e3            # expert 4 must win every token
    L = O.router_logits(inp.values("hidden"), inp.values("router_w"), bias)
    assert np.all(O.select_topk(L, 1) == 4)


def test_near_tie_flags_and_alternatives():
    # a gap of 4e-6 at the k/k+1 boundary is ambiguous; 1e-3 is not
    L = np.array([[3.0, 1.0, 1.0 - 4e-6, -2.0], [3.0, 1.0, 0.999, -2.0]])
    f = O.near_tie_flags(L, 2)
    assert f[0] & O.TIE_BOUNDARY and not f[1] & O.TIE_BOUNDARY
    alts = O.valid_selections(L[0], 2)
    assert alts[0] == (0, 1) and (0, 2) in alts and len(alts) == 2
    assert O.valid_selections(L[1], 2) == [(0, 1)]
    Lw = np.array([[2.0, 2.0 - 3e-6, 0.0]])
    assert O.near_tie_flags(Lw, 2)[0] == O.TIE_WITHIN


# ------------------------------------------------------------- counts / permutation

def test_counts_sum_and_match_bincount():
    inp = small(T=50, E=7, k=3)
    L = O.router_logits(inp.values("hidden"), inp.values("router_w"))
    idx = O.select_topk(L, 3)
    c = O.expert_counts(idx, 7)
    assert c.sum() == 50 * 3
    np.testing.assert_array_equal(c, np.bincount(idx.ravel(), minlength=7))


def check_permutation(seed=7):
    inp = small(T=50, E=7, k=3, seed=seed)
    L = O.router_logits(inp.values("hidden"), inp.values("router_w"))
    idx = O.select_topk(L, 3)
    counts, offsets, src, dst = O.stable_permutation(idx, 7)
    n = 150
    # independent formulation: a stable argsort of the flat expert ids
    order = np.argsort(idx.ravel(), kind="stable")
    np.testing.assert_array_equal(src, order // 3)
    ref_dst = np.empty(n, dtype=np.int64)
    ref_dst[order] = np.arange(n)
    np.testing.assert_array_equal(dst, ref_dst)
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(idx.ravel(), minlength=7))]))
    assert sorted(dst.tolist()) == list(range(n))              # bijection
    for t in range(50):
        for j in range(3):
            r = dst[t * 3 + j]
            assert src[r] == t and offsets[idx[t, j]] <= r < offsets[idx[t, j] + 1]
    for e in range(7):
        seg = src[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)                          # stable: tokens ascending


def test_permutation_properties():
    check_permutation()


def test_exclusive_offsets_by_hand():
    # expert blocks start where the earlier experts' rows end; an empty expert's block
    # is empty and starts where the next one does
    np.testing.assert_array_equal(O.exclusive_offsets(np.array([3, 0, 2, 1])), [0, 3, 3, 5, 6])
    np.testing.assert_array_equal(O.exclusive_offsets(np.array([0, 0])), [0, 0, 0])
    np.testing.assert_array_equal(O.exclusive_offsets(np.array([], dtype=np.int64)), [0])


def test_fc1_gate_up_row_orders_by_hand():
    # rows labelled by their index: interleaved fc1 puts gate_i in row 2i and up_i in
    # row 2i + 1; the chunked (Hugging Face) layout puts gate_i in row i, up_i in I + i
    I, H = 3, 2
    fc1 = np.repeat(np.arange(2 * I, dtype=np.float64)[:, None], H, axis=1)
    g, u = O.fc1_gate_up(fc1, "interleaved")
    np.testing.assert_array_equal(g[:, 0], [0, 2, 4])
    np.testing.assert_array_equal(u[:, 0], [1, 3, 5])
    g, u = O.fc1_gate_up(fc1, "chunked")
    np.testing.assert_array_equal(g[:, 0], [0, 1, 2])
    np.testing.assert_array_equal(u[:, 0], [3, 4, 5])
    with pytest.raises(ValueError):
        O.fc1_gate_up(fc1, "gate_up_pairs")


def test_combine_of_permuted_rows_equals_layer():
    inp = small(T=20, E=5, k=2)
    r = fwd(inp)
    counts, offsets, src, dst = O.stable_permutation(r["idx"], 5)
    x_perm = O.gather_rows(inp.values("hidden"), src)
    y_perm = np.zeros((x_perm.shape[0], inp.wl.H))
    for e in range(5):
        a, b = offsets[e], offsets[e + 1]
        if b > a:
            y_perm[a:b] = O.expert_ffn(x_perm[a:b], inp.values("fc1")[e], inp.values("fc2")[e])
    out = O.combine(y_perm, dst, r["w"], 20, 2)
    np.testing.assert_allclose(out, r["out"], rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------ layout / values

def check_chunked_equals_interleaved():
    inp = small(T=12, E=4, k=2, I=8, layout="chunked")
    chunked = inp.values("fc1")
    E, two_i, H = chunked.shape
    # the page's recipe: Reshape [E,2,I,H] -> Transpose [E,I,2,H] -> Reshape [E,2I,H]
    recipe = chunked.reshape(E, 2, two_i // 2, H).transpose(0, 2, 1, 3).reshape(E, two_i, H)
    conv = O.chunked_to_interleaved(chunked)
    np.testing.assert_array_equal(conv, recipe)
    a = fwd(inp, layout="chunked")["out"]
    b = O.moe_forward(inp.values("hidden"), inp.values("router_w"), None, conv,
                      inp.values("fc2"), 2, 1, "interleaved")["out"]
    np.testing.assert_array_equal(a, b)


def test_chunked_equals_interleaved():
    check_chunked_equals_interleaved()


def check_dense_masked_equals_sparse(normalize=1):
    inp = small(T=8, E=5, k=2, bias=0.3)
    a = fwd(inp, normalize=normalize)["out"]
    b = O.moe_dense_masked(inp.values("hidden"), inp.values("router_w"), inp["router_bias"],
                           inp.values("fc1"), inp.values("fc2"), 2, normalize)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("normalize", [0, 1])
def test_dense_masked_equals_sparse(normalize):
    check_dense_masked_equals_sparse(normalize)


def test_k_equals_e_is_softmax_weighted_sum_over_all_experts():
    inp = small(T=6, E=4, k=4)
    r = fwd(inp, k=4)
    L = O.router_logits(inp.values("hidden"), inp.values("router_w"))
    p = sp_softmax(L, axis=1)
    ref = sum(p[:, e:e + 1] * O.expert_ffn(inp.values("hidden"), inp.values("fc1")[e],
                                           inp.values("fc2")[e]) for e in range(4))
    np.testing.assert_allclose(r["out"], ref, rtol=1e-12, atol=1e-14)


def test_zero_up_rows_give_zero():
    inp = small()
    fc1 = inp.values("fc1").copy()
    fc1[:, 1::2, :] = 0.0
    out = O.moe_forward(inp.values("hidden"), inp.values("router_w"), None, fc1,
                        inp.values("fc2"), 2, 1)["out"]
    assert np.all(out == 0.0)


def test_zero_gate_rows_give_zero():
    inp = small()
    fc1 = inp.values("fc1").copy()
    fc1[:, 0::2, :] = 0.0          # silu(0) = 0
    out = O.moe_forward(inp.values("hidden"), inp.values("router_w"), None, fc1,
                        inp.values("fc2"), 2, 1)["out"]
    assert np.all(out == 0.0)


def check_expert_ffn_scalar_loops():
    # brute force with scalar loops on a tiny expert (orientation of every operand)
    rng = np.random.default_rng(1)
    H, I, n = 3, 2, 2
    x = rng.standard_normal((n, H))
    fc1 = rng.standard_normal((2 * I, H))
    fc2 = rng.standard_normal((H, I))
    y = O.expert_ffn(x, fc1, fc2)
    for r in range(n):
        for h in range(H):
            acc = 0.0
            for i in range(I):
                g = sum(x[r, c] * fc1[2 * i, c] for c in range(H))
                u = sum(x[r, c] * fc1[2 * i + 1, c] for c in range(H))
                acc += fc2[h, i] * (g * (1.0 / (1.0 + math.exp(-g)))) * u
            assert abs(acc - y[r, h]) <= 1e-12 * max(1.0, abs(acc))


def test_expert_ffn_scalar_loops():
    check_expert_ffn_scalar_loops()


def test_sparse_evaluation_on_token_subset_matches_full():
    inp = small(T=30, E=6, k=3)
    full = fwd(inp)["out"]
    sub = fwd(inp, tokens=[0, 7, 29])["out"]
    # the BLAS may block a 3-row product differently from a 30-row one: rounding only
    np.testing.assert_allclose(sub, full[[0, 7, 29]], rtol=1e-13, atol=1e-15)


# ------------------------------------------------------------------- pre-FFN RMSNorm

def check_round_to_dtype():
    # float32 values are exact in float64: rounding them to bf16 from float64 must give
    # the generator's float32 -> bf16 round-to-nearest-even, bit for bit
    rng = np.random.default_rng(11)
    v = (rng.standard_normal(4000) * np.exp(rng.uniform(-20, 20, 4000))).astype(np.float32)
    got = O.round_to_dtype(v.astype(np.float64), "bf16")
    np.testing.assert_array_equal(got, bf16_bits_to_f32(round_to_bf16_bits(v)).astype(np.float64))
    # midpoints go to the even neighbour; anything above a midpoint goes up
    y = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 1 + 2 ** -8 + 2 ** -40,
                  2 - 2 ** -9, 0.375 + 2 ** -11])
    np.testing.assert_array_equal(O.round_to_dtype(y, "bf16"),
                                  [1.0, 1 + 2 ** -6, -1.0, 1 + 2 ** -7, 2.0, 0.375])
    np.testing.assert_array_equal(O.round_to_dtype(np.array([1 + 2 ** -24, 1 + 3 * 2 ** -24]), "f32"),
                                  [1.0, 1 + 2 ** -22])
    # a negative zero stays negative (the norm of a -0 input is -0)
    assert np.signbit(O.round_to_dtype(np.array([-0.0]), "bf16"))[0]
    assert np.signbit(O.pre_ffn_norm(np.array([[-0.0, 1.0]]), np.ones(2), 0.0, "bf16"))[0, 0]


def check_rms_norm_closed_forms():
    # a worked example: x = (3, 4), mean of squares 12.5
    got = O.rms_norm(np.array([[3.0, 4.0]]), np.array([2.0, 0.5]), 0.0)
    np.testing.assert_allclose(got, [[6 / np.sqrt(12.5), 2 / np.sqrt(12.5)]], rtol=1e-15)
    # a constant row c: every output is c w / sqrt(c^2 + eps); with eps = c^2, w / sqrt(2)
    w = np.linspace(0.5, 1.5, 16)
    for c, eps in ((3.0, 0.0), (-0.25, 1e-6), (2.0, 4.0)):
        got = O.rms_norm(np.full((1, 16), c), w, eps)
        np.testing.assert_allclose(got[0], c * w / np.sqrt(c * c + eps), rtol=1e-14)
    np.testing.assert_allclose(O.rms_norm(np.full((1, 4), 2.0), np.ones(4), 4.0), 2 ** -0.5, rtol=1e-15)
    # with unit weight and no eps every row has mean square one, whatever its scale,
    # and the weight multiplies column by column
    rng = np.random.default_rng(12)
    x = rng.standard_normal((5, 64)) * np.array([[0.01], [1], [7], [300], [1e-3]])
    y1 = O.rms_norm(x, np.ones(64), 0.0)
    np.testing.assert_allclose(np.mean(y1 * y1, axis=1), 1.0, rtol=1e-13)
    np.testing.assert_allclose(O.rms_norm(9.0 * x, np.ones(64), 0.0), y1, rtol=1e-13)
    wv = rng.uniform(0.5, 2.0, 64)
    np.testing.assert_allclose(O.rms_norm(x, wv, 0.0), y1 * wv, rtol=1e-14)
    # a row of zeros stays zero
    np.testing.assert_array_equal(O.rms_norm(np.zeros((1, 8)), np.ones(8), 1e-6), 0.0)


def check_pre_ffn_norm_rounds_once():
    # the layer's input is the norm rounded to bf16 once: inputs whose norm is exact in
    # bf16 come through unchanged; otherwise it is the nearest bf16 value
    x = np.full((1, 4), 2.0)                       # mean square 4: r = 1/2 exactly
    w = np.array([1.0, 1.5, 0.75, 3.0])
    np.testing.assert_array_equal(O.pre_ffn_norm(x, w, 0.0, "bf16"), [w])
    x = np.full((1, 4), 3.0)                       # x r = 1: y = w = 1/3 -> 0.333984375 in bf16
    np.testing.assert_array_equal(O.pre_ffn_norm(x, np.full(4, 1 / 3), 0.0, "bf16"),
                                  np.full((1, 4), 0.333984375))
    rng = np.random.default_rng(13)
    x = rng.standard_normal((6, 48)) * 5
    w = rng.uniform(0.8, 1.2, 48)
    y = O.pre_ffn_norm(x, w, 1e-6, "bf16")
    exact = O.rms_norm(x, w, 1e-6)
    m, e = np.frexp(exact)
    np.testing.assert_array_less(np.abs(y - exact), np.ldexp(1.0, e - 8) * 0.5 + 1e-300)
    np.testing.assert_array_equal(O.round_to_dtype(y, "bf16"), y)   # already bf16 values


def check_dequantize_rows():
    # closed forms: unit scales return q itself; scale s multiplies row r only
    q = np.array([[1, -2, 127], [-127, 0, 5]], dtype=np.int8)
    np.testing.assert_array_equal(O.dequantize_rows(q, [1.0, 1.0]), q.astype(np.float64))
    np.testing.assert_array_equal(O.dequantize_rows(q, [0.5, 3.0]),
                                  [[0.5, -1.0, 63.5], [-381.0, 0.0, 15.0]])
    # (2q, s/2) is the same weight; an expert FFN on dequantized rows is the FFN of the
    # float64 weights q * s, and doubling one fc2 row's scale doubles that output column
    rng = np.random.default_rng(21)
    q1 = rng.integers(-63, 64, size=(8, 16)).astype(np.int8)
    s1 = rng.uniform(0.01, 0.02, size=8)
    np.testing.assert_array_equal(O.dequantize_rows(2 * q1.astype(np.int16), s1 / 2),
                                  O.dequantize_rows(q1, s1))
    q2 = rng.integers(-127, 128, size=(16, 4)).astype(np.int8)
    s2 = rng.uniform(0.01, 0.02, size=16)
    x = rng.standard_normal((3, 16))
    y = O.expert_ffn(x, O.dequantize_rows(q1, s1), O.dequantize_rows(q2, s2))
    s2b = s2.copy()
    s2b[5] *= 2
    y2 = O.expert_ffn(x, O.dequantize_rows(q1, s1), O.dequantize_rows(q2, s2b))
    np.testing.assert_allclose(y2[:, 5], 2 * y[:, 5], rtol=1e-14)
    np.testing.assert_array_equal(np.delete(y2, 5, axis=1), np.delete(y, 5, axis=1))


def test_dequantize_rows():
    check_dequantize_rows()


def test_round_to_dtype():
    check_round_to_dtype()


def test_rms_norm_closed_forms():
    check_rms_norm_closed_forms()


def test_pre_ffn_norm_rounds_once():
    check_pre_ffn_norm_rounds_once()


# ----------------------------------------------------------------------- inputs

def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -9,
                     3.0e38], dtype=np.float32)
    bits = round_to_bf16_bits(vals)
    np.testing.assert_array_equal(bits, np.array([0x3F80, 0x3F80, 0x3F82, 0xC020, 0x3F80, 0x7F62],
                                                 dtype=np.uint16))
    np.testing.assert_array_equal(bf16_bits_to_f32(bits[:4]), np.array([1.0, 1.0, 1.0 + 2 ** -6, -2.5],
                                                                        dtype=np.float32))


def test_inputs_are_deterministic_and_seeded():
    wl = Workload("d", T=5, H=16, E=3, k=2, I=8, dtype="bf16")
    a, b = make_inputs(wl), make_inputs(wl)
    for name in ("hidden", "router_w", "fc1", "fc2"):
        np.testing.assert_array_equal(a[name], b[name])
    c = make_inputs(wl, seed=1)
    assert not np.array_equal(a["hidden"], c["hidden"])


def test_batched_decode_workload_is_skewed():
    # the workload asks for some experts with no token and some with more than 40
    wl = WORKLOADS["batched_decode_bf16"]
    inp = make_inputs(wl, weights=False)
    L = O.router_logits(inp.values("hidden"), inp.values("router_w"), inp["router_bias"])
    c = O.expert_counts(O.select_topk(L, wl.k), wl.E)
    assert (c == 0).sum() >= 1 and (c > 40).sum() >= 1


def test_outlier_rows():
    wl = WORKLOADS["long_prefill_bf16"].with_(T=1000, H=64, E=4, k=2, I=64)
    inp = make_inputs(wl, weights=False)
    h = inp.values("hidden")
    big = np.abs(h).max(axis=1) > 6.0
    assert 0 < big.sum() <= 10


# ------------------------------------------------- SwiGLU attributes, expert biases
# "Gemma 4 MoE: re-enable fused com.microsoft::MoE op - #326", "Attribute set":
# activation_alpha (the GPT-OSS "1.702 multiplier"), activation_beta (the "+1 bias
# on the up branch"), swiglu_limit (the clipping); and the op's optional expert
# biases.  Closed forms chosen so that each plausible misplacement changes a value.

ALPHAS = [1.0, 1.702, 0.5]


def check_swiglu_closed_forms():
    # gate = ln(3) / alpha makes sigmoid(alpha * gate) = 3/4 exactly (in real
    # arithmetic): act = (up + beta) * gate * 3/4.  A multiplier outside the sigmoid,
    # a bias on the gate or sigmoid(-x) all change the value.
    for alpha in ALPHAS:
        g = math.log(3.0) / alpha
        for beta in (0.0, 1.0, -0.25):
            for u in (0.0, 1.5, -2.0):
                got = float(O.swiglu(np.array([g]), np.array([u]), alpha, beta, 7.0)[0])
                want = (u + beta) * g * 0.75
                assert abs(got - want) <= 1e-14 * max(1.0, abs(want)), (alpha, beta, u, got, want)
    # a zero gate gives exactly zero whatever the other attributes
    assert np.all(O.swiglu(np.zeros(3), np.array([1.0, -3.0, 9.0]), 1.702, 1.0, 7.0) == 0.0)
    # the standard attributes reduce to silu(gate) * up with silu(x) = x / (1 + e^-x)
    g = np.linspace(-6, 6, 25)
    u = np.cos(g)
    want = np.array([x / (1.0 + math.exp(-x)) * y for x, y in zip(g, u)])
    np.testing.assert_allclose(O.swiglu(g, u, *O.STANDARD_SWIGLU), want, rtol=1e-15, atol=0)


def check_swiglu_limit_saturation():
    L = 7.0
    alpha, beta = O.GPT_OSS_SWIGLU[0], O.GPT_OSS_SWIGLU[1]
    f = lambda g, u: float(O.swiglu(np.array([g]), np.array([u]), alpha, beta, L)[0])
    # gate above the limit saturates at the limit; the up branch saturates on both sides
    assert f(9.0, 0.3) == f(L, 0.3) and f(1e6, -2.0) == f(L, -2.0)
    assert f(1.2, 12.0) == f(1.2, L) and f(1.2, -12.0) == f(1.2, -L)
    # the bias is added after the up branch is clipped: at up = -L, (up' + beta) = -L + beta
    g = math.log(3.0) / alpha
    assert abs(f(g, -20.0) - (-L + beta) * g * 0.75) <= 1e-13
    # the gate is not clipped from below (a large negative gate keeps decaying)
    assert abs(f(-9.0, 1.0)) < abs(f(-L, 1.0))
    # no limit: nothing saturates
    assert O.swiglu(np.array([30.0]), np.array([30.0]), 1.0, 0.0, float("inf"))[0] > 800.0


def check_expert_biases_zero_input():
    # Zero input rows: gate = b_gate, up = b_up, y = fc2 act(b_gate, b_up) + b2.  With
    # b_gate = ln(3)/alpha the activation is (b_up + beta) * b_gate * 3/4 in closed form.
    alpha, beta, L = O.GPT_OSS_SWIGLU
    g = math.log(3.0) / alpha
    H, I = 3, 2
    fc1 = np.full((2 * I, H), 0.37)                 # irrelevant: x = 0
    fc2 = np.array([[1.0, 2.0], [0.0, -1.0], [0.5, 0.25]])
    b1 = np.array([g, 0.5, g, -1.5])                 # interleaved: gate0, up0, gate1, up1
    b2 = np.array([0.1, -0.2, 0.3])
    a = np.array([(0.5 + beta) * g * 0.75, (-1.5 + beta) * g * 0.75])
    want = fc2 @ a + b2
    y = O.expert_ffn(np.zeros((2, H)), fc1, fc2, "interleaved", (alpha, beta, L), b1, b2)
    np.testing.assert_allclose(y, np.stack([want, want]), rtol=1e-14, atol=1e-15)
    # the layer: two experts with equal router logits (zero input) share weight 1/2 each
    fc1s = np.stack([fc1, fc1])
    fc2s = np.stack([fc2, 2.0 * fc2])
    b1s = np.stack([b1, b1])
    b2s = np.stack([b2, -b2])
    want_layer = 0.5 * (fc2 @ a + b2) + 0.5 * (2.0 * fc2 @ a - b2)
    r = O.moe_forward(np.zeros((1, H)), np.ones((2, H)), None, fc1s, fc2s, 2, 1,
                      act=(alpha, beta, L), fc1_bias=b1s, fc2_bias=b2s)
    np.testing.assert_allclose(r["out"][0], want_layer, rtol=1e-14, atol=1e-15)


def check_biased_chunked_equals_interleaved():
    # fc1 and its bias given chunked equal the same interleaved by the page's recipe
    inp = small(T=10, E=4, k=2, layout="chunked")
    E, two_i = inp.values("fc1").shape[:2]
    rng = np.random.default_rng(11)
    b1 = rng.standard_normal((E, two_i))
    b2 = rng.standard_normal((E, inp.wl.H))
    act = O.GPT_OSS_SWIGLU
    a = fwd(inp, layout="chunked", act=act, fc1_bias=b1, fc2_bias=b2)["out"]
    b = O.moe_forward(inp.values("hidden"), inp.values("router_w"), None,
                      O.chunked_to_interleaved(inp.values("fc1")), inp.values("fc2"), 2, 1,
                      "interleaved", act=act, fc1_bias=O.chunked_to_interleaved(b1), fc2_bias=b2)["out"]
    np.testing.assert_array_equal(a, b)
    # and the dense per-expert unroll agrees with the sparse layer
    d = O.moe_dense_masked(inp.values("hidden"), inp.values("router_w"), None,
                           O.chunked_to_interleaved(inp.values("fc1")), inp.values("fc2"), 2, 1,
                           "interleaved", act, O.chunked_to_interleaved(b1), b2)
    np.testing.assert_allclose(b, d, rtol=1e-12, atol=1e-13)


def test_swiglu_closed_forms():
    check_swiglu_closed_forms()


def test_swiglu_limit_saturation():
    check_swiglu_limit_saturation()


def test_expert_biases_zero_input():
    check_expert_biases_zero_input()


def test_biased_chunked_equals_interleaved():
    check_biased_chunked_equals_interleaved()


# ---------------------------------------------------------------- mutation tests

def _mut_drop_sigmoid(g):
    return g


def _mut_swap_gate_up(gate, up, *attrs):
    return O.silu(up) * gate


def _mut_alpha_outside_sigmoid(gate, up, alpha=1.0, beta=0.0, limit=float("inf")):
    return alpha * _real_swiglu(gate, up, 1.0, beta, limit)


def _mut_beta_on_gate(gate, up, alpha=1.0, beta=0.0, limit=float("inf")):
    return _real_swiglu(gate + beta, up, alpha, 0.0, limit)


def _mut_clip_gate_both_sides(gate, up, alpha=1.0, beta=0.0, limit=float("inf")):
    return _real_swiglu(np.clip(gate, -limit, limit), up, alpha, beta, limit)


def _mut_beta_before_clip(gate, up, alpha=1.0, beta=0.0, limit=float("inf")):
    return _real_swiglu(gate, up + beta, alpha, 0.0, limit)


def _mut_fc2_bias_dropped(x_rows, fc1_e, fc2_e, layout="interleaved", act=O.STANDARD_SWIGLU,
                          fc1_bias_e=None, fc2_bias_e=None):
    return _real_expert_ffn(x_rows, fc1_e, fc2_e, layout, act, fc1_bias_e, None)


def _mut_fc1_bias_chunked(x_rows, fc1_e, fc2_e, layout="interleaved", act=O.STANDARD_SWIGLU,
                          fc1_bias_e=None, fc2_bias_e=None):
    if fc1_bias_e is not None and layout == "interleaved":
        b = np.asarray(fc1_bias_e)
        I = b.shape[0] // 2
        fc1_bias_e = np.stack([b[:I], b[I:]], axis=1).ravel()   # read as if chunked
    return _real_expert_ffn(x_rows, fc1_e, fc2_e, layout, act, fc1_bias_e, fc2_bias_e)


def _mut_fc1_chunked_read(fc1_e, layout):
    I = fc1_e.shape[0] // 2
    return fc1_e[:I], fc1_e[I:]


def _mut_ties_to_higher(L, k):
    L32 = np.asarray(L).astype(np.float32)
    out = np.empty((L32.shape[0], k), dtype=np.int32)
    for t in range(L32.shape[0]):
        order = sorted(range(L32.shape[1]), key=lambda e: (-float(L32[t, e]), -e))
        out[t] = order[:k]
    return out


def _mut_no_renormalise(L, idx, normalize):
    p = O.softmax_all(np.asarray(L, dtype=np.float64))
    return np.take_along_axis(p, idx.astype(np.int64), axis=1)


def _mut_unstable_perm(idx, E):
    counts, offsets, src, dst = _real_perm(idx, E)
    T, k = idx.shape
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        src[a:b] = src[a:b][::-1].copy()
    for r, t in enumerate(src):
        for j in range(k):
            if idx[t, j] >= 0 and offsets[idx[t, j]] <= r < offsets[idx[t, j] + 1]:
                dst[t * k + j] = r
    return counts, offsets, src, dst


def _mut_gemma2_offset(x, weight, eps):
    return _real_rms_norm(x, 1.0 + np.asarray(weight, dtype=np.float64), eps)


def _mut_eps_outside_sqrt(x, weight, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / (np.sqrt(np.mean(x * x, axis=1, keepdims=True)) + eps) * weight


def _mut_sum_not_mean(x, weight, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=1, keepdims=True) + eps) * weight


def _mut_round_half_up(y, dtype):
    y = np.asarray(y, dtype=np.float64)
    if dtype == "f32":
        return y.astype(np.float32).astype(np.float64)
    m, e = np.frexp(y)
    return np.ldexp(np.floor(np.ldexp(m, 8) + 0.5), e - 8)


def _mut_round_truncate(y, dtype):
    y = np.asarray(y, dtype=np.float64)
    m, e = np.frexp(y)
    return np.ldexp(np.trunc(np.ldexp(m, 8)), e - 8)


def _mut_scale_per_column(q, scale):
    q = np.asarray(q, dtype=np.float64)
    sc = np.asarray(scale, dtype=np.float64)
    return q * np.resize(sc, q.shape[1])[None, :]


_real_rms_norm = O.rms_norm
_real_perm = O.stable_permutation
_real_swiglu = O.swiglu
_real_expert_ffn = O.expert_ffn

MUTATIONS = [
    ("silu", _mut_drop_sigmoid),
    ("swiglu", _mut_swap_gate_up),
    ("swiglu", _mut_alpha_outside_sigmoid),
    ("swiglu", _mut_beta_on_gate),
    ("swiglu", _mut_clip_gate_both_sides),
    ("swiglu", _mut_beta_before_clip),
    ("expert_ffn", _mut_fc2_bias_dropped),
    ("expert_ffn", _mut_fc1_bias_chunked),
    ("fc1_gate_up", _mut_fc1_chunked_read),
    ("select_topk", _mut_ties_to_higher),
    ("routing_weights", _mut_no_renormalise),
    ("stable_permutation", _mut_unstable_perm),
    ("rms_norm", _mut_gemma2_offset),
    ("rms_norm", _mut_eps_outside_sqrt),
    ("rms_norm", _mut_sum_not_mean),
    ("round_to_dtype", _mut_round_half_up),
    ("round_to_dtype", _mut_round_truncate),
    ("dequantize_rows", _mut_scale_per_column),
]

PIN_CHECKS = [check_golden_values, check_golden_routing, check_topk_brute_force,
              check_weights_sum_to_one, check_permutation, check_chunked_equals_interleaved,
              check_dense_masked_equals_sparse, check_expert_ffn_scalar_loops,
              check_swiglu_closed_forms, check_swiglu_limit_saturation,
              check_expert_biases_zero_input, check_biased_chunked_equals_interleaved,
              check_round_to_dtype, check_rms_norm_closed_forms, check_pre_ffn_norm_rounds_once,
              check_dequantize_rows]


@pytest.mark.parametrize("name,mutant", MUTATIONS, ids=[f"{m[0]}-{m[1].__name__}" for m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, name, mutant):
    monkeypatch.setattr(O, name, mutant)
    caught = 0
    for check in PIN_CHECKS:
        try:
            check()
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin catches a mistake planted in {name}"
