"""CPU oracle for the fused mixture-of-experts FFN layer (com.microsoft::MoE, standard SwiGLU).

TEST INFRASTRUCTURE.  Only the tests, the smoke entry point and the benchmark's
CPU-baseline leg may import this module.  The product path (the CUDA library and
its Python binding) never calls it, and it shares no code with that path.

What it computes is the plain definition of the layer, in float64 with numpy,
following the pages in their order:

* "Gemma 4 MoE: re-enable fused com.microsoft::MoE op - #326" (onnxruntime/mobius
  pull request), description and "Attribute set": activation_type swiglu with
  activation_alpha = 1.0, activation_beta = 0.0, swiglu_limit = inf, i.e. standard
  SwiGLU y = silu(gate) * up; swiglu_fusion = 1 (interleaved gate/up rows);
  normalize_routing_weights = 1; k = top_k.
* same page, "Weight layout": Hugging Face stores experts.gate_up_proj chunked as
  [E, 2*inter, H], the first inter rows gate and the next inter rows up; the
  fused op takes the interleaved layout, made by Reshape -> Transpose -> Reshape.
* same page, "Fallback": the static per-expert unroll computes the same layer one
  expert at a time; `moe_dense_masked` is that reading, used as a brute-force pin.
* same page, "Changes": the fused op is wrapped in CastLike, so the output has the
  input's dtype (the oracle reports float64; callers compare after widening).
* same page, "Attribute set" and description: the op takes activation_alpha,
  activation_beta and swiglu_limit (GPT-OSS: 1.702, 1.0, 7.0 -- the "1.702
  multiplier", the "+1 bias on the up branch" and the clipping); `swiglu` implements
  the family, standard SwiGLU being (1, 0, inf); the op's optional fc1/fc2 expert
  biases are added to the pre-activation gate/up values and to the output.
* "Contributing Gemma 4 support and ONNX export optimizations" (Hugging Face forum),
  "Key Technical Contributions", RMSNorm formulation realignment: Gemma 4's norms are
  Llama-style, the normalised activations multiplied by the weight (not by 1 +
  weight as in Gemma 2); the Rust weight-loader page lists a pre-FFN norm among the
  four norms of each layer.  `rms_norm` is that norm, `pre_ffn_norm` the layer's
  input made from a residual activation by it.
* "Gemma 4 MoE: re-enable fused com.microsoft::MoE op - #326", description: the CUDA
  pull request it cites adds a quantised MoE operator (QMoE); the Rust weight-loader
  page loads 4-bit MLP weights.  Neither gives a format; `dequantize_rows` is the
  reading used here for weight-only int8 experts (see below).
* same forum page, "Key Technical Contributions", ONNX tracing compatibility: inside
  grouped_mm_experts_forward the per-expert token count is a bincount over the
  chosen expert ids, followed by a grouped matmul over experts.

Readings where the pages are silent (each is listed with its reason in the design
notes of the repository):

* router logits are hidden @ router_w^T (+ an optional per-expert bias added before
  selection and softmax); no pre-norm or scale;
* top-k picks the k largest logits in descending order, ties to the lower expert
  index; the selection is taken in float32, the precision of the CUDA kernels'
  logits, so that both sides decide in the same precision;
* normalize_routing_weights = 1 means softmax over all E logits, keep the k chosen
  probabilities, divide by their sum; with 0 the chosen probabilities are kept as is;
* interleaved means row 2i = gate_i and row 2i+1 = up_i (the fc1 bias follows the
  same layout as the fc1 rows);
* SwiGLU attributes: act = (up' + beta) * gate' * sigmoid(alpha * gate') with
  gate' = min(gate, limit) and up' = clip(up, -limit, limit) -- the multiplier acts
  inside the sigmoid, the bias on the up branch after its clipping, and the clipping
  bounds the gate from above only (the pages name the clipping but not its form);
* the stable permutation puts the (token, slot) pairs of expert e in ascending
  token order, experts in ascending order;
* the RMSNorm is y = (x / sqrt(mean(x^2) + eps)) * weight evaluated in float64 and
  rounded once to the storage dtype (round to nearest, ties to even): the pages fix
  the formula, not its precision, and one rounding of the exact value is the plain
  definition; eps is the caller's;
* int8 experts: every weight row r holds int8 values q[r, :] in [-127, 127] and one
  scale s[r]; its weights are q[r, :] * s[r] (symmetric, one scale per output row);
  the layer is the same layer on those weights.

Parity pins for every function here live in tests/test_oracle_pins.py.  No
function in this file is "parity unpinned".
"""

from __future__ import annotations

import itertools
from typing import Callable, Optional, Sequence, Union

import numpy as np

F64 = np.float64
STANDARD_SWIGLU = (1.0, 0.0, float("inf"))   # (activation_alpha, activation_beta, swiglu_limit)
GPT_OSS_SWIGLU = (1.702, 1.0, 7.0)
NEAR_TIE_GAP = 1e-5          # float32 logit gap below which a selection is ambiguous
TIE_BOUNDARY = 1             # flag bit: k-th and (k+1)-th logits within the gap
TIE_WITHIN = 2               # flag bit: two adjacent chosen logits within the gap

ArrayOrGetter = Union[np.ndarray, Callable[[int], np.ndarray]]


def _expert(w: ArrayOrGetter, e: int) -> np.ndarray:
    return (w(e) if callable(w) else w[e]).astype(F64)


# --------------------------------------------------------------------------- routing

def router_logits(hidden, router_w, router_bias=None) -> np.ndarray:
    """L[t, e] = sum_h hidden[t, h] * router_w[e, h] + router_bias[e], float64 [T, E]."""
    L = np.asarray(hidden, dtype=F64) @ np.asarray(router_w, dtype=F64).T
    if router_bias is not None:
        L = L + np.asarray(router_bias, dtype=F64)[None, :]
    return L


def select_topk(L: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest logits per token, descending, ties to the lower index.

    The comparison is made on the float32-rounded logits: the CUDA kernels decide in
    float32, and the decision must be taken in the same precision on both sides.
    """
    L32 = np.asarray(L, dtype=F64).astype(np.float32)
    T, E = L32.shape
    idx = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        # a stable sort on the negated logits keeps equal logits in index order
        order = np.argsort(-L32[t], kind="stable")
        idx[t] = order[:k]
    return idx


def softmax_all(L: np.ndarray) -> np.ndarray:
    """Softmax over the E experts of each token, float64."""
    m = L.max(axis=1, keepdims=True)
    z = np.exp(L - m)
    return z / z.sum(axis=1, keepdims=True)


def routing_weights(L: np.ndarray, idx: np.ndarray, normalize: int) -> np.ndarray:
    """Mixing weights of the chosen experts, float64 [T, k].

    normalize_routing_weights = 1: softmax over all experts, keep the chosen k
    probabilities, divide them by their sum.  0: keep the chosen probabilities.
    """
    p = softmax_all(np.asarray(L, dtype=F64))
    chosen = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    if normalize:
        chosen = chosen / chosen.sum(axis=1, keepdims=True)
    return chosen


def near_tie_flags(L: np.ndarray, k: int, gap: float = NEAR_TIE_GAP) -> np.ndarray:
    """Per-token flags for ambiguous selections, computed on float32 logits.

    TIE_BOUNDARY: the k-th and (k+1)-th largest logits differ by less than `gap`
    (the chosen set may legitimately differ); TIE_WITHIN: two adjacent chosen logits
    differ by less than `gap` (only the slot order may differ).
    """
    L32 = np.asarray(L, dtype=F64).astype(np.float32)
    T, E = L32.shape
    flags = np.zeros(T, dtype=np.int32)
    for t in range(T):
        s = np.sort(L32[t])[::-1]
        if k < E and (s[k - 1] - s[k]) < gap:
            flags[t] |= TIE_BOUNDARY
        if k > 1 and np.any((s[: k - 1] - s[1:k]) < gap):
            flags[t] |= TIE_WITHIN
    return flags


def valid_selections(L_row: np.ndarray, k: int, gap: float = NEAR_TIE_GAP):
    """All k-sets a float32 selection may return when logits within `gap` are tied.

    A set S is valid when no expert outside S beats a member of S by `gap` or more.
    Each set is returned in the canonical slot order (descending float32 logit, ties
    to the lower index).  The oracle's own choice is always the first entry.
    """
    L32 = np.asarray(L_row, dtype=F64).astype(np.float32)
    E = L32.shape[0]
    order = list(np.argsort(-L32, kind="stable"))
    first = tuple(int(e) for e in order[:k])
    if k == E:
        return [first]
    v_k, v_k1 = L32[order[k - 1]], L32[order[k]]
    fixed = [e for e in order if L32[e] > v_k + gap]
    band = [e for e in order if (v_k1 - gap) <= L32[e] <= (v_k + gap) and e not in fixed]
    out = [first]
    need = k - len(fixed)
    if need <= 0 or len(band) > 12:
        return out
    for combo in itertools.combinations(band, need):
        S = set(fixed) | set(combo)
        inside = [L32[e] for e in S]
        outside = [L32[e] for e in range(E) if e not in S]
        if min(inside) > max(outside) - gap:
            ordered = tuple(int(e) for e in order if e in S)
            if ordered not in out:
                out.append(ordered)
    return out


# ------------------------------------------------------------------ counts, permutation

def expert_counts(idx: np.ndarray, E: int) -> np.ndarray:
    """Tokens routed to each expert: a literal bincount over the flat expert ids."""
    counts = [0] * E
    for e in np.asarray(idx).ravel().tolist():
        counts[e] += 1
    return np.array(counts, dtype=np.int32)


def exclusive_offsets(counts: np.ndarray) -> np.ndarray:
    """offsets[e] = sum of counts[0..e-1]; offsets[E] = total.  int32 [E+1]."""
    off = [0]
    for c in np.asarray(counts).tolist():
        off.append(off[-1] + c)
    return np.array(off, dtype=np.int32)


def stable_permutation(idx: np.ndarray, E: int):
    """Group the (token, slot) pairs by expert, tokens ascending within an expert.

    Returns (counts [E], offsets [E+1], perm_src [T*k], perm_dst [T*k]):
    permuted row r holds token perm_src[r]; pair (t, j) lands in row perm_dst[t*k + j].
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    buckets = [[] for _ in range(E)]
    for t in range(T):
        for j in range(k):
            buckets[int(idx[t, j])].append((t, j))
    counts = expert_counts(idx, E)
    offsets = exclusive_offsets(counts)
    perm_src = np.empty(T * k, dtype=np.int32)
    perm_dst = np.empty(T * k, dtype=np.int32)
    r = 0
    for e in range(E):
        for (t, j) in buckets[e]:
            perm_src[r] = t
            perm_dst[t * k + j] = r
            r += 1
    return counts, offsets, perm_src, perm_dst


def gather_rows(hidden, perm_src) -> np.ndarray:
    """x_perm[r] = hidden[perm_src[r]] (a copy, same dtype)."""
    return np.asarray(hidden)[np.asarray(perm_src, dtype=np.int64)]


# ------------------------------------------------------------------------ experts

def silu(g: np.ndarray) -> np.ndarray:
    """silu(g) = g * sigmoid(g) = g / (1 + exp(-g))."""
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def swiglu(gate: np.ndarray, up: np.ndarray, alpha: float = 1.0, beta: float = 0.0,
           limit: float = float("inf")) -> np.ndarray:
    """SwiGLU with the op's attributes: (up' + beta) * gate' * sigmoid(alpha * gate'),
    gate' = min(gate, limit), up' = clip(up, -limit, limit).

    The standard attributes (1, 0, inf) give silu(gate) * up.
    """
    if limit != float("inf"):
        gate = np.minimum(gate, limit)
        up = np.clip(up, -limit, limit)
    if alpha == 1.0:
        s = silu(gate)
    else:
        with np.errstate(over="ignore"):
            s = gate / (1.0 + np.exp(-alpha * gate))
    return s * (up + beta) if beta != 0.0 else s * up


def fc1_gate_up(fc1_e: np.ndarray, layout: str):
    """Split one expert's fc1 [2I, H] into its gate rows and up rows, each [I, H]."""
    if layout == "interleaved":
        return fc1_e[0::2], fc1_e[1::2]
    if layout == "chunked":
        I = fc1_e.shape[0] // 2
        return fc1_e[:I], fc1_e[I:]
    raise ValueError(f"unknown fc1 layout {layout!r}")


def expert_ffn(x_rows, fc1_e, fc2_e, layout: str = "interleaved", act=STANDARD_SWIGLU,
               fc1_bias_e=None, fc2_bias_e=None) -> np.ndarray:
    """One expert on rows x [n, H]: gate = x W_gate^T (+ b_gate), up = x W_up^T (+ b_up),
    a = swiglu(gate, up, *act), y = a fc2^T (+ b2).  [n, H]; biases in fc1's layout."""
    x = np.asarray(x_rows, dtype=F64)
    w_gate, w_up = fc1_gate_up(np.asarray(fc1_e, dtype=F64), layout)
    gate, up = x @ w_gate.T, x @ w_up.T
    if fc1_bias_e is not None:
        b_gate, b_up = fc1_gate_up(np.asarray(fc1_bias_e, dtype=F64)[:, None], layout)
        gate, up = gate + b_gate[:, 0], up + b_up[:, 0]
    a = swiglu(gate, up, *act)
    y = a @ np.asarray(fc2_e, dtype=F64).T
    if fc2_bias_e is not None:
        y = y + np.asarray(fc2_bias_e, dtype=F64)
    return y


def combine(y_perm, perm_dst, w, T: int, k: int) -> np.ndarray:
    """out[t] = sum_j w[t, j] * y_perm[perm_dst[t*k + j]], float64 [T, H]."""
    y = np.asarray(y_perm, dtype=F64)
    out = np.zeros((T, y.shape[1]), dtype=F64)
    for j in range(k):
        rows = np.asarray(perm_dst, dtype=np.int64).reshape(T, k)[:, j]
        out += np.asarray(w, dtype=F64)[:, j:j + 1] * y[rows]
    return out


# ------------------------------------------------------------------------ pre-FFN norm

def dequantize_rows(q, scale) -> np.ndarray:
    """Weight-only int8 weights of one expert: w[r, :] = q[r, :] * scale[r], float64."""
    return np.asarray(q, dtype=F64) * np.asarray(scale, dtype=F64)[:, None]


def round_to_dtype(y, dtype: str) -> np.ndarray:
    """float64 values rounded once to the storage dtype, round to nearest, ties to
    even, returned as float64.  "f32": numpy's correctly rounded cast.  "bf16" (8
    significant bits, float32's exponent range): y = m 2^e with m in [0.5, 1) from
    frexp, m 2^8 rounded to an integer with ties to even (numpy's rint), scaled back
    -- every step exact in float64.  Values here stay in bf16's normal range."""
    y = np.asarray(y, dtype=F64)
    if dtype == "f32":
        return y.astype(np.float32).astype(F64)
    if dtype != "bf16":
        raise ValueError(f"unknown dtype {dtype!r}")
    m, e = np.frexp(y)
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def rms_norm(x, weight, eps: float) -> np.ndarray:
    """Llama-style RMSNorm of each row of x [T, H]: (x / sqrt(mean_h x^2 + eps)) * weight,
    float64, unrounded."""
    x = np.asarray(x, dtype=F64)
    r = 1.0 / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + F64(eps))
    return (x * r) * np.asarray(weight, dtype=F64)[None, :]


def pre_ffn_norm(x, weight, eps: float, dtype: str) -> np.ndarray:
    """The layer's input made from the residual activation x by the pre-FFN norm: the
    RMSNorm rounded to the storage dtype (float64 values of that dtype)."""
    return round_to_dtype(rms_norm(x, weight, eps), dtype)


# ------------------------------------------------------------------------ the layer

def moe_forward(hidden, router_w, router_bias, fc1: ArrayOrGetter, fc2: ArrayOrGetter,
                k: int, normalize: int, layout: str = "interleaved",
                idx: Optional[np.ndarray] = None,
                tokens: Optional[Sequence[int]] = None, act=STANDARD_SWIGLU,
                fc1_bias: Optional[ArrayOrGetter] = None,
                fc2_bias: Optional[ArrayOrGetter] = None) -> dict:
    """The fused MoE layer on the given tensors, float64.

    `idx` forces the routing (its weights are still computed from the logits);
    `tokens` restricts the expert evaluation to those tokens (routing is always over
    all tokens) and the returned `out` then has one row per listed token.  `act` is
    (alpha, beta, limit); fc1_bias [E, 2I] (fc1's layout) and fc2_bias [E, H] optional.
    Returns dict(logits, idx, w, out).
    """
    x = np.asarray(hidden)
    T = x.shape[0]
    L = router_logits(x, router_w, router_bias)
    if idx is None:
        idx = select_topk(L, k)
    w = routing_weights(L, idx, normalize)
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    out = np.zeros((tok.size, x.shape[1]), dtype=F64)
    if tok.size == 0:
        return dict(logits=L, idx=idx, w=w, out=out)
    sub_idx = idx[tok]
    E = np.asarray(router_w).shape[0]
    for e in range(E):
        rows, slots = np.nonzero(sub_idx == e)
        if rows.size == 0:
            continue
        y = expert_ffn(x[tok[rows]], _expert(fc1, e), _expert(fc2, e), layout, act,
                       None if fc1_bias is None else _expert(fc1_bias, e),
                       None if fc2_bias is None else _expert(fc2_bias, e))
        out[rows] += w[tok[rows], slots][:, None] * y
    return dict(logits=L, idx=idx, w=w, out=out)


def moe_dense_masked(hidden, router_w, router_bias, fc1, fc2, k: int, normalize: int,
                     layout: str = "interleaved", act=STANDARD_SWIGLU, fc1_bias=None,
                     fc2_bias=None) -> np.ndarray:
    """Brute force: every expert on every token, weighted by the routing mask.

    This is the static per-expert unroll of the fallback: expert e's output for all
    tokens times the token's weight for e (zero where e was not chosen).
    """
    x = np.asarray(hidden)
    T, H = x.shape
    E = np.asarray(router_w).shape[0]
    L = router_logits(x, router_w, router_bias)
    idx = select_topk(L, k)
    w = routing_weights(L, idx, normalize)
    mask = np.zeros((T, E), dtype=F64)
    for t in range(T):
        for j in range(k):
            mask[t, idx[t, j]] = w[t, j]
    out = np.zeros((T, H), dtype=F64)
    for e in range(E):
        out += mask[:, e:e + 1] * expert_ffn(
            x, _expert(fc1, e), _expert(fc2, e), layout, act,
            None if fc1_bias is None else _expert(fc1_bias, e),
            None if fc2_bias is None else _expert(fc2_bias, e))
    return out


def chunked_to_interleaved(fc1_chunked: np.ndarray) -> np.ndarray:
    """[E, 2I, H] chunked -> interleaved: dst[e, 2j+s] = src[e, s*I + j] for s in {0, 1}.
    Also for a bias [E, 2I] (rows of one element)."""
    src = np.asarray(fc1_chunked)
    E, two_i = src.shape[:2]
    I = two_i // 2
    dst = np.empty_like(src)
    for j in range(I):
        for s in (0, 1):
            dst[:, 2 * j + s] = src[:, s * I + j]
    return dst
