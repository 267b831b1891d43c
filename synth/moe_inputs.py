"""Seeded synthetic inputs for the fused mixture-of-experts FFN layer.

This module only draws numbers and stores them; it holds none of the layer's
arithmetic.  Both the CUDA path (through the tests and the benchmark) and the
CPU oracle read the arrays it returns, so they see identical bits.

Distribution recipe (one workload = one row of the workload table below):

* hidden        ~ N(0, 1)                      [T, H]
* router_w      ~ N(0, 0.02)                   [E, H]   (the second argument is a std)
* router_bias   ~ N(0, bias_std), float32      [E]      (only where the workload has one)
* fc1           ~ N(0, 1/sqrt(H))              [E, 2I, H]  (fan-in H)
* fc2           ~ N(0, 1/sqrt(I))              [E, H, I]   (fan-in I)
* outliers      round(frac * T) distinct rows of hidden, drawn without replacement,
                scaled by `outlier_scale` before rounding.

Every tensor has its own stream, `numpy.random.default_rng([seed, stream, ...])`
(PCG64 seeded through SeedSequence), so a tensor's values do not depend on which
other tensors were drawn.  The expert weights are drawn one expert at a time with
stream `[seed, stream, e]`.  Values are drawn in float32 and, for bf16 workloads,
rounded to bfloat16 with round-to-nearest-even on the host; bf16 tensors are kept
as uint16 bit patterns, and `values()` widens them back to float32 exactly.

`fc1` is produced in the layout the workload names: "interleaved" (row 2i is the
gate of intermediate unit i, row 2i+1 its up projection) or "chunked" (the
Hugging Face `experts.gate_up_proj` layout: rows 0..I-1 gate, rows I..2I-1 up).
The draw is the same array either way; only the name of the layout changes how
the consumer reads it.
"""

from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional

import numpy as np

# Stream identifiers: fixed forever, so that a seed always means the same tensors.
_S_HIDDEN, _S_ROUTER, _S_BIAS, _S_FC1, _S_FC2, _S_OUTLIER = 1, 2, 3, 4, 5, 6
_S_FC1_BIAS, _S_FC2_BIAS, _S_NORM_W, _S_RESIDUAL = 7, 8, 9, 10
_S_Q1, _S_Q2, _S_QS1, _S_QS2 = 11, 12, 13, 14


@dataclass(frozen=True)
class Workload:
    name: str
    T: int            # tokens
    H: int            # hidden size
    E: int            # experts
    k: int            # experts per token
    I: int            # expert intermediate size
    dtype: str        # "f32" or "bf16": storage of activations and weights
    normalize: int = 1
    router_bias_std: Optional[float] = None
    fc1_layout: str = "interleaved"
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    seed: int = 0

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the fused MoE layer, smallest first.
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", T=64, H=256, E=8, k=2, I=128, dtype="f32"),
    "decode_bf16": Workload("decode_bf16", T=4, H=2816, E=128, k=8, I=704, dtype="bf16"),
    "batched_decode_bf16": Workload(
        "batched_decode_bf16", T=256, H=2816, E=128, k=8, I=704, dtype="bf16",
        router_bias_std=0.5),
    "prefill_bf16": Workload(
        "prefill_bf16", T=8192, H=2816, E=128, k=8, I=704, dtype="bf16",
        fc1_layout="chunked"),
    "long_prefill_bf16": Workload(
        "long_prefill_bf16", T=32768, H=4096, E=64, k=4, I=1536, dtype="bf16",
        outlier_frac=0.01, outlier_scale=8.0),
}


def round_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float32 values (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(seed_key, shape, std) -> np.ndarray:
    rng = np.random.default_rng(list(seed_key))
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


class MoEInputs:
    """The tensors of one workload, in storage form.

    bf16 tensors are uint16 bit arrays, f32 tensors float32 arrays.  `values(name)`
    returns float32 values for either; `router_bias` is float32 or None.
    """

    def __init__(self, wl: Workload, arrays: dict):
        self.wl = wl
        self.arrays = arrays

    def __getitem__(self, name):
        return self.arrays[name]

    def values(self, name) -> Optional[np.ndarray]:
        a = self.arrays[name]
        if a is None:
            return None
        if a.dtype == np.uint16:
            return bf16_bits_to_f32(a)
        return a

    def expert_values(self, name, e) -> np.ndarray:
        """float32 values of expert e's slice of fc1 or fc2."""
        a = self.arrays[name][e]
        return bf16_bits_to_f32(a) if a.dtype == np.uint16 else a


def _store(a32: np.ndarray, dtype: str) -> np.ndarray:
    return round_to_bf16_bits(a32) if dtype == "bf16" else a32


def outlier_rows(wl: Workload, seed: int) -> np.ndarray:
    """Sorted indices of the hidden rows scaled as outliers (empty if none)."""
    n = int(round(wl.outlier_frac * wl.T))
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    rng = np.random.default_rng([seed, _S_OUTLIER])
    return np.sort(rng.choice(wl.T, size=n, replace=False))


def make_inputs(wl: Workload, seed: Optional[int] = None, weights: bool = True) -> MoEInputs:
    """Draw the tensors of `wl` (optionally with another seed).

    With weights=False only hidden, router_w and router_bias are drawn (cheap
    routing-only studies); fc1 and fc2 are then None.
    """
    s = wl.seed if seed is None else seed
    T, H, E, I = wl.T, wl.H, wl.E, wl.I

    hidden = _normal((s, _S_HIDDEN), (T, H), 1.0)
    rows = outlier_rows(wl, s)
    if rows.size:
        hidden[rows] *= np.float32(wl.outlier_scale)
    router_w = _normal((s, _S_ROUTER), (E, H), 0.02)
    bias = None
    if wl.router_bias_std is not None:
        bias = _normal((s, _S_BIAS), (E,), wl.router_bias_std)

    arrays = {
        "hidden": _store(hidden, wl.dtype),
        "router_w": _store(router_w, wl.dtype),
        "router_bias": bias,
        "fc1": None,
        "fc2": None,
    }
    if weights:
        store_dt = np.uint16 if wl.dtype == "bf16" else np.float32
        fc1 = np.empty((E, 2 * I, H), dtype=store_dt)
        fc2 = np.empty((E, H, I), dtype=store_dt)
        s1, s2 = 1.0 / np.sqrt(H), 1.0 / np.sqrt(I)
        for e in range(E):
            fc1[e] = _store(_normal((s, _S_FC1, e), (2 * I, H), s1), wl.dtype)
            fc2[e] = _store(_normal((s, _S_FC2, e), (H, I), s2), wl.dtype)
        arrays["fc1"] = fc1
        arrays["fc2"] = fc2
    return MoEInputs(wl, arrays)


def make_expert_biases(wl: Workload, std: float = 0.5, seed: Optional[int] = None):
    """The op's optional expert biases for `wl`: fc1_bias [E, 2I] (in the row order of
    the workload's fc1 layout) and fc2_bias [E, H], N(0, std), stored like the weights
    (bf16 bits or float32)."""
    s = wl.seed if seed is None else seed
    b1 = _normal((s, _S_FC1_BIAS), (wl.E, 2 * wl.I), std)
    b2 = _normal((s, _S_FC2_BIAS), (wl.E, wl.H), std)
    return _store(b1, wl.dtype), _store(b2, wl.dtype)


def make_pre_norm_inputs(wl: Workload, scale: float = 4.0, seed: Optional[int] = None):
    """Inputs of the pre-FFN RMSNorm for `wl`: a residual-stream activation [T, H]
    (N(0, scale), a scale other than 1 so that the normalisation shows) and the norm
    weight [H] (N(1, 0.1): a trained Llama-style weight sits near one), both stored
    like the workload's activations (bf16 bits or float32)."""
    s = wl.seed if seed is None else seed
    x = _normal((s, _S_RESIDUAL), (wl.T, wl.H), scale)
    w = 1.0 + _normal((s, _S_NORM_W), (wl.H,), 0.1)
    return _store(x, wl.dtype), _store(w.astype(np.float32), wl.dtype)


def make_q8_experts(wl: Workload, seed: Optional[int] = None):
    """Weight-only int8 experts for `wl`: per expert, q = round(N(0, 1) * 127 / 4)
    clipped to [-127, 127] (int8) and one float32 scale per weight row, the layer's
    weight std (1/sqrt(H) for fc1, 1/sqrt(I) for fc2) * 4 / 127 times U(0.75, 1.25), so
    that q * scale has about the std of the bf16 weights.  Returns (fc1_q [E, 2I, H]
    int8 in the workload's fc1 layout, fc1_scale [E, 2I] float32, fc2_q [E, H, I] int8,
    fc2_scale [E, H] float32), drawn expert by expert."""
    s = wl.seed if seed is None else seed
    E, H, I = wl.E, wl.H, wl.I
    fc1_q = np.empty((E, 2 * I, H), dtype=np.int8)
    fc2_q = np.empty((E, H, I), dtype=np.int8)
    for e in range(E):
        for dst, key, shape in ((fc1_q, _S_Q1, (2 * I, H)), (fc2_q, _S_Q2, (H, I))):
            z = _normal((s, key, e), shape, 127.0 / 4.0)
            dst[e] = np.clip(np.rint(z), -127, 127).astype(np.int8)
    u1 = np.random.default_rng([s, _S_QS1]).uniform(0.75, 1.25, size=(E, 2 * I))
    u2 = np.random.default_rng([s, _S_QS2]).uniform(0.75, 1.25, size=(E, H))
    fc1_scale = (u1 * (4.0 / 127.0) / np.sqrt(H)).astype(np.float32)
    fc2_scale = (u2 * (4.0 / 127.0) / np.sqrt(I)).astype(np.float32)
    return fc1_q, fc1_scale, fc2_q, fc2_scale
