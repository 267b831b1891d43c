"""moe_forward_static: the layer for callers that cannot allocate device memory.

Such callers (an engine plugin or serving loop that forbids allocation once it
runs, a plain C host without an allocator) pass only inputs and outputs; the
scratch lives in a fixed array inside the library.  These tests call the entry
point through the C ABI, one call after another on the shared array, each on other
sizes and inputs and on another path of the layer, so that whatever one call leaves
in the array would show up in the next.  Each output must be bit for bit the output
of moe_forward on a caller-allocated workspace (the same kernels on the same
inputs) and match the oracle within the stated tolerance.
"""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_ffn_15_b200 as moe
from mixture_experts_ffn_15_b200 import _abi
from oracle import moe_oracle as O
from parity_util import assert_close, device_inputs, from_dev, match_routing, tol
from synth import Workload, make_inputs

pytestmark = pytest.mark.gpu

PATH_FUSED_ROUTE, PATH_TC_ROUTER, PATH_SMALL_ROUTE = 32, 4, 1


def _static_forward(dev, wl, out):
    lib = _abi.load()
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.moe_forward_static(p(dev["hidden"]), None, 1e-6, p(dev["router_w"]),
                                  p(dev["router_bias"]),
                                  p(dev["fc1"]), p(dev["fc2"]), None, None, wl.T, wl.H, wl.E,
                                  wl.k, wl.I,
                                  wl.normalize, _abi.STANDARD_SWIGLU, _abi.MOE_FC1_INTERLEAVED,
                                  _abi.MOE_BF16, p(out),
                                  stream)


# one call after another on the shared array: the one-launch decode path, the decode
# shape's tensor-core router (72 tokens: near the array's limit there), the one-CTA
# router for an expert count the tensor-core router does not take, and the one-launch
# path again
CALLS = [
    (Workload("static_a", T=9, H=512, E=16, k=4, I=256, dtype="bf16", seed=11), PATH_FUSED_ROUTE),
    (Workload("static_decode72", T=72, H=2816, E=128, k=8, I=704, dtype="bf16", seed=13),
     PATH_TC_ROUTER),
    (Workload("static_small", T=100, H=512, E=16, k=4, I=256, dtype="bf16", seed=14),
     PATH_SMALL_ROUTE),
    (Workload("static_b", T=5, H=512, E=16, k=4, I=256, dtype="bf16", seed=12,
              router_bias_std=0.5), PATH_FUSED_ROUTE),
]


def test_static_scratch_matches_workspace_forward_and_oracle_on_calls_in_a_row():
    lib = _abi.load()
    for wl, path_bit in CALLS:
        assert lib.moe_workspace_size(wl.T, wl.H, wl.E, wl.k, wl.I, _abi.MOE_BF16) <= (8 << 20)
        assert lib.moe_forward_path(wl.T, wl.H, wl.E, wl.k, wl.I, _abi.MOE_BF16) & path_bit, wl.name
        inp = make_inputs(wl)
        dev = device_inputs(inp)
        ref = moe.forward(dev["hidden"], dev["router_w"], dev["fc1"], dev["fc2"], wl.k,
                          router_bias=dev["router_bias"])
        out = torch.full_like(ref, float("nan"))
        st = _static_forward(dev, wl, out)
        assert st == _abi.MOE_OK, lib.moe_status_string(st)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), \
            f"{wl.name}: static scratch differs from the caller's workspace"
        # and against the oracle, on the routing the GPU chose (near ties resolved)
        r = moe.route(dev["hidden"], dev["router_w"], wl.k, router_bias=dev["router_bias"])
        torch.cuda.synchronize()
        L = O.router_logits(inp.values("hidden"), inp.values("router_w"), inp["router_bias"])
        idx, _ = match_routing(L, from_dev(r["idx"]).astype(np.int64), wl.k)
        want = O.moe_forward(inp.values("hidden"), inp.values("router_w"), inp["router_bias"],
                             lambda e: inp.expert_values("fc1", e),
                             lambda e: inp.expert_values("fc2", e), wl.k, wl.normalize,
                             idx=idx)["out"]
        atol, rtol = tol("bf16", want)
        assert_close(from_dev(out), want, atol, rtol, f"{wl.name} static vs oracle")


def test_static_scratch_rejects_sizes_beyond_its_array():
    wl = Workload("static_big", T=512, H=2816, E=128, k=8, I=704, dtype="bf16")
    need = _abi.load().moe_workspace_size(wl.T, wl.H, wl.E, wl.k, wl.I, _abi.MOE_BF16)
    assert need > (8 << 20)
    x = torch.zeros((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    dev = dict(hidden=x, router_w=x[:wl.E], router_bias=None, fc1=x, fc2=x)
    assert _static_forward(dev, wl, x) == _abi.MOE_ERR_INVALID_ARG
