"""moe_forward_static: the layer for callers that cannot allocate device memory.

Such callers (an engine plugin or serving loop that forbids allocation once it
runs, a plain C host without an allocator) pass only inputs and outputs; the
scratch lives in a fixed array inside the library.  These tests call the entry
point through the C ABI and compare it with moe_forward, which takes a
caller-allocated workspace, on two calls in a row with different inputs, so that
whatever the first call leaves in the shared array cannot leak into the second.
"""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_ffn_15_b200 as moe
from mixture_experts_ffn_15_b200 import _abi
from parity_util import BF16_ATOL, BF16_RTOL, assert_close, device_inputs, from_dev
from synth import Workload, make_inputs

pytestmark = pytest.mark.gpu


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


def test_static_scratch_matches_workspace_forward_on_two_calls():
    first = Workload("static_a", T=9, H=512, E=16, k=4, I=256, dtype="bf16", seed=11)
    second = Workload("static_b", T=5, H=512, E=16, k=4, I=256, dtype="bf16", seed=12,
                      router_bias_std=0.5)
    for wl in (first, second):
        dev = device_inputs(make_inputs(wl))
        ref = moe.forward(dev["hidden"], dev["router_w"], dev["fc1"], dev["fc2"], wl.k,
                          router_bias=dev["router_bias"])
        out = torch.full_like(ref, float("nan"))
        st = _static_forward(dev, wl, out)
        assert st == _abi.MOE_OK, _abi.load().moe_status_string(st)
        torch.cuda.synchronize()
        got = from_dev(out)
        assert np.isfinite(got).all()
        assert_close(got, from_dev(ref), BF16_ATOL, BF16_RTOL, f"{wl.name} static vs workspace")


def test_static_scratch_rejects_sizes_beyond_its_array():
    wl = Workload("static_big", T=512, H=2816, E=128, k=8, I=704, dtype="bf16")
    need = _abi.load().moe_workspace_size(wl.T, wl.H, wl.E, wl.k, wl.I, _abi.MOE_BF16)
    assert need > (8 << 20)
    x = torch.zeros((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    dev = dict(hidden=x, router_w=x[:wl.E], router_bias=None, fc1=x, fc2=x)
    assert _static_forward(dev, wl, x) == _abi.MOE_ERR_INVALID_ARG
