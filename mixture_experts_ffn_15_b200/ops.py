"""Torch-facing wrappers of the C ABI.

PyTorch provides device memory and streams only: every step of the layer runs in
the CUDA kernels of libmoe_b200.so.  These functions check dtypes, devices, shapes
and contiguity, allocate outputs and workspaces with torch when the caller does
not pass them, and raise MoEError on any non-OK status.
"""
import ctypes

import torch

from . import _abi
from ._abi import STANDARD_SWIGLU, MoeSwiglu, check

_DT = {torch.bfloat16: _abi.MOE_BF16, torch.float32: _abi.MOE_F32}


def _lib():
    return _abi.load()


def _dtcode(t):
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}: bfloat16 or float32") from None


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype=None, shape=None):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _swiglu(alpha, beta, limit):
    return MoeSwiglu(alpha, beta, limit)


_LAYOUT = {"interleaved": 0, "chunked": 1}


def _layout(fc1_layout):
    if fc1_layout not in _LAYOUT:
        raise ValueError(f"fc1_layout must be 'interleaved' or 'chunked', got {fc1_layout!r}")
    return _LAYOUT[fc1_layout]


def workspace_size(T, H, E, k, I, dtype):
    """Bytes of workspace moe_forward needs (0 for sizes it rejects)."""
    return _lib().moe_workspace_size(T, H, E, k, I, _DT[dtype])


def alloc_workspace(nbytes, device):
    """Device workspace, zero-filled (moe_forward wants zeros before its first call)."""
    return torch.zeros(int(nbytes), dtype=torch.uint8, device=device)


def _biases(fc1_bias, fc2_bias, dt, E, I, H):
    if fc1_bias is not None:
        _need(fc1_bias, "fc1_bias", dt, (E, 2 * I))
    if fc2_bias is not None:
        _need(fc2_bias, "fc2_bias", dt, (E, H))


def forward(hidden, router_w, fc1, fc2, k, normalize=True, router_bias=None, out=None,
            workspace=None, stream=None, swiglu=(1.0, 0.0, float("inf")), fc1_bias=None,
            fc2_bias=None, fc1_layout="interleaved", norm_weight=None, norm_eps=1e-6):
    """The fused MoE layer: out[T, H] = sum_j w[t, j] * FFN_{idx[t, j]}(hidden[t]).

    swiglu = (alpha, beta, limit) of the op; fc1_layout "interleaved" (rows 2i, 2i+1 =
    gate_i, up_i) or "chunked" (rows i, I+i), read in place either way; fc1_bias
    [E, 2I] (fc1's layout) and fc2_bias [E, H] are the optional expert biases.  With
    norm_weight [H], hidden is the residual activation and the layer runs on its
    pre-FFN RMSNorm (computed inside the call, see rmsnorm)."""
    _need(hidden, "hidden")
    dt = hidden.dtype
    T, H = hidden.shape
    E = router_w.shape[0]
    I = fc2.shape[2]
    _need(router_w, "router_w", dt, (E, H))
    _need(fc1, "fc1", dt, (E, 2 * I, H))
    _need(fc2, "fc2", dt, (E, H, I))
    if router_bias is not None:
        _need(router_bias, "router_bias", torch.float32, (E,))
    _biases(fc1_bias, fc2_bias, dt, E, I, H)
    if norm_weight is not None:
        _need(norm_weight, "norm_weight", dt, (H,))
    if out is None:
        out = torch.empty_like(hidden)
    _need(out, "out", dt, (T, H))
    need = workspace_size(T, H, E, k, I, dt)
    if workspace is None:
        # invalid sizes give 0 bytes; the C call then reports them
        workspace = alloc_workspace(max(need, 256), hidden.device)
    _need(workspace, "workspace", torch.uint8)
    st = _lib().moe_forward(_ptr(hidden), _ptr(norm_weight), float(norm_eps), _ptr(router_w),
                            _ptr(router_bias), _ptr(fc1), _ptr(fc2),
                            _ptr(fc1_bias), _ptr(fc2_bias), T, H, E, k, I, int(bool(normalize)),
                            _swiglu(*swiglu), _layout(fc1_layout), _dtcode(hidden), _ptr(out),
                            _ptr(workspace),
                            workspace.numel(), _stream(stream))
    check(st, "moe_forward")
    return out


def _q8(q, scale, name, rows_shape):
    _need(q, name, torch.int8, rows_shape)
    _need(scale, name + "_scale", torch.float32, rows_shape[:2])


def forward_q8(hidden, router_w, fc1_q, fc1_scale, fc2_q, fc2_scale, k, normalize=True,
               router_bias=None, out=None, workspace=None, stream=None,
               swiglu=(1.0, 0.0, float("inf")), fc1_bias=None, fc2_bias=None,
               fc1_layout="interleaved", norm_weight=None, norm_eps=1e-6):
    """The layer with weight-only int8 experts: weight = q * scale of its row (fc1_q
    [E, 2I, H] int8 with fc1_scale [E, 2I] float32, fc2_q [E, H, I] with fc2_scale
    [E, H]); hidden and the rest bf16, as in forward.  Decode-sized batches only."""
    _need(hidden, "hidden", torch.bfloat16)
    T, H = hidden.shape
    E = router_w.shape[0]
    I = fc2_q.shape[2]
    _need(router_w, "router_w", torch.bfloat16, (E, H))
    _q8(fc1_q, fc1_scale, "fc1", (E, 2 * I, H))
    _q8(fc2_q, fc2_scale, "fc2", (E, H, I))
    if router_bias is not None:
        _need(router_bias, "router_bias", torch.float32, (E,))
    _biases(fc1_bias, fc2_bias, torch.bfloat16, E, I, H)
    if norm_weight is not None:
        _need(norm_weight, "norm_weight", torch.bfloat16, (H,))
    if out is None:
        out = torch.empty_like(hidden)
    _need(out, "out", torch.bfloat16, (T, H))
    need = workspace_size(T, H, E, k, I, torch.bfloat16)
    if workspace is None:
        workspace = alloc_workspace(max(need, 256), hidden.device)
    _need(workspace, "workspace", torch.uint8)
    st = _lib().moe_forward_q8(_ptr(hidden), _ptr(norm_weight), float(norm_eps), _ptr(router_w),
                               _ptr(router_bias), _ptr(fc1_q), _ptr(fc1_scale), _ptr(fc2_q),
                               _ptr(fc2_scale), _ptr(fc1_bias), _ptr(fc2_bias), T, H, E, k, I,
                               int(bool(normalize)), _swiglu(*swiglu), _layout(fc1_layout),
                               _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream))
    check(st, "moe_forward_q8")
    return out


def expert_ffn_q8(x_perm, offsets, fc1_q, fc1_scale, fc2_q, fc2_scale, y_perm=None, stream=None,
                  swiglu=(1.0, 0.0, float("inf")), fc1_bias=None, fc2_bias=None,
                  fc1_layout="interleaved"):
    """expert_ffn with weight-only int8 experts (see forward_q8)."""
    _need(x_perm, "x_perm", torch.bfloat16)
    rows, H = x_perm.shape
    E, two_i, _ = fc1_q.shape
    I = two_i // 2
    _need(offsets, "offsets", torch.int32, (E + 1,))
    _q8(fc1_q, fc1_scale, "fc1", (E, 2 * I, H))
    _q8(fc2_q, fc2_scale, "fc2", (E, H, I))
    _biases(fc1_bias, fc2_bias, torch.bfloat16, E, I, H)
    if y_perm is None:
        y_perm = torch.zeros_like(x_perm)
    ws = alloc_workspace(_lib().moe_expert_ffn_workspace_size(rows, I, _DT[torch.bfloat16]),
                         x_perm.device)
    st = _lib().moe_expert_ffn_q8(_ptr(x_perm), _ptr(offsets), _ptr(fc1_q), _ptr(fc1_scale),
                                  _ptr(fc2_q), _ptr(fc2_scale), _ptr(fc1_bias), _ptr(fc2_bias), rows,
                                  H, E, I, _swiglu(*swiglu), _layout(fc1_layout), _ptr(y_perm),
                                  _ptr(ws), ws.numel(), _stream(stream))
    check(st, "moe_expert_ffn_q8")
    return y_perm


def rmsnorm(x, weight, eps=1e-6, out=None, stream=None):
    """Pre-FFN RMSNorm: (x / sqrt(mean(x^2) + eps)) * weight per row, float64 inside,
    rounded once to x's dtype."""
    _need(x, "x")
    T, H = x.shape
    _need(weight, "weight", x.dtype, (H,))
    if out is None:
        out = torch.empty_like(x)
    _need(out, "out", x.dtype, (T, H))
    check(_lib().moe_rmsnorm(_ptr(x), _ptr(weight), T, H, float(eps), _dtcode(x), _ptr(out),
                             _stream(stream)), "moe_rmsnorm")
    return out


def workspace_error_word(workspace):
    """The int32 error word at the start of a moe_forward workspace, as a tensor view."""
    return workspace[:4].view(torch.int32)


def route(hidden, router_w, k, normalize=True, router_bias=None, stream=None):
    """Router logits, top-k (descending, ties to the lower index) and routing weights."""
    _need(hidden, "hidden")
    T, H = hidden.shape
    E = router_w.shape[0]
    _need(router_w, "router_w", hidden.dtype, (E, H))
    if router_bias is not None:
        _need(router_bias, "router_bias", torch.float32, (E,))
    dev = hidden.device
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    near = torch.empty((T,), dtype=torch.int32, device=dev)
    st = _lib().moe_route(_ptr(hidden), _ptr(router_w), _ptr(router_bias), T, H, E, k,
                          int(bool(normalize)), _dtcode(hidden), _ptr(idx), _ptr(w), _ptr(logits),
                          _ptr(near), _stream(stream))
    check(st, "moe_route")
    return dict(idx=idx, w=w, logits=logits, near_tie=near)


def permute(topk_idx, E, hidden=None, err_word=None, stream=None):
    """Bincount, offsets, stable permutation and (with hidden) the gathered rows."""
    _need(topk_idx, "topk_idx", torch.int32)
    T, k = topk_idx.shape
    dev = topk_idx.device
    H = hidden.shape[1] if hidden is not None else 8
    dt = _dtcode(hidden) if hidden is not None else _abi.MOE_BF16
    counts = torch.empty((E,), dtype=torch.int32, device=dev)
    offsets = torch.empty((E + 1,), dtype=torch.int32, device=dev)
    perm_src = torch.full((T * k,), -1, dtype=torch.int32, device=dev)
    perm_dst = torch.empty((T * k,), dtype=torch.int32, device=dev)
    x_perm = None
    if hidden is not None:
        _need(hidden, "hidden")
        x_perm = torch.empty((T * k, H), dtype=hidden.dtype, device=dev)
    if err_word is None:
        err_word = torch.zeros((1,), dtype=torch.int32, device=dev)
    ws = alloc_workspace(_lib().moe_permute_workspace_size(T, E), dev)
    st = _lib().moe_permute(_ptr(hidden), _ptr(topk_idx), T, H, E, k, dt, _ptr(counts),
                            _ptr(offsets), _ptr(perm_src), _ptr(perm_dst), _ptr(x_perm),
                            _ptr(err_word), _ptr(ws), ws.numel(), _stream(stream))
    check(st, "moe_permute")
    return dict(counts=counts, offsets=offsets, perm_src=perm_src, perm_dst=perm_dst,
                x_perm=x_perm, err_word=err_word)


def expert_ffn(x_perm, offsets, fc1, fc2, y_perm=None, stream=None,
               swiglu=(1.0, 0.0, float("inf")), fc1_bias=None, fc2_bias=None,
               fc1_layout="interleaved"):
    """y_perm[r] = fc2_e act(x fc1_gate^T + b_gate, x fc1_up^T + b_up) + b2_e over each
    expert's rows (act: SwiGLU with the op's (alpha, beta, limit); fc1 and fc1_bias in
    fc1_layout, "interleaved" or "chunked")."""
    _need(x_perm, "x_perm")
    rows, H = x_perm.shape
    E, two_i, _ = fc1.shape
    I = two_i // 2
    _need(offsets, "offsets", torch.int32, (E + 1,))
    _need(fc1, "fc1", x_perm.dtype, (E, 2 * I, H))
    _need(fc2, "fc2", x_perm.dtype, (E, H, I))
    _biases(fc1_bias, fc2_bias, x_perm.dtype, E, I, H)
    if y_perm is None:
        y_perm = torch.zeros_like(x_perm)
    dt = _dtcode(x_perm)
    ws = alloc_workspace(_lib().moe_expert_ffn_workspace_size(rows, I, dt), x_perm.device)
    st = _lib().moe_expert_ffn(_ptr(x_perm), _ptr(offsets), _ptr(fc1), _ptr(fc2), _ptr(fc1_bias),
                               _ptr(fc2_bias), rows, H, E, I, _swiglu(*swiglu),
                               _layout(fc1_layout), dt, _ptr(y_perm),
                               _ptr(ws), ws.numel(), _stream(stream))
    check(st, "moe_expert_ffn")
    return y_perm


def combine(y_perm, perm_dst, topk_w, T, k, out=None, stream=None):
    """out[t] = sum_j topk_w[t, j] * y_perm[perm_dst[t*k + j]] (float32 sum, slot order)."""
    _need(y_perm, "y_perm")
    H = y_perm.shape[1]
    _need(perm_dst, "perm_dst", torch.int32)
    _need(topk_w, "topk_w", torch.float32)
    if out is None:
        out = torch.empty((T, H), dtype=y_perm.dtype, device=y_perm.device)
    st = _lib().moe_combine(_ptr(y_perm), _ptr(perm_dst), _ptr(topk_w), T, H, k, _dtcode(y_perm),
                            _ptr(out), _stream(stream))
    check(st, "moe_combine")
    return out


def convert_chunked_to_interleaved(src, dst=None, stream=None):
    """[E, 2I, H] gate-rows-then-up-rows -> interleaved (row 2j gate_j, row 2j+1 up_j)."""
    _need(src, "src")
    E, two_i, H = src.shape
    if dst is None:
        dst = torch.empty_like(src)
    _need(dst, "dst", src.dtype, src.shape)
    st = _lib().convert_chunked_to_interleaved(_ptr(src), _ptr(dst), E, two_i // 2, H,
                                               _dtcode(src), _stream(stream))
    check(st, "convert_chunked_to_interleaved")
    return dst


def get_error(err_word, stream=None):
    """(status, bits) of a device error word; synchronises the stream."""
    bits = ctypes.c_int32(0)
    st = _lib().moe_get_error(_ptr(err_word), _stream(stream), ctypes.byref(bits))
    return st, bits.value


def set_stage_events(events):
    """Record 6 cudaEvent handles around the stages of every moe_forward (None: off)."""
    lib = _lib()
    if events is None:
        check(lib.moe_set_stage_events(None, 0), "moe_set_stage_events")
        return
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e) for e in events])
    check(lib.moe_set_stage_events(arr, len(events)), "moe_set_stage_events")
