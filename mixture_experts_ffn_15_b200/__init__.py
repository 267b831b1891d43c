"""Fused mixture-of-experts FFN layer (com.microsoft::MoE with standard SwiGLU) for B200.

The layer runs in the CUDA kernels of libmoe_b200.so (sm_100a), behind the C ABI
declared in include/moe_b200.h; this package is the thin Python binding.
"""
from ._abi import MoEError, load as load_library  # noqa: F401
from .ops import (alloc_workspace, combine, convert_chunked_to_interleaved,  # noqa: F401
                  expert_ffn, expert_ffn_q8, forward, forward_q8, get_error, permute, rmsnorm,
                  route, set_stage_events,
                  workspace_error_word, workspace_size)

__all__ = ["forward", "forward_q8", "rmsnorm", "route", "permute", "expert_ffn", "expert_ffn_q8",
           "combine",
           "convert_chunked_to_interleaved", "get_error", "set_stage_events",
           "workspace_size", "alloc_workspace", "workspace_error_word", "load_library",
           "MoEError"]
