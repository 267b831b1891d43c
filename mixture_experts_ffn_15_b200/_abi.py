"""ctypes declarations of the C ABI in include/moe_b200.h (argument marshalling only)."""
import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_DEVICE, MOE_ERR_TIMEOUT = range(6)
MOE_F32, MOE_BF16 = 0, 1
MOE_FC1_INTERLEAVED, MOE_FC1_CHUNKED = 0, 1
MOE_DEVERR_BAD_EXPERT, MOE_DEVERR_TIMEOUT = 1, 2


class MoeSwiglu(ctypes.Structure):
    _fields_ = [("alpha", ctypes.c_float), ("beta", ctypes.c_float), ("limit", ctypes.c_float)]


STANDARD_SWIGLU = MoeSwiglu(1.0, 0.0, float("inf"))
GPT_OSS_SWIGLU = MoeSwiglu(1.702, 1.0, 7.0)

_vp, _i, _sz, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float

# name -> (restype, argtypes), in the order of include/moe_b200.h
SIGNATURES = {
    "moe_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "moe_permute_workspace_size": (_sz, [_i, _i]),
    "moe_expert_ffn_workspace_size": (_sz, [_i, _i, _i]),
    "moe_workspace_error_word": (_vp, [_vp]),
    "moe_route": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp]),
    "moe_permute": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_expert_ffn": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, MoeSwiglu, _i, _i, _vp,
                            _vp, _sz, _vp]),
    "moe_combine": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp]),
    "moe_rmsnorm": (_i, [_vp, _vp, _i, _i, _f, _i, _vp, _vp]),
    "moe_forward": (_i, [_vp, _vp, _f, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                         MoeSwiglu, _i, _i, _vp, _vp, _sz, _vp]),
    "moe_forward_static": (_i, [_vp, _vp, _f, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                _i, MoeSwiglu, _i, _i, _vp, _vp]),
    "moe_forward_q8": (_i, [_vp, _vp, _f, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                            _i, _i, MoeSwiglu, _i, _vp, _vp, _sz, _vp]),
    "moe_expert_ffn_q8": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, MoeSwiglu,
                               _i, _vp, _vp, _sz, _vp]),
    "convert_chunked_to_interleaved": (_i, [_vp, _vp, _i, _i, _i, _i, _vp]),
    "moe_get_error": (_i, [_vp, _vp, ctypes.POINTER(ctypes.c_int32)]),
    "moe_status_string": (ctypes.c_char_p, [_i]),
    "moe_set_stage_events": (_i, [ctypes.POINTER(_vp), _i]),
    "moe_forward_path": (_i, [_i, _i, _i, _i, _i, _i]),
    "moe_kernel_launches": (ctypes.c_ulonglong, []),
    "moe_debug_arm_route_barrier_timeout": (None, []),
    "moe_version": (_i, []),
}

_lib = None


def load():
    """Load libmoe_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m mixture_experts_ffn_15_b200.build` "
            "(the layer has no other implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class MoEError(RuntimeError):
    def __init__(self, status, where):
        lib = load()
        super().__init__(f"{where}: {lib.moe_status_string(status).decode()} ({status})")
        self.status = status


def check(status, where):
    if status != MOE_OK:
        raise MoEError(status, where)
