"""The C ABI without a GPU: the library loads, exports every symbol include/*.h
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import glob
import os
import re

import pytest

from mixture_experts_ffn_15_b200 import _abi
from mixture_experts_ffn_15_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib():
    build()
    return _abi.load()


def declared_functions():
    names = set()
    for path in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(path).read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        src = re.sub(r"#[^\n]*", " ", src)
        for stmt in src.split(";"):
            stmt = " ".join(stmt.split())
            if not stmt or stmt.startswith("typedef") or "{" in stmt or "}" in stmt:
                continue
            m = re.match(r"^[\w\s\*]+?\b(\w+)\s*\(", stmt)
            if m:
                names.add(m.group(1))
    return names


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_forward",
              "convert_chunked_to_interleaved", "moe_workspace_size", "moe_get_error",
              "moe_rmsnorm", "moe_forward_static"):
        assert n in names


def test_header_compiles_as_c_and_cxx(tmp_path):
    """include/moe_b200.h is a plain C header (also valid C++)."""
    import shutil
    import subprocess
    hdr = os.path.join(ROOT, "include", "moe_b200.h")
    for cc, lang, std in (("gcc", "c", "-std=c99"), ("g++", "c++", "-std=c++17")):
        if shutil.which(cc) is None:
            pytest.skip(f"{cc} not installed")
        r = subprocess.run([cc, std, "-Wall", "-Werror", "-fsyntax-only", "-x", lang, hdr],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_package_exports_every_binding():
    import mixture_experts_ffn_15_b200 as moe
    from mixture_experts_ffn_15_b200 import ops
    public = [n for n, v in vars(ops).items() if callable(v) and not n.startswith("_")
              and getattr(v, "__module__", "") == ops.__name__]
    missing = [n for n in public if not hasattr(moe, n)]
    assert not missing, missing


def test_library_exports_every_declared_symbol():
    lib = _lib()
    missing = [n for n in sorted(declared_functions()) if not hasattr(lib, n)]
    assert not missing, missing
    # the binding declares the same set
    assert set(_abi.SIGNATURES) == declared_functions()


def test_status_strings_and_version():
    lib = _lib()
    assert lib.moe_status_string(0) == b"MOE_OK"
    assert lib.moe_status_string(2) == b"MOE_ERR_UNSUPPORTED"
    assert lib.moe_version() >= 100


def test_workspace_sizes():
    lib = _lib()
    # bf16: act and y_perm (every bf16 path gathers its token rows from hidden); float32
    # also keeps the permuted copy x_perm
    assert lib.moe_workspace_size(4, 2816, 128, 8, 704, _abi.MOE_BF16) > 4 * 8 * (2816 + 704) * 2
    assert lib.moe_workspace_size(4, 2816, 128, 8, 704, _abi.MOE_F32) > 4 * 8 * (2 * 2816 + 704) * 4
    assert lib.moe_workspace_size(4, 2816, 128, 300, 704, _abi.MOE_BF16) == 0     # k > E
    assert lib.moe_workspace_size(4, 2816, 300, 8, 704, _abi.MOE_BF16) == 0       # E > 256
    assert lib.moe_workspace_size(4, 2817, 128, 8, 704, _abi.MOE_BF16) == 0       # H % 8
    assert lib.moe_workspace_size(4, 2816, 128, 8, 704, 7) == 0                   # dtype
    a = lib.moe_workspace_size(100, 256, 8, 2, 128, _abi.MOE_BF16)
    b = lib.moe_workspace_size(200, 256, 8, 2, 128, _abi.MOE_BF16)
    assert b > a and a % 256 == 0
    assert lib.moe_permute_workspace_size(1000, 64) >= 8 * 64 * 4   # per-tile counts


def _fwd(lib, T=4, H=128, E=8, k=2, I=64, act=_abi.STANDARD_SWIGLU, dt=_abi.MOE_BF16, ptr=16,
         layout=_abi.MOE_FC1_INTERLEAVED, norm=None, eps=1e-6):
    p = ctypes.c_void_p(ptr)
    return lib.moe_forward(p, norm, eps, p, None, p, p, None, None, T, H, E, k, I, 1, act, layout,
                           dt, p, ctypes.c_void_p(256), 1 << 40, None)


def test_host_validation_before_any_device_work():
    lib = _lib()
    assert _fwd(lib, k=9) == _abi.MOE_ERR_INVALID_ARG
    assert _fwd(lib, T=-1) == _abi.MOE_ERR_INVALID_ARG
    assert _fwd(lib, H=100) == _abi.MOE_ERR_INVALID_ARG
    nan = float("nan")
    assert _fwd(lib, act=_abi.MoeSwiglu(nan, 1.0, 7.0)) == _abi.MOE_ERR_INVALID_ARG     # alpha
    assert _fwd(lib, act=_abi.MoeSwiglu(1.702, float("inf"), 7.0)) == _abi.MOE_ERR_INVALID_ARG
    assert _fwd(lib, act=_abi.MoeSwiglu(1.702, 1.0, 0.0)) == _abi.MOE_ERR_INVALID_ARG   # limit
    assert _fwd(lib, layout=2) == _abi.MOE_ERR_INVALID_ARG  # no such fc1 layout
    assert _fwd(lib, layout=-1) == _abi.MOE_ERR_INVALID_ARG
    assert _fwd(lib, T=0, layout=_abi.MOE_FC1_CHUNKED) == _abi.MOE_OK
    q = ctypes.c_void_p(32)
    assert _fwd(lib, norm=q, eps=-1.0) == _abi.MOE_ERR_INVALID_ARG        # eps < 0
    assert _fwd(lib, norm=q, eps=float("nan")) == _abi.MOE_ERR_INVALID_ARG
    assert _fwd(lib, norm=ctypes.c_void_p(34)) == _abi.MOE_ERR_INVALID_ARG  # misaligned weight
    assert _fwd(lib, norm=q, eps=-1.0, T=0) == _abi.MOE_ERR_INVALID_ARG
    assert lib.moe_rmsnorm(q, q, 4, 64, 1e-6, _abi.MOE_BF16, ctypes.c_void_p(64), None) == \
        _abi.MOE_ERR_INVALID_ARG                                           # y overlaps x
    assert lib.moe_rmsnorm(q, q, 4, 60, 1e-6, _abi.MOE_BF16, ctypes.c_void_p(8192), None) == \
        _abi.MOE_ERR_INVALID_ARG                                           # H % 8
    assert lib.moe_rmsnorm(q, q, 0, 64, 1e-6, _abi.MOE_BF16, q, None) == _abi.MOE_OK
    assert _fwd(lib, H=72) == _abi.MOE_ERR_UNSUPPORTED      # bf16 needs H % 64 == 0
    assert _fwd(lib, T=0) == _abi.MOE_OK                   # empty batch: nothing to do
    assert _fwd(lib, ptr=18) == _abi.MOE_ERR_INVALID_ARG    # misaligned tensors
    p = ctypes.c_void_p(4096)
    assert lib.convert_chunked_to_interleaved(p, ctypes.c_void_p(4096 + 64), 2, 8, 64,
                                              _abi.MOE_BF16, None) == _abi.MOE_ERR_INVALID_ARG
    assert lib.moe_get_error(None, None, None) == _abi.MOE_ERR_INVALID_ARG
    assert lib.moe_set_stage_events((ctypes.c_void_p * 2)(), 2) == _abi.MOE_ERR_INVALID_ARG
    assert lib.moe_set_stage_events(None, 0) == _abi.MOE_OK


def _fwd_q8(lib, T=4, H=128, E=8, k=2, I=64, s1=32, s2=32, ptr=16):
    p = ctypes.c_void_p(ptr)
    sc = lambda v: None if v is None else ctypes.c_void_p(v)
    return lib.moe_forward_q8(p, None, 1e-6, p, None, p, sc(s1), p, sc(s2), None, None, T, H, E, k,
                              I, 1, _abi.STANDARD_SWIGLU, _abi.MOE_FC1_INTERLEAVED, p,
                              ctypes.c_void_p(256), 1 << 40, None)


def test_q8_host_validation_before_any_device_work():
    """The int8-expert entry points refuse bad arguments and sizes outside the decode FFN
    before anything is enqueued (every call here returns before a launch)."""
    lib = _lib()
    assert _fwd_q8(lib, s1=None) == _abi.MOE_ERR_INVALID_ARG           # no scales
    assert _fwd_q8(lib, s2=None) == _abi.MOE_ERR_INVALID_ARG
    assert _fwd_q8(lib, s1=34) == _abi.MOE_ERR_INVALID_ARG             # misaligned scales
    assert _fwd_q8(lib, k=9) == _abi.MOE_ERR_INVALID_ARG
    assert _fwd_q8(lib, H=72) == _abi.MOE_ERR_UNSUPPORTED              # no tensor-core tiling
    assert _fwd_q8(lib, T=0) == _abi.MOE_OK
    assert _fwd_q8(lib, T=4096, E=8, k=2) == _abi.MOE_ERR_UNSUPPORTED  # 1024 rows per expert
    p = ctypes.c_void_p(16)
    q8 = lambda rows, s1=32, H=128, I=64: lib.moe_expert_ffn_q8(
        p, p, p, None if s1 is None else ctypes.c_void_p(s1), p, ctypes.c_void_p(32), None, None,
        rows, H, 8, I, _abi.STANDARD_SWIGLU, _abi.MOE_FC1_INTERLEAVED, p, ctypes.c_void_p(256),
        1 << 40, None)
    assert q8(-1) == _abi.MOE_ERR_INVALID_ARG
    assert q8(16, s1=None) == _abi.MOE_ERR_INVALID_ARG
    assert q8(8 * 65) == _abi.MOE_ERR_UNSUPPORTED                     # > 64 rows per expert
    assert q8(16, I=96) == _abi.MOE_ERR_UNSUPPORTED                   # 2I not a multiple of 128
    assert q8(0) == _abi.MOE_OK


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_abi, "_lib", None)
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(ImportError, match="build"):
        _abi.load()


def test_forward_path_per_workload():
    """moe_forward_path: which kernels run for each workload (host arithmetic only)."""
    lib = _lib()
    bf, f32 = _abi.MOE_BF16, _abi.MOE_F32
    small, fused, tc_router, token, fma, one_launch = 1, 2, 4, 8, 16, 32
    assert lib.moe_forward_path(64, 256, 8, 2, 128, f32) == small | fma
    assert lib.moe_forward_path(4, 2816, 128, 8, 704, bf) == one_launch | fused
    assert lib.moe_forward_path(64, 2816, 128, 8, 704, bf) == one_launch | fused
    assert lib.moe_forward_path(65, 2816, 128, 8, 704, bf) == tc_router | fused
    assert lib.moe_forward_path(16, 2816, 128, 8, 704, bf) == one_launch | fused
    assert lib.moe_forward_path(256, 2816, 128, 8, 704, bf) == tc_router | fused
    assert lib.moe_forward_path(16, 192, 8, 2, 704, bf) == small | token      # H % 128 != 0
    assert lib.moe_forward_path(8192, 2816, 128, 8, 704, bf) == tc_router | token
    assert lib.moe_forward_path(32768, 4096, 64, 4, 1536, bf) == tc_router | token
    assert lib.moe_forward_path(300, 128, 8, 2, 704, bf) == small | token   # > 64 rows per expert
    assert lib.moe_forward_path(4, 2816, 128, 300, 704, bf) == 0
