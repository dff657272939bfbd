"""ctypes binding of libfp8q.so (the C ABI declared in include/fp8q.h).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels. There is no fallback: if the library is missing
or fails to load, loading raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfp8q.so")

_lock = threading.Lock()
_lib = None

P = ctypes.c_void_p
U32 = ctypes.c_uint32
I32 = ctypes.c_int32
SZ = ctypes.c_size_t


class QuantPick(ctypes.Structure):
    """Mirror of fp8q_quant_pick_t."""
    _fields_ = [
        ("variant", ctypes.c_int32),
        ("grid_x", ctypes.c_uint32),
        ("block_x", ctypes.c_uint32),
        ("groups_per_cta", ctypes.c_uint32),
        ("multi_ctas", ctypes.c_uint32),
        ("floor_ctas", ctypes.c_uint32),
        ("forced", ctypes.c_int32),
    ]


# name -> (restype, argtypes), one entry per function declared in include/fp8q.h
SIGNATURES = {
    "fp8q_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "fp8q_version": (ctypes.c_char_p, []),
    "fp8q_m_pad": (U32, [U32]),
    "fp8q_quant_floor_min_m": (U32, [U32, U32, U32, U32, ctypes.c_float]),
    "fp8q_quant_pick": (ctypes.c_int, [U32, U32, U32, I32, ctypes.POINTER(QuantPick)]),
    "fp8q_quant_act": (ctypes.c_int, [P, P, P, P, U32, U32, P]),
    "fp8q_quant_act_variant": (ctypes.c_int, [P, P, P, P, U32, U32, I32, P]),
    "fp8q_quant_weight": (ctypes.c_int, [P, P, P, U32, U32, P]),
    "fp8q_gemm_blockscaled": (ctypes.c_int, [P, P, P, P, P, U32, U32, U32, P]),
    "fp8q_quant_weight_rowwise": (ctypes.c_int, [P, P, P, U32, U32, P]),
    "fp8q_gemm_ex": (ctypes.c_int, [P, P, P, P, I32, P, U32, U32, U32, P]),
    "fp8q_linear_ex": (ctypes.c_int, [P, P, P, I32, P, P, SZ, U32, U32, U32, P]),
    "fp8q_linear_decode_fused": (ctypes.c_int, [P, P, P, I32, P, P, SZ, U32, U32, U32, P]),
    "fp8q_linear_workspace_bytes": (SZ, [U32, U32]),
    "fp8q_linear_scale_offset": (SZ, [U32, U32]),
    "fp8q_linear": (ctypes.c_int, [P, P, P, P, P, SZ, U32, U32, U32, P]),
    "fp8q_linear_noalloc": (ctypes.c_int, [P, P, P, P, U32, U32, U32, P]),
    "fp8q_diag_stalled_linear": (ctypes.c_int, [P, P, P, P, P, SZ, U32, U32, U32, ctypes.c_uint64, P]),
    "fp8q_silu_mul_quant": (ctypes.c_int, [P, P, U32, P, P, P, U32, U32, P]),
    "fp8q_ffn_workspace_layout": (ctypes.c_int, [U32, U32, U32, ctypes.POINTER(SZ)]),
    "fp8q_ffn_workspace_bytes": (SZ, [U32, U32, U32]),
    "fp8q_ffn": (ctypes.c_int, [P, P, P, P, P, P, P, SZ, U32, U32, U32, P]),
    "fp8q_check_silu_mul": (ctypes.c_int, [P, P, P]),
    "fp8q_nvfp4_sf_mma_bytes": (SZ, [U32, U32]),
    "fp8q_nvfp4_quant": (ctypes.c_int, [P, P, P, P, ctypes.c_float, U32, U32, P]),
    "fp8q_nvfp4_gemm": (ctypes.c_int, [P, P, ctypes.c_float, P, P, ctypes.c_float, P, U32, U32, U32, P]),
    "fp8q_nvfp4_linear_workspace_bytes": (SZ, [U32, U32]),
    "fp8q_nvfp4_linear": (ctypes.c_int, [P, ctypes.c_float, P, P, ctypes.c_float, P, P, SZ, U32, U32, U32, P]),
    "fp8q_dequant_fp8_bf16": (ctypes.c_int, [P, P, I32, P, U32, U32, P]),
    "fp8q_convert_e2m1": (ctypes.c_int, [P, P, SZ, P]),
    "fp8q_convert_e4m3": (ctypes.c_int, [P, P, SZ, P]),
    "fp8q_check_division": (ctypes.c_int, [P, P]),
    "fp8q_launch_count": (ctypes.c_uint64, []),
    "fp8q_device_error": (ctypes.c_int, [P, ctypes.POINTER(ctypes.c_uint32)]),
}


def load():
    """Load libfp8q.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -c 'import __graft_entry__ as g; g.build()'`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


class Fp8qError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = load().fp8q_status_string(status).decode()
        super().__init__(f"{what}: {msg}" if what else msg)


def check(status: int, what: str = "") -> None:
    if status != 0:
        raise Fp8qError(status, what)
