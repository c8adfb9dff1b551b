"""ctypes binding of the C ABI in ``include/qlora_nf4.h``.

Argument marshalling only: every function takes torch CUDA tensors, passes
their device pointers, sizes and the current CUDA stream to the library, and
turns a non-OK status into an exception.  All arithmetic runs in the
library's kernels.  There is no fallback: if the library is missing, loading
fails loudly.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# QLORA_LIBRARY=debug selects the bounds-checked build (libqlora_nf4_debug.so)
LIB_PATH = os.path.join(HERE, "libqlora_nf4_debug.so" if os.environ.get("QLORA_LIBRARY") == "debug"
                        else "libqlora_nf4.so")

QLORA_OK = 0
QLORA_ERR_INVALID_ARG = 1
QLORA_ERR_UNSUPPORTED = 2
QLORA_ERR_CUDA = 3
QLORA_ERR_TIMEOUT = 4
QLORA_ERR_WORKSPACE = 5
QLORA_ERR_BOUNDS = 6
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "TIMEOUT", 5: "WORKSPACE", 6: "BOUNDS"}
QLORA_F32 = 0
QLORA_BF16 = 1
CODE_TYPES = {"nf4": 0, "fp4": 1}
DQ_TYPES = {"int8": 0, "e4m3": 1}
QLORA_STATIC_QUANTIZE_MAX_ELEMS = 1 << 26

# Every function the header declares (checked against the header by the tests).
EXPORTS = (
    "qlora_nf4_quantize_workspace",
    "qlora_nf4_quantize",
    "qlora_nf4_quantize_static",
    "qlora_nf4_dequantize",
    "qlora_linear_workspace",
    "qlora_linear_fwd",
    "qlora_linear_bwd",
    "qlora_fused_linear_workspace",
    "qlora_fused_linear_fwd",
    "qlora_fused_linear_bwd",
    "qlora_lora_merge",
    "qlora_lora_unmerge",
    "qlora_adamw_step",
    "qlora_paged_alloc",
    "qlora_paged_free",
    "qlora_paged_prefetch",
    "qlora_get_last_error",
    "qlora_nf4_table",
    "qlora_nf4_encode",
    "qlora_dq_encode",
    "qlora_set_wait_timeout_ns",
    "qlora_debug_inject",
    "qlora_kernel_launches",
    "qlora_profile_enable",
    "qlora_profile_read",
)
KERNEL_KINDS = {"quantize": 0, "dequantize": 1, "fwd_gemm": 2, "dx_gemm": 3, "smallm_gemm": 4, "lora_gemm": 5,
                "merge": 6}


class QloraError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")
        self.status = status


class CNF4Weight(ctypes.Structure):
    """Mirror of ``qlora_nf4_weight``."""

    _fields_ = [
        ("rows", ctypes.c_int64),
        ("cols", ctypes.c_int64),
        ("blocksize", ctypes.c_int32),
        ("double_quant", ctypes.c_int32),
        ("codes", ctypes.c_void_p),
        ("absmax", ctypes.c_void_p),
        ("absmax_q8", ctypes.c_void_p),
        ("absmax_scale", ctypes.c_void_p),
        ("absmax_offset", ctypes.c_void_p),
        ("code_type", ctypes.c_int32),
        ("dq_type", ctypes.c_int32),
    ]


class CAdamWConfig(ctypes.Structure):
    """Mirror of ``qlora_adamw_config``."""

    _fields_ = [
        ("lr", ctypes.c_float),
        ("beta1", ctypes.c_float),
        ("beta2", ctypes.c_float),
        ("eps", ctypes.c_float),
        ("weight_decay", ctypes.c_float),
        ("grad_scale", ctypes.c_float),
        ("step", ctypes.c_int64),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"CUDA library {LIB_PATH} is missing; build it with "
            "`python -m bit_nf4_quantized_08_b200.build` (add --debug for the bounds-checked build; "
            "there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    W = ctypes.POINTER(CNF4Weight)
    L.qlora_nf4_quantize_workspace.argtypes = [i64, i64, i32, i32]
    L.qlora_nf4_quantize_workspace.restype = sz
    L.qlora_nf4_quantize.argtypes = [vp, i32, W, vp, sz, vp]
    L.qlora_nf4_quantize.restype = i32
    L.qlora_nf4_quantize_static.argtypes = [vp, i32, W, vp]
    L.qlora_nf4_quantize_static.restype = i32
    L.qlora_nf4_dequantize.argtypes = [W, vp, vp]
    L.qlora_nf4_dequantize.restype = i32
    L.qlora_linear_workspace.argtypes = [i64, W, i32, i32]
    L.qlora_linear_workspace.restype = sz
    L.qlora_linear_fwd.argtypes = [vp, i64, W, vp, vp, i32, f32, vp, vp, sz, vp]
    L.qlora_linear_fwd.restype = i32
    L.qlora_linear_bwd.argtypes = [vp, vp, i64, W, vp, vp, i32, f32, vp, vp, vp, vp, sz, vp]
    L.qlora_linear_bwd.restype = i32
    L.qlora_fused_linear_workspace.argtypes = [i64, W, i32, i32, i32]
    L.qlora_fused_linear_workspace.restype = sz
    L.qlora_fused_linear_fwd.argtypes = [vp, i64, W, i32, vp, vp, i32, f32, vp, vp, sz, vp]
    L.qlora_fused_linear_fwd.restype = i32
    L.qlora_fused_linear_bwd.argtypes = [vp, vp, i64, W, i32, vp, vp, i32, f32, vp, vp, vp, vp, sz, vp]
    L.qlora_fused_linear_bwd.restype = i32
    L.qlora_lora_merge.argtypes = [W, vp, vp, i32, f32, vp, vp]
    L.qlora_lora_merge.restype = i32
    L.qlora_lora_unmerge.argtypes = [vp, i64, i64, vp, vp, i32, f32, vp, vp]
    L.qlora_lora_unmerge.restype = i32
    L.qlora_adamw_step.argtypes = [vp, vp, vp, vp, vp, i64, ctypes.POINTER(CAdamWConfig), vp]
    L.qlora_adamw_step.restype = i32
    L.qlora_paged_alloc.argtypes = [sz, ctypes.POINTER(ctypes.c_void_p)]
    L.qlora_paged_alloc.restype = i32
    L.qlora_paged_free.argtypes = [vp]
    L.qlora_paged_free.restype = i32
    L.qlora_paged_prefetch.argtypes = [vp, sz, i32, vp]
    L.qlora_paged_prefetch.restype = i32
    L.qlora_get_last_error.argtypes = [vp]
    L.qlora_get_last_error.restype = i32
    L.qlora_nf4_table.argtypes = [vp]
    L.qlora_nf4_table.restype = None
    L.qlora_nf4_encode.argtypes = [vp, i64, vp, vp]
    L.qlora_nf4_encode.restype = i32
    L.qlora_dq_encode.argtypes = [vp, i64, vp, i32, vp]
    L.qlora_dq_encode.restype = i32
    L.qlora_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    L.qlora_set_wait_timeout_ns.restype = None
    L.qlora_debug_inject.argtypes = [i32]
    L.qlora_debug_inject.restype = None
    L.qlora_kernel_launches.argtypes = []
    L.qlora_kernel_launches.restype = ctypes.c_uint64
    L.qlora_profile_enable.argtypes = [i32]
    L.qlora_profile_enable.restype = None
    L.qlora_profile_read.argtypes = [i32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]
    L.qlora_profile_read.restype = i32
    env = os.environ.get("QLORA_WAIT_TIMEOUT_NS")
    if env:
        L.qlora_set_wait_timeout_ns(int(env))
    _lib = L
    return L


def check(status: int, what: str) -> None:
    if status != QLORA_OK:
        raise QloraError(status, what)
