"""ctypes declarations of the libint8mm C-ABI (include/int8mm.h).

Marshalling only: every step of the computation runs in the CUDA library.
Loading fails loudly when the library is missing; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libint8mm.so")

OK = 0
STATUS_NAMES = {
    0: "INT8MM_OK",
    1: "INT8MM_ERR_INVALID_ARGUMENT",
    2: "INT8MM_ERR_MISALIGNED",
    3: "INT8MM_ERR_WORKSPACE_TOO_SMALL",
    4: "INT8MM_ERR_UNSUPPORTED_DEVICE",
    5: "INT8MM_ERR_CUDA",
    6: "INT8MM_ERR_TIMEOUT",
    7: "INT8MM_ERR_OUTLIER_OVERFLOW",
}
PATH_AUTO, PATH_GEMM, PATH_DECODE, PATH_GEMM_1SM = 0, 1, 2, 3

# Every symbol the header declares.
EXPORTS = (
    "int8mm_status_string", "int8mm_version", "int8mm_weight_bytes", "int8mm_prepare_weight",
    "int8mm_workspace_bytes", "int8mm_workspace_init", "int8mm_forward", "int8mm_forward_ex",
    "int8mm_forward_host",
    "int8mm_workspace_view_get", "int8mm_get_device_status",
    "int8mm_forward_decode_noalloc", "int8mm_noalloc_device_status",
    "int8mm_block_quantize", "int8mm_block_dequantize",
    "int8mm_int4_weight_bytes", "int8mm_prepare_weight_int4", "int8mm_forward_int4",
    "int8mm_grouped_weight_bytes", "int8mm_prepare_weight_grouped", "int8mm_grouped_workspace_bytes",
    "int8mm_grouped_workspace_view_get", "int8mm_forward_grouped",
)


class Int8mmError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}" if what else STATUS_NAMES.get(status, str(status)))


class Weight(ctypes.Structure):
    _fields_ = [
        ("K", ctypes.c_int32), ("N", ctypes.c_int32), ("n_keep", ctypes.c_int32),
        ("wq", ctypes.c_void_p), ("col_absmax", ctypes.c_void_p), ("w_keep", ctypes.c_void_p),
        ("keep_idx", ctypes.c_void_p), ("keep_slot", ctypes.c_void_p),
    ]


class GroupedWeight(ctypes.Structure):
    _fields_ = [
        ("K", ctypes.c_int32), ("N", ctypes.c_int32), ("G", ctypes.c_int32), ("n_keep", ctypes.c_int32),
        ("wq", ctypes.c_void_p), ("col_absmax", ctypes.c_void_p), ("w_keep", ctypes.c_void_p),
        ("keep_idx", ctypes.c_void_p), ("keep_slot", ctypes.c_void_p),
    ]


class Int4Weight(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int32), ("N", ctypes.c_int32), ("G", ctypes.c_int32),
                ("codes", ctypes.c_void_p), ("absmax", ctypes.c_void_p)]


class ForwardOpts(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("acc_out", ctypes.c_void_p), ("wait_limit_ns", ctypes.c_uint64),
                ("main_start_event", ctypes.c_void_p), ("main_stop_event", ctypes.c_void_p),
                ("test_flags", ctypes.c_uint32)]


TEST_WITHHOLD_SIGNAL = 1


class WorkspaceView(ctypes.Structure):
    _fields_ = [
        ("status", ctypes.c_void_p), ("n_outliers", ctypes.c_void_p), ("outlier_idx", ctypes.c_void_p),
        ("row_absmax", ctypes.c_void_p), ("xq", ctypes.c_void_p), ("xo", ctypes.c_void_p), ("kp", ctypes.c_int32),
    ]


_lib = None


def load(path: str | None = None):
    """Load libint8mm.so (built by ``int8_quantized_matmul_02_b200.build``)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"libint8mm.so not found at {p}; build it with "
                          "`python -m int8_quantized_matmul_02_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(p)
    I, P, S, F = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float
    lib.int8mm_status_string.argtypes = [I]
    lib.int8mm_status_string.restype = ctypes.c_char_p
    lib.int8mm_version.argtypes = []
    lib.int8mm_version.restype = I
    lib.int8mm_weight_bytes.argtypes = [I, I, I]
    lib.int8mm_weight_bytes.restype = S
    lib.int8mm_prepare_weight.argtypes = [P, I, I, P, I, P, S, ctypes.POINTER(Weight), P]
    lib.int8mm_prepare_weight.restype = I
    lib.int8mm_workspace_bytes.argtypes = [I, I, I, I]
    lib.int8mm_workspace_bytes.restype = S
    lib.int8mm_workspace_init.argtypes = [P, S, P]
    lib.int8mm_workspace_init.restype = I
    lib.int8mm_forward.argtypes = [P, I, ctypes.POINTER(Weight), F, I, P, P, S, P]
    lib.int8mm_forward.restype = I
    lib.int8mm_forward_ex.argtypes = [P, I, ctypes.POINTER(Weight), F, I, P, P, S, ctypes.POINTER(ForwardOpts), P]
    lib.int8mm_forward_ex.restype = I
    lib.int8mm_forward_host.argtypes = [P, I, ctypes.POINTER(Weight), F, I, P, P, P, P, S, P]
    lib.int8mm_forward_host.restype = I
    lib.int8mm_workspace_view_get.argtypes = [P, S, I, I, I, I, ctypes.POINTER(WorkspaceView)]
    lib.int8mm_workspace_view_get.restype = I
    lib.int8mm_get_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
    lib.int8mm_get_device_status.restype = I
    lib.int8mm_forward_decode_noalloc.argtypes = [P, I, ctypes.POINTER(Weight), F, P, P]
    lib.int8mm_forward_decode_noalloc.restype = I
    lib.int8mm_noalloc_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_int32)]
    lib.int8mm_noalloc_device_status.restype = I
    L64 = ctypes.c_int64
    lib.int8mm_block_quantize.argtypes = [P, L64, I, P, P, P]
    lib.int8mm_block_quantize.restype = I
    lib.int8mm_block_dequantize.argtypes = [P, P, L64, I, P, P]
    lib.int8mm_block_dequantize.restype = I
    lib.int8mm_int4_weight_bytes.argtypes = [I, I, I]
    lib.int8mm_int4_weight_bytes.restype = S
    lib.int8mm_prepare_weight_int4.argtypes = [P, I, I, I, P, S, ctypes.POINTER(Int4Weight), P]
    lib.int8mm_prepare_weight_int4.restype = I
    lib.int8mm_forward_int4.argtypes = [P, I, ctypes.POINTER(Int4Weight), P, P, P]
    lib.int8mm_forward_int4.restype = I
    lib.int8mm_grouped_weight_bytes.argtypes = [I, I, I, I]
    lib.int8mm_grouped_weight_bytes.restype = S
    lib.int8mm_prepare_weight_grouped.argtypes = [P, I, I, I, P, I, P, S, ctypes.POINTER(GroupedWeight), P]
    lib.int8mm_prepare_weight_grouped.restype = I
    lib.int8mm_grouped_workspace_bytes.argtypes = [I, I, I, I, I]
    lib.int8mm_grouped_workspace_bytes.restype = S
    lib.int8mm_grouped_workspace_view_get.argtypes = [P, S, I, I, I, I, I, ctypes.POINTER(WorkspaceView)]
    lib.int8mm_grouped_workspace_view_get.restype = I
    lib.int8mm_forward_grouped.argtypes = [P, I, ctypes.POINTER(GroupedWeight), F, I, P, P, S,
                                           ctypes.POINTER(ForwardOpts), P]
    lib.int8mm_forward_grouped.restype = I
    if path is None:
        _lib = lib
    return lib


def check(status: int, what: str = "") -> None:
    if status != OK:
        raise Int8mmError(status, what)
