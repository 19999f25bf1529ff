"""ctypes loader for libmx.so, the C ABI declared in include/mx.h.

Only argument marshalling lives here.  There is no fallback: if the shared library is
missing or cannot be loaded, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("MX_LIB_PATH") or os.path.join(_PKG, "libmx.so")

# enum values of include/mx.h
MX_OK, MX_ERR_ARG, MX_ERR_SHAPE, MX_ERR_ALIGN, MX_ERR_LAYOUT, MX_ERR_CUDA, MX_ERR_TIMEOUT = range(7)
MX_FMT_E4M3, MX_FMT_E5M2, MX_FMT_E2M1, MX_FMT_NVFP4, MX_FMT_E2M3, MX_FMT_E3M2, MX_FMT_INT8 = 0, 1, 2, 3, 4, 5, 6
MX_AXIS_ROW, MX_AXIS_COL = 0, 1
MX_SCALE_FLOOR_OCP, MX_SCALE_CEIL_RECIPE = 0, 1
MX_LAYOUT_ROWMAJOR, MX_LAYOUT_TCGEN05 = 1, 2

# Every function the header declares (the CPU test checks the library exports them all).
EXPORTS = ("mx_scale_bytes", "mx_quantize", "mx_quantize_dual", "mx_dequantize", "mx_cast",
           "mx_gemm", "mx_status_string", "mx_last_cuda_error", "mx_watchdog_status",
           "mx_quantize_nvfp4_noalloc", "mx_mxfp4_to_fp8_blocks", "mx_quantize_nvfp4_2d", "mx_quantize_train",
           "mx_watchdog_selftest", "mx_quantize_mx_nvfp4")
WD_SELFTEST = 9
MX_NOALLOC_MAX_PARTIALS = 1024


class MxOperand(ctypes.Structure):
    _fields_ = [("elems", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("fmt", ctypes.c_int),
                ("global_scale", ctypes.c_void_p)]


class MxError(RuntimeError):
    def __init__(self, status: int, where: str, lib):
        self.status = status
        msg = lib.mx_status_string(status).decode()
        if status == MX_ERR_CUDA:
            msg += f" (cudaError {lib.mx_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmx.so not built ({LIB_PATH}); run python -m microscaling_precision_number_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I, U8P = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    lib.mx_scale_bytes.argtypes = [I64, I64, I]
    lib.mx_scale_bytes.restype = I64
    lib.mx_quantize.argtypes = [P, I64, I64, I, I, I, P, U8P, I, U8P, P, P]
    lib.mx_quantize.restype = I
    lib.mx_quantize_dual.argtypes = [P, I64, I64, I, I, P, U8P, P, U8P, I, U8P, U8P, P]
    lib.mx_quantize_dual.restype = I
    lib.mx_dequantize.argtypes = [P, U8P, P, I64, I64, I, I, P, P]
    lib.mx_dequantize.restype = I
    lib.mx_cast.argtypes = [P, I64, I, P, P]
    lib.mx_cast.restype = I
    lib.mx_gemm.argtypes = [MxOperand, MxOperand, P, I64, I64, I64, P]
    lib.mx_mxfp4_to_fp8_blocks.argtypes = [P, P, I64, I64, P, P, P, P]
    lib.mx_quantize_nvfp4_2d.argtypes = [P, I64, I64, P, P, I, P, P, P]
    lib.mx_quantize_nvfp4_2d.restype = I
    lib.mx_quantize_train.argtypes = [P, I64, I64, I, I, I, ctypes.c_uint, P, P, P, I, P, P, P]
    lib.mx_quantize_train.restype = I
    lib.mx_mxfp4_to_fp8_blocks.restype = I
    lib.mx_gemm.restype = I
    lib.mx_status_string.argtypes = [I]
    lib.mx_status_string.restype = ctypes.c_char_p
    lib.mx_last_cuda_error.argtypes = []
    lib.mx_last_cuda_error.restype = I
    lib.mx_watchdog_status.argtypes = [ctypes.POINTER(ctypes.c_int), I]
    lib.mx_watchdog_status.restype = I
    lib.mx_quantize_mx_nvfp4.argtypes = [P, I64, I64, I, I, P, U8P, I, U8P, P, U8P, I, U8P, P, P]
    lib.mx_quantize_mx_nvfp4.restype = I
    lib.mx_watchdog_selftest.argtypes = [ctypes.c_uint32, P]
    lib.mx_watchdog_selftest.restype = I
    # NVFP4 quantisation without any device allocation (static scratch array)
    lib.mx_quantize_nvfp4_noalloc.argtypes = [P, I64, I64, P, U8P, I, U8P, P, P]
    lib.mx_quantize_nvfp4_noalloc.restype = I
    return lib


class _LazyLib:
    """Loads libmx.so on first use (so that importing the package never needs the
    library, e.g. to build it); raises ImportError then if it is missing."""
    _handle = None

    def load(self):
        if _LazyLib._handle is None:
            _LazyLib._handle = _load()
        return _LazyLib._handle

    def __getattr__(self, name):
        return getattr(self.load(), name)


lib = _LazyLib()


def check(status: int, where: str) -> None:
    if status != MX_OK:
        raise MxError(status, where, lib)
