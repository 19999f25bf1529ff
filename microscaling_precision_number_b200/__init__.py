"""Microscaling (MX) number formats on NVIDIA B200 (sm_100a).

MXFP8 (E4M3/E5M2) and MXFP4 (E2M1) quantisation with E8M0 block scales, NVFP4 (E2M1 with
UE4M3 block scales and an FP32 tensor scale), dequantisation, the direct cast, and the
tcgen05 block-scaled matmul (MXFP8 x MXFP8, MXFP8 x MXFP4, MXFP4 x MXFP4, NVFP4 x NVFP4) -- all in hand-written CUDA kernels behind the C ABI of
include/mx.h (libmx.so).  This package is the thin Python binding over that ABI.
"""
from . import _lib
from ._lib import MxError
from .api import (Quantized, block_of, cast, dequantize, elem_bytes, gemm, is_fp4, quantize,
                  quantize_dual, quantize_mx_nvfp4, quantize_nvfp4_2d, quantize_train, scale_bytes,
                  watchdog_status)

__all__ = ["MxError", "Quantized", "block_of", "cast", "dequantize", "elem_bytes", "gemm", "is_fp4", "quantize",
           "quantize_dual", "quantize_mx_nvfp4", "quantize_nvfp4_2d", "quantize_train", "scale_bytes",
           "watchdog_status", "_lib"]
