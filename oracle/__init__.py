"""CPU oracle for MX / NVFP4 quantisation, dequantisation and the block-scaled matmul.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this package.
The product library never imports, links or calls it, and it never imports the product.

The arithmetic lives in ``mx_oracle.c`` (plain C, integer bit manipulation, one plain
loop per block).  This module only marshals numpy arrays through ctypes and builds the
shared object with gcc when it is missing.

Every function's definition and the passage it follows are documented in ``mx_oracle.c``.
Parity status: every function here is pinned by the ``-m "not gpu"`` oracle tests, the
NVFP4 element step (the E2M1 code of the fp32 quotient x / d) exhaustively against
numpy's IEEE division and an exact nearest-code search, and the whole NVFP4 quantiser
against vLLM's torch reference quantiser (equal codes except one-step differences at
rounding midpoints, where the two place their fp32 roundings differently).  The tcgen05
scale tiling, which
the pages do not define, is pinned on the CPU against vLLM's implementation of the
block-scaling-factor layout cuBLAS documents, and on hardware by the block-scaled matmul
and by cuBLASLt's MXFP8 matmul reading the same scale bytes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mx_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

# Format and code-kind identifiers (the same numbering as mx_oracle.c).
E4M3, E5M2, E2M1, NVFP4, E2M3, E3M2, INT8 = 0, 1, 2, 3, 4, 5, 6
K_E4M3, K_E5M2, K_E2M1, K_UE4M3, K_E8M0, K_BF16, K_E2M3, K_E3M2, K_INT8 = 0, 1, 2, 3, 4, 5, 6, 7, 8
FLOOR, CEIL = 0, 1
ROW, COL = 0, 1


def build(force: bool = False) -> str:
    """Compile mx_oracle.c with gcc (no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
            "-fno-fast-math", "-frounding-math", "-o", tmp, _SRC, "-lm",
        ])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        _lib.mxo_decode.argtypes = [I, ctypes.c_uint]
        _lib.mxo_decode.restype = ctypes.c_double
        _lib.mxo_encode.argtypes = [ctypes.c_double, I]
        _lib.mxo_encode.restype = ctypes.c_uint
        _lib.mxo_scale_exponent.argtypes = [ctypes.c_double, I, I]
        _lib.mxo_scale_exponent.restype = I
        _lib.mxo_quantize_mx.argtypes = [P, I64, I64, I, I, I, P, P]
        _lib.mxo_quantize_mx.restype = I
        _lib.mxo_cast.argtypes = [P, I64, I, P]
        _lib.mxo_cast.restype = I
        _lib.mxo_quantize_nvfp4.argtypes = [P, I64, I64, P, P, P]
        _lib.mxo_quantize_nvfp4.restype = I
        _lib.mxo_dequantize_mx.argtypes = [P, P, I64, I64, I, P]
        _lib.mxo_dequantize_mx.restype = I
        _lib.mxo_dequantize_nvfp4.argtypes = [P, P, ctypes.c_float, I64, I64, P]
        _lib.mxo_dequantize_nvfp4.restype = I
        _lib.mxo_tcgen05_scale_bytes.argtypes = [I64, I64]
        _lib.mxo_tcgen05_scale_bytes.restype = I64
        _lib.mxo_tcgen05_scale_offset.argtypes = [I64, I64, I64, I64]
        _lib.mxo_tcgen05_scale_offset.restype = I64
        _lib.mxo_gemm_ref.argtypes = [P, P, I, ctypes.c_double, P, P, I, ctypes.c_double, I64, I64, I64, P, I64, P, P]
        _lib.mxo_gemm_ref.restype = I
        _lib.mxo_gemm_ref_block.argtypes = [P, P, I, ctypes.c_double, P, P, I, ctypes.c_double, I64, I64, I64,
                                            I64, I64, I64, I64, P, P, P, P]
        _lib.mxo_gemm_ref_block.restype = I
        _lib.mxo_to_tcgen05_layout.argtypes = [P, I64, I64, P]
        _lib.mxo_to_tcgen05_layout.restype = I
        _lib.mxo_from_tcgen05_layout.argtypes = [P, I64, I64, P]
        _lib.mxo_from_tcgen05_layout.restype = I
        _lib.mxo_quantize_mx_sr.argtypes = [P, I64, I64, I, I, P, P, P]
        _lib.mxo_quantize_mx_sr.restype = I
        _lib.mxo_quantize_nvfp4_sr.argtypes = [P, I64, I64, P, P, P, P]
        _lib.mxo_quantize_nvfp4_sr.restype = I
        _lib.mxo_rht16.argtypes = [P, I64, I64, ctypes.c_uint, P]
        _lib.mxo_rht16.restype = I
        _lib.mxo_quantize_nvfp4_2d.argtypes = [P, I64, I64, P, P, P]
        _lib.mxo_quantize_nvfp4_2d.restype = I
        _lib.mxo_mxfp4_to_fp8_blocks.argtypes = [P, P, I64, I64, P, P, P]
        _lib.mxo_mxfp4_to_fp8_blocks.restype = I
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments (rc={rc})")


# ---------------------------------------------------------------- scalar codecs
def decode(kind: int, code: int) -> float:
    """Exact value of one code (E4M3, E5M2, E2M1, UE4M3, E8M0, bf16 bits, E2M3, E3M2 or INT8)."""
    return lib().mxo_decode(kind, code)


def encode(value: float, kind: int) -> int:
    """Saturating round-to-nearest-even code of one value (no block scale)."""
    return lib().mxo_encode(float(value), kind)


def scale_exponent(amax: float, fmt: int, rounding: int) -> int:
    """Shared exponent s (clamped to [-127, 127]) for a block maximum."""
    return lib().mxo_scale_exponent(float(amax), fmt, rounding)


def code_bits(fmt: int) -> int:
    """Stored width of one element code: FP4 4, FP6 6, FP8 / INT8 8."""
    return 4 if fmt in (E2M1, NVFP4) else 6 if fmt in (E2M3, E3M2) else 8


def elem_bytes(n_elems: int, fmt: int) -> int:
    """Bytes of n densely packed element codes (n * width / 8)."""
    return n_elems * code_bits(fmt) // 8


# ---------------------------------------------------------------- block operations
def quantize_mx(x_bf16_bits: np.ndarray, fmt: int, axis: int = ROW, rounding: int = CEIL):
    """MX quantisation of a 2-D bf16 matrix given as uint16 bit patterns.

    Returns (elems, scales): row-wise elems rows x bytes(cols), scales rows x cols/32;
    col-wise the output is transposed: elems cols x bytes(rows), scales cols x rows/32.
    """
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    rows, cols = x.shape
    orow, ocol = (rows, cols) if axis == ROW else (cols, rows)
    elems = np.zeros((orow, elem_bytes(ocol, fmt)), dtype=np.uint8)
    scales = np.zeros((orow, ocol // 32), dtype=np.uint8)
    _check(lib().mxo_quantize_mx(_ptr(x), rows, cols, fmt, axis, rounding, _ptr(elems), _ptr(scales)),
           "quantize_mx")
    return elems, scales


def cast(x_bf16_bits: np.ndarray, fmt: int) -> np.ndarray:
    """Direct element cast with no block scale (codes densely packed: FP4 two per byte,
    FP6 four per three bytes)."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16).reshape(-1)
    out = np.zeros(elem_bytes(x.size, fmt), dtype=np.uint8)
    _check(lib().mxo_cast(_ptr(x), x.size, fmt, _ptr(out)), "cast")
    return out


def quantize_nvfp4(x_bf16_bits: np.ndarray):
    """NVFP4 quantisation. Returns (elems rows x cols/2, scales rows x cols/16, g)."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    rows, cols = x.shape
    elems = np.zeros((rows, cols // 2), dtype=np.uint8)
    scales = np.zeros((rows, cols // 16), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    _check(lib().mxo_quantize_nvfp4(_ptr(x), rows, cols, _ptr(elems), _ptr(scales), _ptr(g)),
           "quantize_nvfp4")
    return elems, scales, float(g[0])


def quantize_nvfp4_2d(x_bf16_bits: np.ndarray):
    """NVFP4 with 16 x 16 weight blocks.  Returns (elems rows x cols/2, scales rows x cols/16
    with each 2-D block's code on its 16 rows, g)."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    rows, cols = x.shape
    elems = np.zeros((rows, cols // 2), dtype=np.uint8)
    scales = np.zeros((rows, cols // 16), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    _check(lib().mxo_quantize_nvfp4_2d(_ptr(x), rows, cols, _ptr(elems), _ptr(scales), _ptr(g)),
           "quantize_nvfp4_2d")
    return elems, scales, float(g[0])


def dequantize_mx(elems: np.ndarray, scales: np.ndarray, rows: int, cols: int, fmt: int) -> np.ndarray:
    """bf16 bits (uint16) of dec(q) * 2^(s-127); scale 0xFF gives NaN."""
    e = np.ascontiguousarray(elems, dtype=np.uint8)
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    out = np.zeros((rows, cols), dtype=np.uint16)
    _check(lib().mxo_dequantize_mx(_ptr(e), _ptr(s), rows, cols, fmt, _ptr(out)), "dequantize_mx")
    return out


def dequantize_nvfp4(elems: np.ndarray, scales: np.ndarray, g: float, rows: int, cols: int) -> np.ndarray:
    e = np.ascontiguousarray(elems, dtype=np.uint8)
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    out = np.zeros((rows, cols), dtype=np.uint16)
    _check(lib().mxo_dequantize_nvfp4(_ptr(e), _ptr(s), ctypes.c_float(g), rows, cols, _ptr(out)),
           "dequantize_nvfp4")
    return out


# ---------------------------------------------------------------- tcgen05 scale tiling
def tcgen05_scale_bytes(rows: int, scale_cols: int) -> int:
    return lib().mxo_tcgen05_scale_bytes(rows, scale_cols)


def to_tcgen05_layout(scales_rowmajor: np.ndarray) -> np.ndarray:
    """Re-index a row-major scale matrix into the tcgen05 tiling (padding bytes zero)."""
    s = np.ascontiguousarray(scales_rowmajor, dtype=np.uint8)
    rows, scols = s.shape
    out = np.zeros(tcgen05_scale_bytes(rows, scols), dtype=np.uint8)
    _check(lib().mxo_to_tcgen05_layout(_ptr(s), rows, scols, _ptr(out)), "to_tcgen05_layout")
    return out


def from_tcgen05_layout(tiled: np.ndarray, rows: int, scale_cols: int) -> np.ndarray:
    """The row-major scale matrix held in a tcgen05-tiled buffer."""
    t = np.ascontiguousarray(tiled, dtype=np.uint8).reshape(-1)
    assert t.size >= tcgen05_scale_bytes(rows, scale_cols)
    out = np.zeros((rows, scale_cols), dtype=np.uint8)
    _check(lib().mxo_from_tcgen05_layout(_ptr(t), rows, scale_cols, _ptr(out)), "from_tcgen05_layout")
    return out


def tcgen05_offsets(rows: int, scale_cols: int) -> np.ndarray:
    """Offset of every (r, c) entry in the tcgen05 tiling, as a rows x scale_cols array."""
    L = lib()
    out = np.empty((rows, scale_cols), dtype=np.int64)
    for r in range(rows):
        for c in range(scale_cols):
            out[r, c] = L.mxo_tcgen05_scale_offset(r, c, rows, scale_cols)
    return out


# ---------------------------------------------------------------- matmul reference
def gemm_ref(a_elems, a_scales, a_fmt, b_elems, b_scales, b_fmt, M, N, K, pairs, a_g=1.0, b_g=1.0):
    """fp64 C[m, n] and sum_k |a b| for the requested (m, n) pairs (an array n x 2).
    a_g / b_g: the per-tensor scale of an NVFP4 operand (ignored for MX operands)."""
    pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
    c = np.zeros(pr.shape[0], dtype=np.float64)
    mag = np.zeros(pr.shape[0], dtype=np.float64)
    ae = np.ascontiguousarray(a_elems, dtype=np.uint8)
    as_ = np.ascontiguousarray(a_scales, dtype=np.uint8)
    be = np.ascontiguousarray(b_elems, dtype=np.uint8)
    bs = np.ascontiguousarray(b_scales, dtype=np.uint8)
    _check(lib().mxo_gemm_ref(_ptr(ae), _ptr(as_), a_fmt, ctypes.c_double(a_g), _ptr(be), _ptr(bs), b_fmt,
                              ctypes.c_double(b_g), M, N, K,
                              _ptr(pr), pr.shape[0], _ptr(c), _ptr(mag)), "gemm_ref")
    return c, mag


def gemm_ref_block(a_elems, a_scales, a_fmt, b_elems, b_scales, b_fmt, M, N, K, m0, m1, n0, n1, a_g=1.0, b_g=1.0):
    """fp64 C and sum_k |a b| for every entry of [m0, m1) x [n0, n1), as two arrays."""
    ae = np.ascontiguousarray(a_elems, dtype=np.uint8)
    as_ = np.ascontiguousarray(a_scales, dtype=np.uint8)
    be = np.ascontiguousarray(b_elems, dtype=np.uint8)
    bs = np.ascontiguousarray(b_scales, dtype=np.uint8)
    c = np.zeros((m1 - m0, n1 - n0), dtype=np.float64)
    mag = np.zeros_like(c)
    ar = np.zeros((m1 - m0, K), dtype=np.float64)
    br = np.zeros((n1 - n0, K), dtype=np.float64)
    _check(lib().mxo_gemm_ref_block(_ptr(ae), _ptr(as_), a_fmt, ctypes.c_double(a_g), _ptr(be), _ptr(bs), b_fmt,
                                    ctypes.c_double(b_g), M, N, K, m0, m1, n0, n1, _ptr(c), _ptr(mag), _ptr(ar),
                                    _ptr(br)), "gemm_ref_block")
    return c, mag


def mxfp4_to_fp8_blocks(elems: np.ndarray, scales: np.ndarray, rows: int, cols: int):
    """MXFP4 (packed E2M1, row-major E8M0 per 32) -> E4M3 codes rows x cols, one fp32 scale
    and one exactness flag per 128 x 128 block (the nested blocks of the pages)."""
    e = np.ascontiguousarray(elems, dtype=np.uint8)
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    out = np.zeros((rows, cols), dtype=np.uint8)
    bs = np.zeros((rows // 128, cols // 128), dtype=np.float32)
    ok = np.zeros((rows // 128, cols // 128), dtype=np.uint8)
    _check(lib().mxo_mxfp4_to_fp8_blocks(_ptr(e), _ptr(s), rows, cols, _ptr(out), _ptr(bs), _ptr(ok)),
           "mxfp4_to_fp8_blocks")
    return out, bs, ok


def rht16(x_bf16_bits: np.ndarray, sign_mask: int) -> np.ndarray:
    """16 x 16 random Hadamard transform of every 16 consecutive elements of each row
    (H16 D x / 4, fp32 butterflies, bf16 result), as bf16 bits."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    out = np.zeros_like(x)
    _check(lib().mxo_rht16(_ptr(x), x.shape[0], x.shape[1], sign_mask, _ptr(out)), "rht16")
    return out


def quantize_mx_sr(x_bf16_bits: np.ndarray, fmt: int, rounding: int, rnd: np.ndarray):
    """Row-wise MX quantisation with stochastic rounding (one random byte per element)."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    r = np.ascontiguousarray(rnd, dtype=np.uint8)
    assert r.shape == x.shape
    rows, cols = x.shape
    elems = np.zeros((rows, elem_bytes(cols, fmt)), dtype=np.uint8)
    scales = np.zeros((rows, cols // 32), dtype=np.uint8)
    _check(lib().mxo_quantize_mx_sr(_ptr(x), rows, cols, fmt, rounding, _ptr(r), _ptr(elems), _ptr(scales)),
           "quantize_mx_sr")
    return elems, scales


def quantize_nvfp4_sr(x_bf16_bits: np.ndarray, rnd: np.ndarray):
    """NVFP4 with stochastic rounding of the element cast (one random byte per element)."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    r = np.ascontiguousarray(rnd, dtype=np.uint8)
    assert r.shape == x.shape
    rows, cols = x.shape
    elems = np.zeros((rows, cols // 2), dtype=np.uint8)
    scales = np.zeros((rows, cols // 16), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    _check(lib().mxo_quantize_nvfp4_sr(_ptr(x), rows, cols, _ptr(r), _ptr(elems), _ptr(scales), _ptr(g)),
           "quantize_nvfp4_sr")
    return elems, scales, float(g[0])
