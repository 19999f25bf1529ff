"""Torch-facing wrappers over the C ABI: allocate outputs with torch (device memory),
pass raw pointers and the current CUDA stream, check the status.  No arithmetic of the
method happens here; every step runs in the CUDA kernels behind libmx.so.
"""
from __future__ import annotations

from typing import NamedTuple, Optional

import torch

from . import _lib as L

FMTS = {"e4m3": L.MX_FMT_E4M3, "e5m2": L.MX_FMT_E5M2, "e2m1": L.MX_FMT_E2M1, "nvfp4": L.MX_FMT_NVFP4,
        "e2m3": L.MX_FMT_E2M3, "e3m2": L.MX_FMT_E3M2, "int8": L.MX_FMT_INT8}
ROUNDING = {"floor": L.MX_SCALE_FLOOR_OCP, "ceil": L.MX_SCALE_CEIL_RECIPE}
LAYOUTS = {"rowmajor": L.MX_LAYOUT_ROWMAJOR, "tcgen05": L.MX_LAYOUT_TCGEN05,
           "both": L.MX_LAYOUT_ROWMAJOR | L.MX_LAYOUT_TCGEN05}


def _fmt(f) -> int:
    return FMTS[f] if isinstance(f, str) else int(f)


def block_of(fmt) -> int:
    return 16 if _fmt(fmt) == L.MX_FMT_NVFP4 else 32


def is_fp4(fmt) -> bool:
    return _fmt(fmt) in (L.MX_FMT_E2M1, L.MX_FMT_NVFP4)


def code_bits(fmt) -> int:
    """Stored width of one element code: codes are packed densely along a row (FP4 two per
    byte, FP6 four per three bytes, FP8 / INT8 one per byte)."""
    f = _fmt(fmt)
    return 4 if is_fp4(f) else 6 if f in (L.MX_FMT_E2M3, L.MX_FMT_E3M2) else 8


def elem_bytes(rows: int, cols: int, fmt) -> int:
    return rows * cols * code_bits(fmt) // 8


def scale_bytes(rows: int, scale_cols: int, layout) -> int:
    lay = LAYOUTS[layout] if isinstance(layout, str) else int(layout)
    n = L.lib.mx_scale_bytes(rows, scale_cols, lay)
    if n < 0:
        raise ValueError("invalid scale layout")
    return n


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _check_src(x: torch.Tensor):
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous() or x.dim() != 2:
        raise ValueError("expected a contiguous 2-D bf16 CUDA tensor")


class Quantized(NamedTuple):
    elems: torch.Tensor          # uint8 codes, packed densely (FP4 two per byte, even index low; FP6 four per three bytes)
    scales: torch.Tensor         # uint8 scales in the first layout
    scales_alt: Optional[torch.Tensor]   # tcgen05 scales when layout == "both"
    global_scale: Optional[torch.Tensor]  # NVFP4 fp32 g
    rows: int                    # shape of the quantised (possibly transposed) matrix
    cols: int
    fmt: int


def _buf(out: Optional[torch.Tensor], n: int, dtype, dev, what: str) -> torch.Tensor:
    """A caller-provided output (checked for size, type and device) or a new one."""
    if out is None:
        return torch.empty(n, dtype=dtype, device=dev)
    if out.dtype != dtype or out.device != dev or not out.is_contiguous() or out.numel() < n:
        raise ValueError(f"output buffer '{what}' must be a contiguous {dtype} tensor of >= {n} elements on {dev}")
    return out


def quantize(x: torch.Tensor, fmt="e4m3", axis: str = "row", rounding: str = "ceil",
             layout: str = "rowmajor", stream=None, out: Optional[Quantized] = None) -> Quantized:
    """Block-scaled quantisation of a bf16 matrix.  `out` (a Quantized from an earlier
    call with the same arguments) reuses its buffers instead of allocating new ones."""
    _check_src(x)
    f = _fmt(fmt)
    rows, cols = x.shape
    orows, ocols = (rows, cols) if axis == "row" else (cols, rows)
    B = block_of(f)
    dev = x.device
    lay = LAYOUTS[layout]
    first = "rowmajor" if layout in ("rowmajor", "both") else "tcgen05"
    elems = _buf(out and out.elems, elem_bytes(orows, ocols, f), torch.uint8, dev, "elems")
    scales = _buf(out and out.scales, scale_bytes(orows, ocols // B, first), torch.uint8, dev, "scales")
    alt = _buf(out and out.scales_alt, scale_bytes(orows, ocols // B, "tcgen05"), torch.uint8, dev, "scales_alt") \
        if layout == "both" else None
    g = _buf(out and out.global_scale, 1, torch.float32, dev, "global_scale") if f == L.MX_FMT_NVFP4 else None
    st = L.lib.mx_quantize(x.data_ptr(), rows, cols, f, L.MX_AXIS_ROW if axis == "row" else L.MX_AXIS_COL,
                           ROUNDING[rounding], elems.data_ptr(), scales.data_ptr(), lay, _ptr(alt), _ptr(g),
                           _stream(stream))
    L.check(st, "mx_quantize")
    return Quantized(elems, scales, alt, g, orows, ocols, f)


def quantize_train(x: torch.Tensor, fmt="e2m1", rounding: str = "floor", rht_signs: Optional[int] = None,
                   sr_random: Optional[torch.Tensor] = None, layout: str = "tcgen05", stream=None) -> Quantized:
    """Row-wise quantisation with an optional 16 x 16 random Hadamard transform (rht_signs:
    the 16-bit sign mask; None for no transform) and optional stochastic rounding
    (sr_random: a uint8 tensor of x's shape; None for round-to-nearest-even)."""
    _check_src(x)
    f = _fmt(fmt)
    rows, cols = x.shape
    dev = x.device
    B = block_of(f)
    first = "rowmajor" if layout in ("rowmajor", "both") else "tcgen05"
    elems = torch.empty(elem_bytes(rows, cols, f), dtype=torch.uint8, device=dev)
    scales = torch.empty(scale_bytes(rows, cols // B, first), dtype=torch.uint8, device=dev)
    alt = torch.empty(scale_bytes(rows, cols // B, "tcgen05"), dtype=torch.uint8, device=dev) \
        if layout == "both" else None
    g = torch.empty(1, dtype=torch.float32, device=dev) if f == L.MX_FMT_NVFP4 else None
    if sr_random is not None and (sr_random.dtype != torch.uint8 or sr_random.numel() != rows * cols
                                  or not sr_random.is_contiguous() or sr_random.device != dev):
        raise ValueError("sr_random must be a contiguous uint8 tensor with one byte per element")
    L.check(L.lib.mx_quantize_train(x.data_ptr(), rows, cols, f, ROUNDING[rounding], 0 if rht_signs is None else 1,
                                    0 if rht_signs is None else int(rht_signs) & 0xFFFF, _ptr(sr_random),
                                    elems.data_ptr(), scales.data_ptr(), LAYOUTS[layout], _ptr(alt), _ptr(g),
                                    _stream(stream)), "mx_quantize_train")
    return Quantized(elems, scales, alt, g, rows, cols, f)


def quantize_mx_nvfp4(x: torch.Tensor, fmt="e2m1", rounding: str = "floor", layout: str = "both",
                      nv_layout: str = "both", stream=None):
    """Row-wise MX quantisation (any MX format) and NVFP4 quantisation of the same tensor in
    one call, reading its maximum once (the MX pass also yields the NVFP4 tensor maximum).
    Returns (mx Quantized, nvfp4 Quantized), bit-identical to two quantize() calls."""
    _check_src(x)
    f = _fmt(fmt)
    rows, cols = x.shape
    dev = x.device

    def outs(fm, B, lay):
        first = "rowmajor" if lay in ("rowmajor", "both") else "tcgen05"
        e = torch.empty(elem_bytes(rows, cols, fm), dtype=torch.uint8, device=dev)
        sc = torch.empty(scale_bytes(rows, cols // B, first), dtype=torch.uint8, device=dev)
        alt = torch.empty(scale_bytes(rows, cols // B, "tcgen05"), dtype=torch.uint8, device=dev) \
            if lay == "both" else None
        return e, sc, alt

    me, ms, ma = outs(f, 32, layout)
    ne, ns, na = outs(L.MX_FMT_NVFP4, 16, nv_layout)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    L.check(L.lib.mx_quantize_mx_nvfp4(x.data_ptr(), rows, cols, f, ROUNDING[rounding], me.data_ptr(), ms.data_ptr(),
                                       LAYOUTS[layout], _ptr(ma), ne.data_ptr(), ns.data_ptr(), LAYOUTS[nv_layout],
                                       _ptr(na), g.data_ptr(), _stream(stream)), "mx_quantize_mx_nvfp4")
    return (Quantized(me, ms, ma, None, rows, cols, f), Quantized(ne, ns, na, g, rows, cols, L.MX_FMT_NVFP4))


def quantize_nvfp4_2d(x: torch.Tensor, layout: str = "tcgen05", stream=None) -> Quantized:
    """NVFP4 with 16 x 16 weight blocks (scales repeated on the 16 rows of each block)."""
    _check_src(x)
    rows, cols = x.shape
    dev = x.device
    first = "rowmajor" if layout in ("rowmajor", "both") else "tcgen05"
    elems = torch.empty(rows * cols // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(scale_bytes(rows, cols // 16, first), dtype=torch.uint8, device=dev)
    alt = torch.empty(scale_bytes(rows, cols // 16, "tcgen05"), dtype=torch.uint8, device=dev) \
        if layout == "both" else None
    g = torch.empty(1, dtype=torch.float32, device=dev)
    L.check(L.lib.mx_quantize_nvfp4_2d(x.data_ptr(), rows, cols, elems.data_ptr(), scales.data_ptr(),
                                       LAYOUTS[layout], _ptr(alt), g.data_ptr(), _stream(stream)),
            "mx_quantize_nvfp4_2d")
    return Quantized(elems, scales, alt, g, rows, cols, L.MX_FMT_NVFP4)


def quantize_dual(x: torch.Tensor, fmt="e4m3", rounding: str = "ceil", layout: str = "tcgen05", stream=None,
                  out: Optional[tuple] = None):
    """Row-wise and column-wise (transposed) quantisation from one read of x.  `out` (the
    pair returned by an earlier call with the same arguments) reuses its buffers."""
    _check_src(x)
    f = _fmt(fmt)
    rows, cols = x.shape
    dev = x.device
    o_r, o_c = out if out is not None else (None, None)
    first = "rowmajor" if layout in ("rowmajor", "both") else "tcgen05"
    re = _buf(o_r and o_r.elems, elem_bytes(rows, cols, f), torch.uint8, dev, "row elems")
    ce = _buf(o_c and o_c.elems, elem_bytes(rows, cols, f), torch.uint8, dev, "col elems")
    rs = _buf(o_r and o_r.scales, scale_bytes(rows, cols // 32, first), torch.uint8, dev, "row scales")
    cs = _buf(o_c and o_c.scales, scale_bytes(cols, rows // 32, first), torch.uint8, dev, "col scales")
    ra = ca = None
    if layout == "both":
        ra = _buf(o_r and o_r.scales_alt, scale_bytes(rows, cols // 32, "tcgen05"), torch.uint8, dev, "row scales_alt")
        ca = _buf(o_c and o_c.scales_alt, scale_bytes(cols, rows // 32, "tcgen05"), torch.uint8, dev, "col scales_alt")
    st = L.lib.mx_quantize_dual(x.data_ptr(), rows, cols, f, ROUNDING[rounding], re.data_ptr(), rs.data_ptr(),
                                ce.data_ptr(), cs.data_ptr(), LAYOUTS[layout], _ptr(ra), _ptr(ca), _stream(stream))
    L.check(st, "mx_quantize_dual")
    return (Quantized(re, rs, ra, None, rows, cols, f), Quantized(ce, cs, ca, None, cols, rows, f))


def dequantize(q: Quantized, layout: str = "rowmajor", stream=None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Codes and scales back to a (rows, cols) bf16 matrix (into `out` when given)."""
    scales = q.scales if (layout == "rowmajor" or q.scales_alt is None) else q.scales_alt
    out = _buf(out, q.rows * q.cols, torch.bfloat16, q.elems.device, "out").reshape(-1)[:q.rows * q.cols] \
        .view(q.rows, q.cols) if out is not None else torch.empty((q.rows, q.cols), dtype=torch.bfloat16, device=q.elems.device)
    st = L.lib.mx_dequantize(q.elems.data_ptr(), scales.data_ptr(), _ptr(q.global_scale), q.rows, q.cols, q.fmt,
                             LAYOUTS[layout], out.data_ptr(), _stream(stream))
    L.check(st, "mx_dequantize")
    return out


def cast(x: torch.Tensor, fmt="e4m3", stream=None) -> torch.Tensor:
    """Direct cast with no block scale (codes, FP4 packed two per byte)."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("expected a contiguous bf16 CUDA tensor")
    f = _fmt(fmt)
    out = torch.empty(elem_bytes(1, x.numel(), f), dtype=torch.uint8, device=x.device)
    L.check(L.lib.mx_cast(x.data_ptr(), x.numel(), f, out.data_ptr(), _stream(stream)), "mx_cast")
    return out


def gemm(a: Quantized, b: Quantized, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """C = A * B^T for A (M x K) and B (N x K) quantised row-wise with tcgen05 scales:
    FP8 / FP6 (E4M3, E5M2, E2M3, E3M2) x FP8 / FP6 / E2M1, E2M1 x E2M1, or NVFP4 x NVFP4
    (whose per-tensor scales are applied to the fp32 sum)."""
    M, K = a.rows, a.cols
    N = b.rows
    if b.cols != K:
        raise ValueError("K mismatch")
    sa = a.scales_alt if a.scales_alt is not None else a.scales
    sb = b.scales_alt if b.scales_alt is not None else b.scales
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.elems.device)
    A = L.MxOperand(a.elems.data_ptr(), sa.data_ptr(), a.fmt, _ptr(a.global_scale))
    B = L.MxOperand(b.elems.data_ptr(), sb.data_ptr(), b.fmt, _ptr(b.global_scale))
    L.check(L.lib.mx_gemm(A, B, out.data_ptr(), M, N, K, _stream(stream)), "mx_gemm")
    return out


def watchdog_status(clear: bool = True) -> int:
    import ctypes
    code = ctypes.c_int(0)
    st = L.lib.mx_watchdog_status(ctypes.byref(code), 1 if clear else 0)
    if st not in (L.MX_OK, L.MX_ERR_TIMEOUT):
        L.check(st, "mx_watchdog_status")
    return code.value
