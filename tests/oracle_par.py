"""Row-slab parallel drivers of the oracle for full-size parity checks (test helpers).

The oracle's functions run one plain loop per block; quantisation blocks are independent,
so a large tensor is split into slabs of whole blocks and each slab goes to the oracle in
its own thread (ctypes releases the interpreter lock during the call).  Nothing here does
any of the method's arithmetic: it only slices inputs and places the oracle's outputs.
"""
from __future__ import annotations

import concurrent.futures as cf
import os

import numpy as np

WORKERS = max(1, min(64, os.cpu_count() or 1))


def quantize_mx_both(oracle, x, fmt, rounding, slab=512):
    """Row-wise and column-wise MX quantisation of x (rows x cols bf16 bits):
    (row_elems rows x bytes(cols), row_scales rows x cols/32,
     col_elems cols x bytes(rows), col_scales cols x rows/32).  Slabs of `slab` rows
    (a multiple of 32)."""
    R, C = x.shape
    assert slab % 32 == 0 and R % 32 == 0
    bits = oracle.code_bits(fmt)
    re_ = np.zeros((R, C * bits // 8), dtype=np.uint8)
    rs = np.zeros((R, C // 32), dtype=np.uint8)
    ce = np.zeros((C, R * bits // 8), dtype=np.uint8)
    cs = np.zeros((C, R // 32), dtype=np.uint8)

    def work(r0):
        r1 = min(R, r0 + slab)
        xs = np.ascontiguousarray(x[r0:r1])
        e, s = oracle.quantize_mx(xs, fmt, oracle.ROW, rounding)
        re_[r0:r1], rs[r0:r1] = e, s
        e, s = oracle.quantize_mx(xs, fmt, oracle.COL, rounding)
        assert (r0 * bits) % 8 == 0
        ce[:, r0 * bits // 8:r1 * bits // 8] = e
        cs[:, r0 // 32:r1 // 32] = s

    with cf.ThreadPoolExecutor(WORKERS) as ex:
        list(ex.map(work, range(0, R, slab)))
    return re_, rs, ce, cs


def quantize_mx_rows(oracle, x, fmt, rounding, slab=512):
    """Row-wise MX quantisation only: (elems, scales)."""
    R, C = x.shape
    bits = oracle.code_bits(fmt)
    re_ = np.zeros((R, C * bits // 8), dtype=np.uint8)
    rs = np.zeros((R, C // 32), dtype=np.uint8)

    def work(r0):
        r1 = min(R, r0 + slab)
        re_[r0:r1], rs[r0:r1] = oracle.quantize_mx(np.ascontiguousarray(x[r0:r1]), fmt, oracle.ROW, rounding)

    with cf.ThreadPoolExecutor(WORKERS) as ex:
        list(ex.map(work, range(0, R, slab)))
    return re_, rs


def gemm_ref_pairs(oracle, ae, as_, a_fmt, be, bs, b_fmt, M, N, K, pairs, chunk=256):
    """oracle.gemm_ref over many (m, n) pairs, in chunks on threads."""
    pairs = np.ascontiguousarray(pairs, dtype=np.int64)
    c = np.zeros(len(pairs))
    mag = np.zeros(len(pairs))

    def work(i0):
        i1 = min(len(pairs), i0 + chunk)
        c[i0:i1], mag[i0:i1] = oracle.gemm_ref(ae, as_, a_fmt, be, bs, b_fmt, M, N, K, pairs[i0:i1])

    with cf.ThreadPoolExecutor(WORKERS) as ex:
        list(ex.map(work, range(0, len(pairs), chunk)))
    return c, mag


def gemm_ref_tile(oracle, ae, as_, a_fmt, be, bs, b_fmt, M, N, K, m0, m1, n0, n1, rows_per_task=16):
    """oracle.gemm_ref_block over [m0, m1) x [n0, n1), split by rows over threads."""
    c = np.zeros((m1 - m0, n1 - n0))
    mag = np.zeros_like(c)

    def work(r0):
        r1 = min(m1, r0 + rows_per_task)
        c[r0 - m0:r1 - m0], mag[r0 - m0:r1 - m0] = oracle.gemm_ref_block(ae, as_, a_fmt, be, bs, b_fmt, M, N, K,
                                                                         r0, r1, n0, n1)

    with cf.ThreadPoolExecutor(WORKERS) as ex:
        list(ex.map(work, range(m0, m1, rows_per_task)))
    return c, mag


def rht16_rows(oracle, x, signs, slab=512):
    """The oracle's 16 x 16 transform of every row group of x, slab by slab."""
    R, C = x.shape
    out = np.empty_like(x)

    def work(r0):
        r1 = min(R, r0 + slab)
        out[r0:r1] = oracle.rht16(np.ascontiguousarray(x[r0:r1]), signs)

    with cf.ThreadPoolExecutor(WORKERS) as ex:
        list(ex.map(work, range(0, R, slab)))
    return out


def quantize_mx_sr_rows(oracle, x, fmt, rounding, rnd, slab=512):
    """Row-wise MX quantisation with stochastic rounding (rnd: one byte per element)."""
    R, C = x.shape
    bits = oracle.code_bits(fmt)
    re_ = np.zeros((R, C * bits // 8), dtype=np.uint8)
    rs = np.zeros((R, C // 32), dtype=np.uint8)

    def work(r0):
        r1 = min(R, r0 + slab)
        re_[r0:r1], rs[r0:r1] = oracle.quantize_mx_sr(np.ascontiguousarray(x[r0:r1]), fmt, rounding,
                                                      np.ascontiguousarray(rnd[r0:r1]))

    with cf.ThreadPoolExecutor(WORKERS) as ex:
        list(ex.map(work, range(0, R, slab)))
    return re_, rs


def quantize_nvfp4_sr_rows(oracle, x, rnd, slab=512):
    """NVFP4 with stochastic rounding of the whole tensor, slab by slab.  The per-tensor
    scale depends on the tensor's largest finite magnitude, so every slab goes to the
    oracle together with one row that holds that maximum (appended after the slab; its
    outputs are dropped): the oracle then derives the tensor's own scale for each slab.
    Returns (elems rows x cols/2, scales rows x cols/16, g)."""
    R, C = x.shape
    mag = (x & 0x7FFF).astype(np.uint16)
    finite = mag < 0x7F80
    r_max = int(np.argmax(np.where(finite, mag, 0).max(axis=1)))
    extra = np.ascontiguousarray(x[r_max:r_max + 1])
    extra_rnd = np.zeros((1, C), dtype=np.uint8)
    re_ = np.zeros((R, C // 2), dtype=np.uint8)
    rs = np.zeros((R, C // 16), dtype=np.uint8)
    gs = {}

    def work(r0):
        r1 = min(R, r0 + slab)
        xs = np.concatenate([x[r0:r1], extra])
        rn = np.concatenate([rnd[r0:r1], extra_rnd])
        e, s, g = oracle.quantize_nvfp4_sr(np.ascontiguousarray(xs), np.ascontiguousarray(rn))
        re_[r0:r1], rs[r0:r1] = e[:r1 - r0], s[:r1 - r0]
        gs[r0] = g

    with cf.ThreadPoolExecutor(WORKERS) as ex:
        list(ex.map(work, range(0, R, slab)))
    g_all = set(gs.values())
    assert len(g_all) == 1
    return re_, rs, g_all.pop()
