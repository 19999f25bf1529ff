"""Pins of the oracle's stochastic rounding of the element cast ([Q] §4: gradients are
rounded stochastically in the 4-bit recipe), no GPU.

Independent references: the E2M1 / E4M3 value tables of ml_dtypes and torch (for the two
neighbours of every value) and exact rational means over all 256 random bytes."""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import synth
from conftest import f32_to_bf16_bits
from test_oracle_formats import bf16_bits_to_f64, unpack_fp4

E2M1_GRID = np.unique(np.abs(np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)))
E4M3_GRID = np.unique(np.abs(torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()))
E4M3_GRID = E4M3_GRID[np.isfinite(E4M3_GRID)]


def e2m1_block(values):
    """A 32-block whose first entry (6.0) fixes the floor-rule scale at 2^0, so the scaled
    values are the values themselves."""
    x = np.zeros(32, dtype=np.float32)
    x[0] = 6.0
    x[1:1 + len(values)] = values
    return f32_to_bf16_bits(x).reshape(1, 32)


def sr_e2m1(oracle, values, r):
    """SR codes of `values` (at most 31) with random byte r for all of them."""
    x = e2m1_block(values)
    rnd = np.full((1, 32), r, dtype=np.uint8)
    e, s = oracle.quantize_mx_sr(x, oracle.E2M1, oracle.FLOOR, rnd)
    assert s[0, 0] == 127
    codes = unpack_fp4(e[0], 32)[1:1 + len(values)]
    return codes.astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)


def test_sr_results_are_the_two_neighbours_and_unbiased(oracle):
    """Every positive bf16 value below 6 rounds to one of its two E2M1 neighbours (from
    ml_dtypes' table); over the 256 random bytes the mean is the value itself to within
    1/256 of the step, and larger bytes never round up where smaller ones round down."""
    b = np.arange(0x3C00, 0x40C0, 7, dtype=np.uint32).astype(np.uint16)     # 2^-7 .. 6
    vals = bf16_bits_to_f64(b)
    vals = vals[vals < 6.0]
    for chunk in range(0, len(vals), 31):
        v = vals[chunk:chunk + 31]
        res = np.stack([sr_e2m1(oracle, v.astype(np.float32), r) for r in range(256)])   # 256 x n
        for j, y in enumerate(v):
            lo = E2M1_GRID[E2M1_GRID <= y].max()
            hi = E2M1_GRID[E2M1_GRID > y].min()
            col = res[:, j]
            if y == lo:
                assert np.all(col == lo)
                continue
            assert set(np.unique(col)) <= {lo, hi}
            ups = col == hi
            assert not np.any(ups[1:] & ~ups[:-1])                   # monotone in r
            mean = sum(Fraction(float(c)) for c in col) / 256
            assert abs(mean - Fraction(float(y))) <= Fraction(float(hi - lo)) / 256


def test_sr_saturates_and_keeps_sign(oracle):
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 0] = 6.0
    x[0, 1] = -5.75
    x[0, 2] = -2.0 ** -10
    bits = f32_to_bf16_bits(x).reshape(1, 32)
    for r in (0, 128, 255):
        e, s = oracle.quantize_mx_sr(bits, oracle.E2M1, oracle.FLOOR, np.full((1, 32), r, dtype=np.uint8))
        c = unpack_fp4(e[0], 32)
        assert c[0] == 0x7 and c[1] in (0xE, 0xF) and c[2] in (0x8, 0x9)   # sign bit kept
    # r = 0 rounds every non-representable magnitude up; r = 255 keeps it down unless the
    # fraction exceeds 255/256
    e0, _ = oracle.quantize_mx_sr(bits, oracle.E2M1, oracle.FLOOR, np.zeros((1, 32), dtype=np.uint8))
    assert unpack_fp4(e0[0], 32)[1] == 0xF and unpack_fp4(e0[0], 32)[2] == 0x9


@pytest.mark.parametrize("fmt", ["E4M3", "E5M2", "E2M1"])
def test_sr_scales_equal_rne_and_codes_neighbour_rne(oracle, fmt):
    """The shared scale does not depend on the rounding of the elements; every SR code is
    the RNE code or its neighbour in magnitude."""
    f = getattr(oracle, fmt)
    x = synth.gradients(32, 256, seed=5)
    rnd = np.random.default_rng(6).integers(0, 256, size=x.shape, dtype=np.uint8)
    e_sr, s_sr = oracle.quantize_mx_sr(x, f, oracle.CEIL, rnd)
    e_rn, s_rn = oracle.quantize_mx(x, f, oracle.ROW, oracle.CEIL)
    assert np.array_equal(s_sr, s_rn)
    if fmt == "E2M1":
        a = np.stack([unpack_fp4(r, 256) for r in e_sr]).astype(np.int64)
        b = np.stack([unpack_fp4(r, 256) for r in e_rn]).astype(np.int64)
        mag = 0x7
    else:
        a, b, mag = e_sr.astype(np.int64), e_rn.astype(np.int64), 0x7F
    same_sign = ((a ^ b) & ~mag) == 0
    zero = ((a | b) & mag) == 0
    assert np.all(same_sign | zero)
    assert np.all(np.abs((a & mag) - (b & mag)) <= 1)


def test_nvfp4_sr_keeps_scales_and_neighbours(oracle):
    x = synth.weight_fp4(16, 128, seed=9)
    rnd = np.random.default_rng(10).integers(0, 256, size=x.shape, dtype=np.uint8)
    e_sr, s_sr, g_sr = oracle.quantize_nvfp4_sr(x, rnd)
    e_rn, s_rn, g_rn = oracle.quantize_nvfp4(x)
    assert g_sr == g_rn and np.array_equal(s_sr, s_rn)
    a = np.stack([unpack_fp4(r, 128) for r in e_sr]).astype(np.int64)
    b = np.stack([unpack_fp4(r, 128) for r in e_rn]).astype(np.int64)
    assert np.all(np.abs((a & 7) - (b & 7)) <= 1)
    assert not np.array_equal(a, b)                      # some elements did round the other way
