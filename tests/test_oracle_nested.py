"""Pins of the oracle's nested-block conversion (MXFP4 1 x 32 tiles inside FP8 128 x 128
blocks, the DeepSeek-V4 arrangement of "MXFP4 と NVFP4 は何が違うのか調べてみた" §6), no GPU.

Independent references: ml_dtypes' float4_e2m1fn and torch's float8_e4m3fn decoders, exact
powers of two, and hand-built tiles at the edges of the exactness condition."""
import ml_dtypes
import numpy as np
import pytest
import torch

import synth
from conftest import f32_to_bf16_bits, read_golden


def fp4_values(elems, scales, rows, cols):
    p = np.asarray(elems, dtype=np.uint8)
    codes = np.empty((rows, cols), dtype=np.uint8)
    codes[:, 0::2] = p & 0xF
    codes[:, 1::2] = p >> 4
    v = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    s = np.repeat(scales.astype(np.int64), 32, axis=1)
    with np.errstate(invalid="ignore"):
        out = np.ldexp(v, s - 127)
    out[s == 255] = np.nan
    return out


def fp8_values(codes, block_scale):
    v = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()
    return v * np.kron(block_scale.astype(np.float64), np.ones((128, 128)))


def test_block_geometry_matches_page(oracle):
    g = read_golden("format_constants.txt")
    br, bc = (int(x) for x in g["fp8_block"])
    assert br * bc // 32 == int(g["nested_subblocks_per_fp8_block"][0]) == 4 * 128
    x = synth.weight_fp4(256, 384, seed=7)
    e, s = oracle.quantize_mx(x, oracle.E2M1, oracle.ROW, oracle.FLOOR)
    out, bs, ok = oracle.mxfp4_to_fp8_blocks(e, s, 256, 384)
    assert out.shape == (256, 384) and bs.shape == ok.shape == (256 // br, 384 // bc)


def test_weights_convert_losslessly(oracle):
    """Trained-weight-like tensors satisfy the condition; then FP8 x block scale decodes to
    exactly the FP4 values, element by element."""
    x = synth.weight_fp4(256, 512, seed=8)
    e, s = oracle.quantize_mx(x, oracle.E2M1, oracle.ROW, oracle.FLOOR)
    out, bs, ok = oracle.mxfp4_to_fp8_blocks(e, s, 256, 512)
    assert np.all(ok == 1)
    assert np.array_equal(fp8_values(out, bs), fp4_values(e, s, 256, 512))
    assert np.all(np.log2(bs) == np.round(np.log2(bs)))          # powers of two


def tile(low_exp_gap, low_value, high_value=6.0):
    """One 128 x 128 block: sub-block (0, 0) holds high_value at scale 2^0, sub-block (5, 1)
    holds low_value at scale 2^-gap, everything else zero."""
    x = np.zeros((128, 128), dtype=np.float32)
    x[0, 0] = high_value
    x[5, 32] = low_value * 2.0 ** -low_exp_gap
    return f32_to_bf16_bits(x).reshape(128, 128)


@pytest.mark.parametrize("gap,low,exact", [(14, 0.5, 1), (15, 0.5, 0), (15, 1.0, 1), (16, 1.0, 0),
                                           (13, 1.5, 1), (15, 1.5, 0), (14, 3.0, 1), (0, 0.5, 1)])
def test_exactness_edges(oracle, gap, low, exact):
    """With S = 2^(s_max - 6) the smallest E4M3 step 2^-9 decides: 0.5 survives a scale gap of
    14 (2^-9) but not 15; 1.0 survives 15; 1.5 needs a gap <= 14."""
    x = tile(gap, low)
    e, s = oracle.quantize_mx(x, oracle.E2M1, oracle.ROW, oracle.FLOOR)
    out, bs, ok = oracle.mxfp4_to_fp8_blocks(e, s, 128, 128)
    assert int(ok[0, 0]) == exact
    same = fp8_values(out, bs) == fp4_values(e, s, 128, 128)
    assert bool(np.all(same)) == bool(exact)
    # the largest FP4 value, 6 x 2^s_max, maps to 384 = 1.5 x 2^8 (E4M3 code 0x7C)
    assert out[0, 0] == 0x7C and bs[0, 0] == 2.0 ** (int(s[0, 0]) - 127 - 6)


def test_nan_and_empty_blocks(oracle):
    x = np.zeros((128, 256), dtype=np.uint16)
    x[3, 7] = 0x7FC0                                 # NaN in sub-block (3, 0) of block 0
    x[4, 10] = f32_to_bf16_bits([2.0])[0]
    e, s = oracle.quantize_mx(x, oracle.E2M1, oracle.ROW, oracle.FLOOR)
    out, bs, ok = oracle.mxfp4_to_fp8_blocks(e, s, 128, 256)
    assert s[3, 0] == 0xFF and np.all(out[3, :32] == 0x7F)
    assert ok[0, 0] == 1 and bs[0, 0] == 2.0 ** (int(s[4, 0]) - 127 - 6)   # the NaN block is not the max
    assert ok[0, 1] == 1 and bs[0, 1] == 1.0 and np.all(out[:, 128:] == 0)  # all-zero block: S = 1
