"""Pins of the oracle's block operations: the worked example, effective bits, NaN
scales, landing of real blocks, dequantisation, NVFP4 invariants, the fp64 matmul
reference and the scale tiling (no GPU)."""
import math
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import synth
from conftest import f32_to_bf16_bits, read_golden, unpack_codes
from test_oracle_formats import bf16_bits_to_f64, unpack_fp4


def e2m1_values(codes):
    return np.asarray(codes, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)


# ------------------------------------------------------------------ worked example
def test_worked_example_direct_cast(oracle):
    g = read_golden("p4_worked_example.txt")
    x = f32_to_bf16_bits(g["input"])
    got = e2m1_values(unpack_fp4(oracle.cast(x, oracle.E2M1), 4))
    page = list(g["direct_cast_page"])
    idx, rne = g["direct_cast_tie_rne"]
    for i in range(4):
        if i == int(idx):
            assert got[i] == rne and page[i] != rne   # recorded discrepancy (tie)
        else:
            assert got[i] == page[i]


@pytest.mark.parametrize("rounding", [0, 1])
def test_worked_example_shared_scale(oracle, rounding):
    g = read_golden("p4_worked_example.txt")
    block = np.zeros((1, 32), dtype=np.uint16)          # a 32-block; the rest are zeros
    block[0, :4] = f32_to_bf16_bits(g["input"])
    elems, scales = oracle.quantize_mx(block, oracle.E2M1, oracle.ROW, rounding)
    assert int(scales[0, 0]) - 127 == int(g["shared_scale_exponent"][0])
    got = e2m1_values(unpack_fp4(elems[0], 32))[:4]
    page = list(g["scaled_cast_page"])
    idx, rne = g["scaled_cast_tie_rne"]
    for i in range(4):
        if i == int(idx):
            assert got[i] == rne and page[i] != rne
        else:
            assert got[i] == page[i]
    assert np.all(e2m1_values(unpack_fp4(elems[0], 32))[4:] == 0)


# ------------------------------------------------------------------ effective bits
def test_effective_bits(oracle):
    g = read_golden("format_constants.txt")
    x = synth.normal(64, 256, seed=3)
    n = x.size
    e, s = oracle.quantize_mx(x, oracle.E2M1, oracle.ROW, oracle.FLOOR)
    assert (e.nbytes + s.nbytes) * 8 / n == g["bits_mxfp4"][0]
    for fmt in (oracle.E4M3, oracle.E5M2):
        e, s = oracle.quantize_mx(x, fmt, oracle.ROW, oracle.CEIL)
        assert (e.nbytes + s.nbytes) * 8 / n == g["bits_mxfp8"][0]
    e, s, _ = oracle.quantize_nvfp4(x)
    assert (e.nbytes + s.nbytes) * 8 / n == g["bits_nvfp4"][0]
    # MXFP6: 6-bit codes packed four per three bytes plus the shared scale
    for fmt in (oracle.E2M3, oracle.E3M2):
        e, s = oracle.quantize_mx(x, fmt, oracle.ROW, oracle.FLOOR)
        assert (e.nbytes + s.nbytes) * 8 / n == g["bits_mxfp6"][0]
    e, s = oracle.quantize_mx(x, oracle.INT8, oracle.ROW, oracle.FLOOR)
    assert (e.nbytes + s.nbytes) * 8 / n == g["bits_mxint8"][0]


# ------------------------------------------------------------------ block assembly
@pytest.mark.parametrize("fmt_name,rounding", [("E4M3", 1), ("E4M3", 0), ("E5M2", 1), ("E2M1", 0), ("E2M1", 1),
                                               ("E2M3", 0), ("E2M3", 1), ("E3M2", 0), ("E3M2", 1)])
def test_block_codes_are_the_cast_of_scaled_values(oracle, fmt_name, rounding):
    """Each block's codes equal the (brute-force-pinned) direct cast of x * 2^-s, with s
    read back from the E8M0 byte, and the scaled maximum lands per its school."""
    fmt = getattr(oracle, fmt_name)
    x = synth.mx8_rowwise(16, 128, seed=5)
    e, s = oracle.quantize_mx(x, fmt, oracle.ROW, rounding)
    maxv = {"E4M3": 448.0, "E5M2": 57344.0, "E2M1": 6.0, "E2M3": 7.5, "E3M2": 28.0}[fmt_name]
    xf = bf16_bits_to_f64(x)
    fp4 = fmt_name == "E2M1"
    fp6 = fmt_name in ("E2M3", "E3M2")
    for r in range(x.shape[0]):
        codes = unpack_fp4(e[r], 128) if fp4 else unpack_codes(e[r], 128, 6) if fp6 else e[r]
        for b in range(4):
            sc = int(s[r, b]) - 127
            blk = xf[r, 32 * b:32 * b + 32]
            scaled = np.ldexp(blk, -sc)
            ref = oracle.cast(f32_to_bf16_bits(scaled.astype(np.float32)), fmt) if np.all(
                (scaled.astype(np.float32).view(np.uint32) & 0xFFFF) == 0) else None
            assert ref is not None              # power-of-two scaling keeps bf16 exact here
            ref = unpack_fp4(ref, 32) if fp4 else unpack_codes(ref, 32, 6) if fp6 else ref
            assert np.array_equal(codes[32 * b:32 * b + 32], ref)
            top = np.abs(scaled).max()
            if rounding == 1:
                assert maxv / 2 < top <= maxv
            else:
                assert 2.0 ** {"E4M3": 8, "E5M2": 15, "E2M1": 2, "E2M3": 2, "E3M2": 4}[fmt_name] <= top


@pytest.mark.parametrize("rounding", [0, 1])
def test_int8_block_codes(oracle, rounding):
    """MXINT8 blocks: codes are the saturating RNE of x * 2^-s * 64 (the pinned element
    encoder) and the scaled maximum lands per its school ([1, 2) floor; (127/128, 127/64]
    no-clip)."""
    x = synth.mx8_rowwise(8, 128, seed=6)
    e, s = oracle.quantize_mx(x, oracle.INT8, oracle.ROW, rounding)
    xf = bf16_bits_to_f64(x)
    for r in range(x.shape[0]):
        for b in range(4):
            sc = int(s[r, b]) - 127
            scaled = np.ldexp(xf[r, 32 * b:32 * b + 32], -sc)
            ref = [oracle.encode(float(v), oracle.K_INT8) for v in scaled]
            assert list(e[r, 32 * b:32 * b + 32]) == ref
            top = np.abs(scaled).max()
            if rounding == 1:
                assert 127 / 128 < top <= 127 / 64
            else:
                assert 1.0 <= top < 2.0
    d = bf16_bits_to_f64(oracle.dequantize_mx(e, s, 8, 128, oracle.INT8))
    q = e.view(np.int8).astype(np.float64) / 64.0
    assert np.array_equal(d, q * np.ldexp(1.0, np.repeat(s.astype(np.int64) - 127, 32, axis=1)))


def test_fp4_nibble_order(oracle):
    x = np.zeros((1, 32), dtype=np.uint16)
    x[0, 0] = f32_to_bf16_bits([6.0])[0]      # code 0x7 at even index 0
    x[0, 1] = f32_to_bf16_bits([-1.0])[0]     # code 0xA at odd index 1
    e, s = oracle.quantize_mx(x, oracle.E2M1, oracle.ROW, oracle.CEIL)
    assert s[0, 0] == 127 and e[0, 0] == 0xA7


def test_colwise_is_rowwise_of_transpose(oracle):
    x = synth.activations(64, 96, seed=2)
    for fmt in (oracle.E4M3, oracle.E5M2, oracle.E2M1, oracle.E2M3, oracle.E3M2, oracle.INT8):
        ec, sc = oracle.quantize_mx(x, fmt, oracle.COL, oracle.CEIL)
        er, sr = oracle.quantize_mx(np.ascontiguousarray(x.T), fmt, oracle.ROW, oracle.CEIL)
        assert np.array_equal(ec, er) and np.array_equal(sc, sr)
        assert ec.shape == (96, oracle.elem_bytes(64, fmt)) and sc.shape == (96, 2)


def test_nan_or_inf_makes_block_nan(oracle):
    x = synth.normal(2, 64, seed=1)
    x[0, 5] = 0x7FC0      # NaN in block (0, 0)
    x[1, 40] = 0xFF80     # -Inf in block (1, 1)
    for fmt in (oracle.E4M3, oracle.E5M2, oracle.E2M1, oracle.E2M3, oracle.E3M2, oracle.INT8):
        e, s = oracle.quantize_mx(x, fmt, oracle.ROW, oracle.CEIL)
        assert s[0, 0] == 0xFF and s[1, 1] == 0xFF and s[0, 1] != 0xFF and s[1, 0] != 0xFF
        d = bf16_bits_to_f64(oracle.dequantize_mx(e, s, 2, 64, fmt))
        assert np.all(np.isnan(d[0, :32])) and np.all(np.isnan(d[1, 32:]))
        assert np.all(np.isfinite(d[0, 32:])) and np.all(np.isfinite(d[1, :32]))


def test_zero_block(oracle):
    x = np.zeros((1, 64), dtype=np.uint16)
    x[0, 33] = 0x8000   # -0
    e, s = oracle.quantize_mx(x, oracle.E4M3, oracle.ROW, oracle.CEIL)
    assert list(s[0]) == [0, 0] and e[0, 33] == 0x80 and np.all(np.delete(e[0], 33) == 0)


# ------------------------------------------------------------------ dequantisation
@pytest.mark.parametrize("fmt_name,dtype", [("E4M3", torch.float8_e4m3fn), ("E5M2", torch.float8_e5m2)])
def test_dequant_is_exponent_add(oracle, fmt_name, dtype):
    """dec(q) * 2^(s-127) through a library fp8 decode and ldexp (exact, then bf16)."""
    fmt = getattr(oracle, fmt_name)
    x = synth.mx8_rowwise(8, 256, seed=7)
    e, s = oracle.quantize_mx(x, fmt, oracle.ROW, oracle.CEIL)
    got = bf16_bits_to_f64(oracle.dequantize_mx(e, s, 8, 256, fmt))
    dec = torch.from_numpy(e).view(dtype).double().numpy()
    ref = np.ldexp(dec, np.repeat(s.astype(np.int64) - 127, 32, axis=1))
    ref_bf16 = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()  # single RNE from fp64
    assert np.array_equal(got, ref_bf16)


def test_dequant_value_idempotent(oracle):
    """quantise(dequantise(quantise(x))) reproduces the same dequantised values."""
    x = synth.mx8_rowwise(32, 256, seed=11)
    for fmt in (oracle.E4M3, oracle.E5M2, oracle.E2M1):
        for rnd in (oracle.FLOOR, oracle.CEIL):
            e, s = oracle.quantize_mx(x, fmt, oracle.ROW, rnd)
            d1 = oracle.dequantize_mx(e, s, 32, 256, fmt)
            e2, s2 = oracle.quantize_mx(d1, fmt, oracle.ROW, rnd)
            d2 = oracle.dequantize_mx(e2, s2, 32, 256, fmt)
            assert np.array_equal(d1, d2)


def test_dequant_nan_scale_and_subnormal_output(oracle):
    e = np.full((1, 32), 0x01, dtype=np.uint8)          # E4M3 smallest subnormal 2^-9
    s = np.array([[0]], dtype=np.uint8)                 # 2^-127 -> 2^-136, below bf16 subnormals' quantum
    d = oracle.dequantize_mx(e, s, 1, 32, oracle.E4M3)
    assert np.all(d == 0x0000)                          # 2^-136 rounds to 0 in bf16 (quantum 2^-133)
    e[:] = 0x08                                         # 2^-6 * 2^-127 = 2^-133: the smallest bf16 subnormal
    assert np.all(oracle.dequantize_mx(e, s, 1, 32, oracle.E4M3) == 0x0001)
    s[:] = 0xFF
    assert np.all(np.isnan(bf16_bits_to_f64(oracle.dequantize_mx(e, s, 1, 32, oracle.E4M3))))


# ------------------------------------------------------------------ NVFP4
def test_nvfp4_global_scale_definition(oracle):
    g_fix = read_golden("format_constants.txt")
    assert g_fix["nvfp4_global_divisor"][0] == 6 * 448
    x = synth.weight_fp4(64, 128, seed=4)
    _, _, g = oracle.quantize_nvfp4(x)
    amax = np.abs(bits_to_finite(x)).max()
    assert g == float(np.float32(amax) / np.float32(g_fix["nvfp4_global_divisor"][0]))
    # a tensor whose maximum is exactly 6 * 448 has g = 1 and that block's scale is 448
    y = synth.normal(4, 32, sigma=1.0, seed=9)
    y[2, 17] = f32_to_bf16_bits([2688.0])[0]
    e, s, g = oracle.quantize_nvfp4(y)
    assert g == 1.0 and s[2, 1] == 0x7E and oracle.decode(oracle.K_UE4M3, int(s[2, 1])) == 448.0
    assert unpack_fp4(e[2], 32)[17] == 0x7                  # 2688 / 448 = 6


def bits_to_finite(bits):
    v = bf16_bits_to_f64(bits)
    return np.where(np.isfinite(v), v, 0.0)


def test_nvfp4_block_scale_is_nearest_ue4m3(oracle):
    """sb is the nearest (ties even) UE4M3 code to amax_b / (6 g), found by brute force,
    and the elements are the E2M1 codes of the fp32 quotient x / d (numpy's IEEE division;
    the exhaustive form of this pin is in test_oracle_nvfp4_quotient.py)."""
    x = synth.weight_fp4(32, 256, seed=6)
    e, s, g = oracle.quantize_nvfp4(x)
    ue = np.array([oracle.decode(oracle.K_UE4M3, c) for c in range(0x7F)])
    xf = bf16_bits_to_f64(x).astype(np.float32)
    six_g = np.float32(6.0) * np.float32(g)
    for r in range(32):
        codes = unpack_fp4(e[r], 256)
        for b in range(16):
            blk = xf[r, 16 * b:16 * b + 16]
            t = np.float32(np.abs(blk).max()) / six_g
            d = np.abs(ue - float(t))
            cand = np.nonzero(d == d.min())[0]
            want = cand[0] if cand.size == 1 else [c for c in cand if c % 2 == 0][0]
            assert s[r, b] == want
            dd = np.float32(ue[want]) * np.float32(g)
            if dd == 0:
                assert np.all(codes[16 * b:16 * b + 16] == 0)
                continue
            scaled = blk / dd
            ref = np.array([oracle.encode(float(v), oracle.K_E2M1) for v in scaled])
            assert np.array_equal(codes[16 * b:16 * b + 16], ref)
            # error bound: half the widest E2M1 spacing (1.0) times d, plus clipping above 6
            xh = e2m1_values(codes[16 * b:16 * b + 16]) * float(dd)
            assert np.all(np.abs(xh - blk) <= float(dd) * 1.0 + np.maximum(np.abs(blk) - 6 * float(dd), 0) + 1e-30)


def test_nvfp4_scale_relative_error(oracle):
    """dec(sb) * g * 6 is within the E4M3 half-ulp (2^-4 relative) of the block max."""
    x = synth.weight_fp4(64, 256, seed=8)
    _, s, g = oracle.quantize_nvfp4(x)
    xf = np.abs(bits_to_finite(x)).reshape(64, 16, 16).max(axis=2)
    dec = np.array([[oracle.decode(oracle.K_UE4M3, int(c)) for c in row] for row in s])
    normal = xf / (6 * g) >= 2.0 ** -6
    rel = np.abs(dec * g * 6 - xf) / xf
    assert np.all(rel[normal] <= 2.0 ** -4 + 1e-6)


def test_nvfp4_dequant_order(oracle):
    x = synth.weight_fp4(16, 64, seed=10)
    e, s, g = oracle.quantize_nvfp4(x)
    got = bf16_bits_to_f64(oracle.dequantize_nvfp4(e, s, g, 16, 64))
    q = e2m1_values(np.stack([unpack_fp4(r, 64) for r in e])).astype(np.float32)
    sb = torch.from_numpy(s).view(torch.float8_e4m3fn).float().numpy()
    ref = (q * np.repeat(sb, 16, axis=1)) * np.float32(g)
    ref = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(got, ref)


def test_nvfp4_nonfinite_block(oracle):
    x = synth.normal(2, 32, seed=12)
    x[1, 3] = 0x7F80
    e, s, g = oracle.quantize_nvfp4(x)
    assert s[1, 0] == 0x7F and s[1, 1] != 0x7F and np.all(unpack_fp4(e[1], 32)[:16] == 0)
    assert math.isfinite(g)
    d = bf16_bits_to_f64(oracle.dequantize_nvfp4(e, s, g, 2, 32))
    assert np.all(np.isnan(d[1, :16])) and np.all(np.isfinite(d[1, 16:]))


# ------------------------------------------------------------------ fp64 matmul reference
def test_gemm_ref_exact_brute_force(oracle):
    """Tiny case against exact rational arithmetic over library-decoded operands."""
    M, N, K = 3, 2, 64
    a = synth.normal(M, K, seed=13)
    b = synth.weight_fp4(N, K, seed=14)
    ae, as_ = oracle.quantize_mx(a, oracle.E4M3, oracle.ROW, oracle.CEIL)
    be, bs = oracle.quantize_mx(b, oracle.E2M1, oracle.ROW, oracle.FLOOR)
    pairs = [(m, n) for m in range(M) for n in range(N)]
    c, mag = oracle.gemm_ref(ae, as_, oracle.E4M3, be, bs, oracle.E2M1, M, N, K, pairs)
    av = torch.from_numpy(ae).view(torch.float8_e4m3fn).double().numpy()
    bv = e2m1_values(np.stack([unpack_fp4(r, K) for r in be]))
    for p, (m, n) in enumerate(pairs):
        exact = sum(Fraction(float(av[m, k])) * Fraction(2) ** (int(as_[m, k // 32]) - 127)
                    * Fraction(float(bv[n, k])) * Fraction(2) ** (int(bs[n, k // 32]) - 127)
                    for k in range(K))
        assert abs(Fraction(c[p]) - exact) <= abs(exact) * Fraction(2) ** -50 + Fraction(2) ** -1000
        assert mag[p] >= abs(c[p])


def test_gemm_ref_fp4_operands_exact(oracle):
    """MXFP4 x MXFP4 and NVFP4 x NVFP4 (with both per-tensor scales) against exact rational
    arithmetic over independently decoded operands: E2M1 from its value table, UE4M3 block
    scales by the E4M3 decoder of ml_dtypes, E8M0 as a power of two."""
    M, N, K = 2, 3, 64
    a = synth.weight_fp4(M, K, seed=21)
    b = synth.normal(N, K, seed=22)
    pairs = [(m, n) for m in range(M) for n in range(N)]
    # MXFP4 x MXFP4
    ae, as_ = oracle.quantize_mx(a, oracle.E2M1, oracle.ROW, oracle.FLOOR)
    be, bs = oracle.quantize_mx(b, oracle.E2M1, oracle.ROW, oracle.FLOOR)
    c, mag = oracle.gemm_ref(ae, as_, oracle.E2M1, be, bs, oracle.E2M1, M, N, K, pairs)
    av = e2m1_values(np.stack([unpack_fp4(r, K) for r in ae]))
    bv = e2m1_values(np.stack([unpack_fp4(r, K) for r in be]))
    for p, (m, n) in enumerate(pairs):
        exact = sum(Fraction(float(av[m, k])) * Fraction(2) ** (int(as_[m, k // 32]) - 127)
                    * Fraction(float(bv[n, k])) * Fraction(2) ** (int(bs[n, k // 32]) - 127) for k in range(K))
        assert Fraction(c[p]) == exact
        assert mag[p] >= abs(c[p])
    # NVFP4 x NVFP4: dec(q) * dec(sb) * g on each side
    ae, as_, ga = oracle.quantize_nvfp4(a)
    be, bs, gb = oracle.quantize_nvfp4(b)
    c, mag = oracle.gemm_ref(ae, as_, oracle.NVFP4, be, bs, oracle.NVFP4, M, N, K, pairs, a_g=ga, b_g=gb)
    av = e2m1_values(np.stack([unpack_fp4(r, K) for r in ae]))
    bv = e2m1_values(np.stack([unpack_fp4(r, K) for r in be]))
    sa = as_.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    sb = bs.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert np.all(as_ < 0x7F) and np.all(bs < 0x7F)
    for p, (m, n) in enumerate(pairs):
        exact = sum(Fraction(float(av[m, k])) * Fraction(float(sa[m, k // 16])) * Fraction(float(ga))
                    * Fraction(float(bv[n, k])) * Fraction(float(sb[n, k // 16])) * Fraction(float(gb))
                    for k in range(K))
        # each fp64 product of two 31-bit significands rounds once, then K additions:
        # |error| <= (K + 1) u sum|ab| with u = 2^-53
        assert abs(Fraction(c[p]) - exact) <= (K + 1) * Fraction(2) ** -53 * Fraction(mag[p])
        assert mag[p] >= abs(c[p])
    # g enters linearly
    c2, _ = oracle.gemm_ref(ae, as_, oracle.NVFP4, be, bs, oracle.NVFP4, M, N, K, pairs, a_g=2 * ga, b_g=gb)
    assert np.allclose(c2, 2 * c, rtol=1e-15, atol=0)


def test_gemm_ref_one_hot(oracle):
    K = 96
    a = np.zeros((1, K), dtype=np.uint16)
    a[0, 70] = f32_to_bf16_bits([3.0])[0]
    b = synth.normal(4, K, seed=15)
    ae, as_ = oracle.quantize_mx(a, oracle.E4M3, oracle.ROW, oracle.CEIL)
    be, bs = oracle.quantize_mx(b, oracle.E4M3, oracle.ROW, oracle.CEIL)
    c, _ = oracle.gemm_ref(ae, as_, oracle.E4M3, be, bs, oracle.E4M3, 1, 4, K, [(0, n) for n in range(4)])
    bdec = bf16_bits_to_f64(oracle.dequantize_mx(be, bs, 4, K, oracle.E4M3))
    assert np.array_equal(c, 3.0 * bdec[:, 70])


def test_gemm_ref_block_equals_per_entry_reference(oracle):
    """The rectangle form (rows decoded once) gives exactly the per-entry sums, for MX,
    mixed and NVFP4 operands."""
    M, N, K = 24, 40, 256
    a = synth.normal(M, K, seed=21)
    b = synth.weight_fp4(N, K, seed=22)
    pairs = np.array([(m, n) for m in range(3, 19) for n in range(5, 37)], dtype=np.int64)
    for fa, fb in ((oracle.E4M3, oracle.E4M3), (oracle.E4M3, oracle.E2M1), (oracle.NVFP4, oracle.NVFP4)):
        if fa == oracle.NVFP4:
            ae, as_, ga = oracle.quantize_nvfp4(a)
            be, bs, gb = oracle.quantize_nvfp4(b)
        else:
            (ae, as_), ga = oracle.quantize_mx(a, fa, oracle.ROW, oracle.CEIL), 1.0
            (be, bs), gb = oracle.quantize_mx(b, fb, oracle.ROW, oracle.FLOOR), 1.0
        c, mag = oracle.gemm_ref(ae, as_, fa, be, bs, fb, M, N, K, pairs, a_g=ga, b_g=gb)
        cb, magb = oracle.gemm_ref_block(ae, as_, fa, be, bs, fb, M, N, K, 3, 19, 5, 37, a_g=ga, b_g=gb)
        assert np.array_equal(cb.reshape(-1), c) and np.array_equal(magb.reshape(-1), mag)


# ------------------------------------------------------------------ tcgen05 scale tiling
def test_tcgen05_whole_matrix_tiling_matches_offsets(oracle):
    """to/from_tcgen05_layout place every scale at its offset, zero the padding and invert
    each other."""
    rng = np.random.default_rng(3)
    for rows, scols in [(128, 4), (130, 5), (300, 33), (1, 1)]:
        s = rng.integers(1, 256, (rows, scols), dtype=np.uint8)
        t = oracle.to_tcgen05_layout(s)
        off = oracle.tcgen05_offsets(rows, scols)
        assert np.array_equal(t[off], s)
        pad = np.ones(t.size, dtype=bool)
        pad[off.reshape(-1)] = False
        assert np.all(t[pad] == 0)
        assert np.array_equal(oracle.from_tcgen05_layout(t, rows, scols), s)


def test_tcgen05_tiling_is_a_padded_bijection(oracle):
    for rows, scols in [(128, 4), (256, 8), (130, 5), (1, 1), (300, 33)]:
        off = oracle.tcgen05_offsets(rows, scols)
        total = oracle.tcgen05_scale_bytes(rows, scols)
        assert total == math.ceil(rows / 128) * math.ceil(scols / 4) * 512
        assert len(np.unique(off)) == off.size and off.min() >= 0 and off.max() < total
    # a full 128 x 4 atom is a permutation of 0..511; consecutive scale columns of one
    # row are adjacent bytes, and 32 rows apart are 4 bytes apart
    off = oracle.tcgen05_offsets(128, 4)
    assert sorted(off.ravel()) == list(range(512))
    assert np.all(np.diff(off, axis=1) == 1)
    assert np.all(off[32:64] - off[0:32] == 4)


# ------------------------------------------------------------------ NVFP4 16 x 16 weight blocks
def test_nvfp4_2d_blocks_commute_with_transposition(oracle):
    """Two-dimensional blocks make the weight and its transpose quantise identically ([Q] §4:
    2-D block scaling for weights): codes and block scales of W^T are those of W, transposed."""
    x = synth.weight_fp4(64, 96, seed=31)
    e, s, g = oracle.quantize_nvfp4_2d(x)
    et, st, gt = oracle.quantize_nvfp4_2d(np.ascontiguousarray(x.T))
    assert g == gt
    codes = np.stack([unpack_fp4(r, 96) for r in e])
    codes_t = np.stack([unpack_fp4(r, 64) for r in et])
    assert np.array_equal(codes_t, codes.T)
    blk = s[::16]                                   # one row per 16-row group
    blk_t = st[::16]
    assert np.array_equal(blk_t, blk.T)
    for r in range(64):                             # every row of a group carries its block's scale
        assert np.array_equal(s[r], s[(r // 16) * 16])


def test_nvfp4_2d_reduces_to_1d_on_single_row_blocks(oracle):
    """A matrix whose 16-row groups each hold one nonzero row: every 2-D block's maximum is
    that row's 1 x 16 maximum, so the row's codes and scales equal the (pinned) 1-D NVFP4
    quantisation of the same matrix."""
    x = synth.weight_fp4(48, 64, seed=32)
    keep = np.zeros_like(x)
    for grp in range(3):
        keep[grp * 16 + 5 * grp] = x[grp * 16 + 5 * grp]
    e2, s2, g2 = oracle.quantize_nvfp4_2d(keep)
    e1, s1, g1 = oracle.quantize_nvfp4(keep)
    assert g1 == g2
    for grp in range(3):
        r = grp * 16 + 5 * grp
        assert np.array_equal(e2[r], e1[r]) and np.array_equal(s2[r], s1[r])


def test_nvfp4_2d_nonfinite_block(oracle):
    x = synth.normal(32, 32, seed=33)
    x[20, 3] = 0x7FC0                              # NaN in block (1, 0)
    e, s, g = oracle.quantize_nvfp4_2d(x)
    assert np.all(s[16:32, 0] == 0x7F) and np.all(s[:16, 0] != 0x7F) and np.all(s[:, 1] != 0x7F)
    codes = np.stack([unpack_fp4(r, 32) for r in e])
    assert np.all(codes[16:32, :16] == 0)
    assert math.isfinite(g)


# ------------------------------------------------------------------ 16 x 16 random Hadamard transform
def test_rht16_matches_matrix_product(oracle):
    """On inputs whose butterfly sums are exact in fp32 (small integers and halves), the
    transform equals scipy's Sylvester Hadamard matrix times the sign-flipped input, / 4,
    rounded once to bf16 (torch's RNE conversion)."""
    from scipy.linalg import hadamard
    rng = np.random.default_rng(41)
    x = (rng.integers(-64, 65, size=(8, 64)) * 0.5).astype(np.float32)
    bits = f32_to_bf16_bits(x).reshape(8, 64)
    H = hadamard(16).astype(np.float64)
    for mask in (0x0000, 0xFFFF, 0xA5C3, 0x1234):
        d = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(16)])
        y = bf16_bits_to_f64(oracle.rht16(bits, mask))
        xf = bf16_bits_to_f64(bits)
        ref = np.concatenate([(H @ (d[:, None] * xf[:, c:c + 16].T)).T / 4 for c in range(0, 64, 16)], axis=1)
        ref = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
        assert np.array_equal(y, ref)


def test_rht16_is_orthogonal(oracle):
    """H16 D / 4 is orthogonal: D H16 / 4 undoes it (exactly on exact inputs), and norms are
    kept up to the bf16 rounding of the outputs."""
    from scipy.linalg import hadamard
    rng = np.random.default_rng(42)
    x = (rng.integers(-8, 9, size=(4, 32)) * 0.25).astype(np.float32)   # outputs exact in bf16
    bits = f32_to_bf16_bits(x).reshape(4, 32)
    mask = 0x6C39
    y = bf16_bits_to_f64(oracle.rht16(bits, mask))
    d = np.array([-1.0 if (mask >> i) & 1 else 1.0 for i in range(16)])
    H = hadamard(16).astype(np.float64)
    back = np.concatenate([(d[:, None] * (H @ y[:, c:c + 16].T)).T / 4 for c in (0, 16)], axis=1)
    assert np.array_equal(back, bf16_bits_to_f64(bits))
    z = bf16_bits_to_f64(oracle.rht16(synth.normal(16, 256, seed=43), 0xBEEF))
    zi = bf16_bits_to_f64(synth.normal(16, 256, seed=43))
    for r in range(16):
        for c in range(0, 256, 16):
            n0, n1 = np.linalg.norm(zi[r, c:c + 16]), np.linalg.norm(z[r, c:c + 16])
            assert abs(n1 - n0) <= 2.0 ** -7 * n0
