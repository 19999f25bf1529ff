"""Pins of the oracle's element and scale codecs against what the pages and independent
library routines fix (no GPU).

Independent references used here: torch's float8_e4m3fn / float8_e5m2 / float8_e8m0fnu
dtypes and ml_dtypes' float4_e2m1fn / float6_e2m3fn / float6_e3m2fn (library decoders and
RNE converters), math.ldexp, and a brute-force nearest-code search written over the
decoded code tables.
"""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

from conftest import f32_to_bf16_bits, pack_codes, read_golden, unpack_codes

ALL_BF16 = np.arange(65536, dtype=np.uint32).astype(np.uint16)


def bf16_bits_to_f64(bits):
    with np.errstate(invalid="ignore"):
        return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def library_decode_table(kind, o):
    """Decoded values of every code, from a library dtype (not the oracle)."""
    if kind == o.K_E4M3:
        return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    if kind == o.K_E5M2:
        return torch.arange(256, dtype=torch.uint8).view(torch.float8_e5m2).double().numpy()
    if kind == o.K_E8M0:
        return torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    if kind == o.K_E2M1:
        return np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    if kind == o.K_E2M3:
        return np.arange(64, dtype=np.uint8).view(ml_dtypes.float6_e2m3fn).astype(np.float64)
    if kind == o.K_E3M2:
        return np.arange(64, dtype=np.uint8).view(ml_dtypes.float6_e3m2fn).astype(np.float64)
    raise ValueError(kind)


def unpack_fp4(packed, n):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p & 0xF
    out[1::2] = p >> 4
    return out[:n]


# ------------------------------------------------------------------ decode tables
def test_e2m1_value_set_matches_page(oracle):
    g = read_golden("e2m1_values.txt")
    vals = [oracle.decode(oracle.K_E2M1, c) for c in range(16)]
    assert all(math.isfinite(v) for v in vals), "E2M1 has no Inf/NaN"
    assert sorted(v for v in vals if v >= 0 and not math.copysign(1, v) < 0) == g["nonnegative"]
    assert vals[8:] == [-v for v in vals[:8]], "negative half mirrors the positive half"
    assert len(set(vals)) == int(g["distinct_values"][0])
    assert len(vals) == int(g["codes"][0])
    assert max(vals) == g["max"][0]


@pytest.mark.parametrize("name", ["K_E4M3", "K_E5M2", "K_E2M1", "K_E8M0", "K_E2M3", "K_E3M2"])
def test_decode_tables_match_library(oracle, name):
    kind = getattr(oracle, name)
    ref = library_decode_table(kind, oracle)
    got = np.array([oracle.decode(kind, c) for c in range(ref.size)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(ref[ok]))


def test_format_maxima(oracle):
    g = read_golden("format_constants.txt")
    e4 = [oracle.decode(oracle.K_E4M3, c) for c in range(128)]
    e5 = [oracle.decode(oracle.K_E5M2, c) for c in range(128)]
    assert max(v for v in e4 if math.isfinite(v)) == g["e4m3_max"][0] == 448
    assert math.isnan(e4[0x7F]), "S.1111.111 is the only E4M3 NaN"
    assert sum(math.isnan(v) for v in e4) == 1 and not any(math.isinf(v) for v in e4)
    assert max(v for v in e5 if math.isfinite(v)) == g["e5m2_max"][0] == 1.75 * 2 ** 15
    assert math.isinf(e5[0x7C]) and all(math.isnan(e5[c]) for c in (0x7D, 0x7E, 0x7F))
    # UE4M3: the unsigned E4M3 block scale of NVFP4, same magnitudes, max 448
    ue = [oracle.decode(oracle.K_UE4M3, c) for c in range(128)]
    assert ue[:0x7F] == e4[:0x7F] and math.isnan(ue[0x7F]) and ue[0x7E] == 448


def test_e8m0_definition(oracle):
    g = read_golden("format_constants.txt")
    bias = int(g["e8m0_bias"][0])
    for c in range(255):
        assert oracle.decode(oracle.K_E8M0, c) == math.ldexp(1.0, c - bias)
    assert math.isnan(oracle.decode(oracle.K_E8M0, int(g["e8m0_nan"][0])))
    assert oracle.decode(oracle.K_E8M0, 0) == 2.0 ** -127 and oracle.decode(oracle.K_E8M0, 254) == 2.0 ** 127


# ------------------------------------------------------------------ exhaustive cast
def brute_force_cast(x, table, mag_codes, sign_bit, nan_code_pos, nan_sign=True):
    """Nearest finite code by exhaustive search; ties to the even code; saturation is
    implied (the nearest finite value of anything above the maximum is the maximum);
    +-Inf saturate; NaN -> nan_code_pos (| sign)."""
    mags = table[mag_codes]
    ax = np.abs(x)
    # anything at or above the maximum has the maximum as its unique nearest finite
    # value; clipping at 2 * max keeps that argmin and avoids fp64 cancellation
    ax_f = np.minimum(np.where(np.isfinite(ax), ax, mags.max()), 2 * mags.max())
    d = np.abs(ax_f[:, None] - mags[None, :])
    mind = d.min(axis=1)
    cand = d == mind[:, None]
    ncand = cand.sum(axis=1)
    first = np.argmax(cand, axis=1)
    last = cand.shape[1] - 1 - np.argmax(cand[:, ::-1], axis=1)
    even_pick = np.where(mag_codes[first] % 2 == 0, first, last)
    pick = np.where(ncand == 1, first, even_pick)
    code = mag_codes[pick].astype(np.int64)
    neg = np.signbit(x)
    code = np.where(neg, code | sign_bit, code)
    nan = np.isnan(x)
    code = np.where(nan, np.where(neg & nan_sign, nan_code_pos | sign_bit, nan_code_pos), code)
    return code


@pytest.mark.parametrize("fmt_name", ["E4M3", "E5M2", "E2M1", "E2M3", "E3M2"])
def test_exhaustive_bf16_cast_against_brute_force(oracle, fmt_name):
    fmt = getattr(oracle, fmt_name)
    kind = getattr(oracle, "K_" + fmt_name)
    table = library_decode_table(kind, oracle)
    if fmt_name == "E4M3":
        mag_codes, sign_bit, nan_pos = np.arange(0x7F), 0x80, 0x7F
    elif fmt_name == "E5M2":
        mag_codes, sign_bit, nan_pos = np.arange(0x7C), 0x80, 0x7F
    elif fmt_name == "E2M1":
        mag_codes, sign_bit, nan_pos = np.arange(8), 0x8, 0x7   # no NaN: reading is +-6
    else:
        mag_codes, sign_bit, nan_pos = np.arange(32), 0x20, 0x1F  # FP6: no NaN, reading +-max
    x = bf16_bits_to_f64(ALL_BF16)
    ref = brute_force_cast(x, table, mag_codes, sign_bit, nan_pos)
    got = oracle.cast(ALL_BF16, fmt)
    if fmt_name == "E2M1":
        got = unpack_fp4(got, ALL_BF16.size)
    elif fmt_name in ("E2M3", "E3M2"):
        got = unpack_codes(got, ALL_BF16.size, 6)
    bad = np.nonzero(got.astype(np.int64) != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first bf16 {ALL_BF16[bad[:5]]}"


@pytest.mark.parametrize("fmt_name,dtype,maxv", [("E4M3", torch.float8_e4m3fn, 448.0),
                                                 ("E5M2", torch.float8_e5m2, 57344.0)])
def test_cast_matches_torch_in_range(oracle, fmt_name, dtype, maxv):
    """torch's fp8 conversion is RNE without saturation: equal to ours below the max."""
    x32 = bf16_bits_to_f64(ALL_BF16).astype(np.float32)
    ok = np.isfinite(x32) & (np.abs(x32) < maxv)
    ref = torch.from_numpy(x32[ok]).to(dtype).view(torch.uint8).numpy()
    got = oracle.cast(ALL_BF16[ok], getattr(oracle, fmt_name))
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("fmt_name,dtype,maxv", [("E2M3", ml_dtypes.float6_e2m3fn, 7.5),
                                                 ("E3M2", ml_dtypes.float6_e3m2fn, 28.0)])
def test_fp6_cast_matches_ml_dtypes_in_range(oracle, fmt_name, dtype, maxv):
    """ml_dtypes' FP6 conversion (round to nearest even) agrees with ours up to the max."""
    x32 = bf16_bits_to_f64(ALL_BF16).astype(np.float32)
    ok = np.isfinite(x32) & (np.abs(x32) <= maxv)
    sel = ALL_BF16[ok][: ok.sum() // 4 * 4]              # FP6 casts take whole bytes: n % 4 == 0
    ref = x32[ok][: sel.size].astype(dtype).view(np.uint8) & 0x3F
    got = unpack_codes(oracle.cast(sel, getattr(oracle, fmt_name)), sel.size, 6)
    assert np.array_equal(got, ref)


def test_fp6_storage_packing(oracle):
    """FP6 codes are stored four per three bytes, code i at bits [6i, 6i + 6) of the row.
    Hand-worked: E2M3 subnormals 0.125, 0.25, 0.375, 0.5 are codes 1, 2, 3, 4 (m / 8 with
    bias 1), i.e. 1 + 2*2^6 + 3*2^12 + 4*2^18 = 0x103081 -> bytes 81 30 10; the E3M2 max
    28 (code 0x1F) and -28 (0x3F) alternating give 0x1F | 0x3F << 6 | 0x1F << 12 | 0x3F << 18
    = 0xFDFFDF -> DF FF FD."""
    assert list(oracle.cast(f32_to_bf16_bits([0.125, 0.25, 0.375, 0.5]), oracle.E2M3)) == [0x81, 0x30, 0x10]
    assert list(oracle.cast(f32_to_bf16_bits([28.0, -28.0, 28.0, -28.0]), oracle.E3M2)) == [0xDF, 0xFF, 0xFD]
    # numpy's bit packing of the per-element codes, over all bf16 inputs
    for fmt, kind in ((oracle.E2M3, oracle.K_E2M3), (oracle.E3M2, oracle.K_E3M2)):
        x = ALL_BF16[::7][:4096]
        codes = np.array([oracle.encode(v, kind) for v in bf16_bits_to_f64(x)], dtype=np.uint8)
        codes[np.isnan(bf16_bits_to_f64(x))] = 0  # NaN inputs: compared separately below
        keep = ~np.isnan(bf16_bits_to_f64(x))
        got = unpack_codes(oracle.cast(x, fmt), x.size, 6)
        assert np.array_equal(got[keep], codes[keep])
        assert np.array_equal(pack_codes(got, 6), oracle.cast(x, fmt))
    # a cast of a count that does not fill whole bytes is refused
    with pytest.raises(ValueError):
        oracle.cast(ALL_BF16[:6], oracle.E2M3)


def test_int8_element_definition(oracle):
    """MXINT8 element: two's complement q read as q / 64, encoded by round half to even
    onto that grid and saturated symmetrically at +-127 (brute force over the 255 values)."""
    codes = np.arange(256)
    vals = np.array([oracle.decode(oracle.K_INT8, int(c)) for c in codes])
    assert np.array_equal(vals, codes.astype(np.uint8).view(np.int8).astype(np.float64) / 64.0)
    grid = np.arange(-127, 128, dtype=np.float64) / 64.0
    x = bf16_bits_to_f64(ALL_BF16)
    fin = np.isfinite(x)
    xs = x[fin]
    # beyond +-4 the nearest grid point is the end point; clipping keeps the distances exact
    d = np.abs(np.clip(xs, -4.0, 4.0)[:, None] - grid[None, :])
    best = d.min(axis=1)
    cand = d == best[:, None]
    q = np.arange(-127, 128)
    # ties: the even integer; beyond the range the end point is nearest anyway
    pick = np.where(cand.sum(axis=1) > 1, np.argmax(cand & (q[None, :] % 2 == 0), axis=1), np.argmax(cand, axis=1))
    ref = (q[pick].astype(np.int64) & 0xFF)
    got = np.array([oracle.encode(float(v), oracle.K_INT8) for v in xs])
    assert np.array_equal(got, ref)
    assert oracle.encode(math.inf, oracle.K_INT8) == 127 and oracle.encode(-math.inf, oracle.K_INT8) == 0x81
    assert oracle.encode(-1e-9, oracle.K_INT8) == 0     # no negative zero in two's complement


def test_e2m1_cast_matches_ml_dtypes_in_range(oracle):
    x32 = bf16_bits_to_f64(ALL_BF16).astype(np.float32)
    ok = np.isfinite(x32) & (np.abs(x32) <= 6.0)
    xs = x32[ok]
    if xs.size % 2:
        xs = xs[:-1]
    ref = xs.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    got = unpack_fp4(oracle.cast(to_bits(xs), oracle.E2M1), xs.size)
    assert np.array_equal(got, ref)


def to_bits(x32):
    return (np.asarray(x32, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_saturation_and_signed_zero(oracle):
    enc = oracle.encode
    assert enc(1e6, oracle.K_E4M3) == 0x7E and enc(-1e6, oracle.K_E4M3) == 0xFE
    assert enc(math.inf, oracle.K_E4M3) == 0x7E and enc(-math.inf, oracle.K_E5M2) == 0xFB
    assert enc(464.0, oracle.K_E4M3) == 0x7E          # tie 448/480: even mantissa, and 480 is NaN
    assert enc(7.0, oracle.K_E2M1) == 0x7 and enc(-100.0, oracle.K_E2M1) == 0xF
    assert enc(-1e-30, oracle.K_E4M3) == 0x80 and enc(-0.0, oracle.K_E2M1) == 0x8
    assert enc(0.25, oracle.K_E2M1) == 0x0            # tie 0 / 0.5 -> even (0)
    assert enc(0.75, oracle.K_E2M1) == 0x2            # tie 0.5 / 1.0 -> even (1.0, code 2)
    assert enc(2.0 ** -10, oracle.K_E4M3) == 0x00     # half of the smallest subnormal -> 0
    assert enc(1.5 * 2.0 ** -10, oracle.K_E4M3) == 0x01


# ------------------------------------------------------------------ shared scale exponent
def positive_finite_bf16():
    b = np.arange(0x0001, 0x7F80, dtype=np.uint32).astype(np.uint16)
    return b, bf16_bits_to_f64(b)


@pytest.mark.parametrize("fmt_name,emax,maxv", [("E4M3", 8, 448.0), ("E5M2", 15, 57344.0), ("E2M1", 2, 6.0),
                                                ("E2M3", 2, 7.5), ("E3M2", 4, 28.0), ("INT8", 0, 127 / 64)])
def test_floor_school_landing_interval(oracle, fmt_name, emax, maxv):
    """Floor school: scaled block maximum in [2^emax, 2^(emax+1)) -- [4, 8) for E2M1."""
    g = read_golden("format_constants.txt")
    if fmt_name == "E2M1":
        assert g["floor_landing_e2m1"] == [2.0 ** emax, 2.0 ** (emax + 1)]
    fmt = getattr(oracle, fmt_name)
    _, amax = positive_finite_bf16()
    for a in amax:
        s = oracle.scale_exponent(a, fmt, oracle.FLOOR)
        if s == -127:
            assert math.ldexp(a, 127) < 2.0 ** (emax + 1)
            continue
        scaled = math.ldexp(a, -s)
        assert 2.0 ** emax <= scaled < 2.0 ** (emax + 1), (a, s)
        assert s == math.frexp(a)[1] - 1 - emax


@pytest.mark.parametrize("fmt_name,maxv", [("E4M3", 448.0), ("E5M2", 57344.0), ("E2M1", 6.0), ("E2M3", 7.5),
                                           ("E3M2", 28.0), ("INT8", 127 / 64)])
def test_ceil_school_landing_interval(oracle, fmt_name, maxv):
    """No-clip school: scaled maximum in (max/2, max] -- (3, 6] for E2M1 -- and the
    scale is the smallest one that does not clip."""
    g = read_golden("format_constants.txt")
    if fmt_name == "E2M1":
        assert g["ceil_landing_e2m1"] == [maxv / 2, maxv]
    fmt = getattr(oracle, fmt_name)
    _, amax = positive_finite_bf16()
    for a in amax:
        s = oracle.scale_exponent(a, fmt, oracle.CEIL)
        scaled = math.ldexp(a, -s)
        if s == 127:                    # clamped to the E8M0 range (INT8 at the largest bf16)
            assert math.ldexp(a, -128) <= maxv
            continue
        assert scaled <= maxv, (a, s)
        if s > -127:
            assert maxv / 2 < scaled, (a, s)
            assert math.ldexp(a, -(s - 1)) > maxv       # one step smaller would clip


def test_zero_block_scale(oracle):
    assert oracle.scale_exponent(0.0, oracle.E4M3, oracle.FLOOR) == -127
    assert oracle.scale_exponent(0.0, oracle.E2M1, oracle.CEIL) == -127
