"""Pins of the oracle's NVFP4 element step (no GPU).

The page that defines NVFP4 ("MXFP4 と NVFP4 は何が違うのか調べてみた", §3) gives the
element as x over the two-level scale (a UE4M3 scale per 16 elements times the FP32
per-tensor scale g) and §7 of the same page fixes only the order of the multiplies that
decode it.  The oracle's reading: the E2M1 code, round to nearest even, of the fp32
quotient RN(x / d) with d = RN(dec(sb) g).

Three readings are set side by side here over every UE4M3 code, a sweep of g and every
finite bf16 x whose quotient is not trivially 0 or saturated:
  S  E2M1(RN32(x / d))            -- the oracle's (one IEEE division)
  R  E2M1(RN32(x * RN32(1 / d)))  -- a reciprocal multiply
  X  E2M1(x / (dec(sb) g))        -- the exact rational quotient, no intermediate rounding
The nearest-code search below is an exact threshold comparison in float64 (every
threshold m * D has at most 31 significant bits), independent of the oracle's integer
encoder, and the fp32 quotients come from numpy's IEEE float32 arithmetic.
"""
import ml_dtypes
import numpy as np
import pytest

import synth
from test_oracle_formats import unpack_fp4

E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
MIDPOINTS = (E2M1_MAG[1:] + E2M1_MAG[:-1]) / 2          # 0.25 0.75 1.25 1.75 2.5 3.5 5
UE4M3 = np.arange(0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def nearest_e2m1(a, D=None):
    """Code magnitude (0..7) of the E2M1 value nearest to a / D for a >= 0 (D = 1 when
    None), ties to the even code, saturating at 6: exact comparisons of a against the
    midpoints times D."""
    a = np.asarray(a, dtype=np.float64)
    T = MIDPOINTS if D is None else MIDPOINTS * np.asarray(D, dtype=np.float64)[..., None]
    T = np.broadcast_to(T, a.shape + (7,))
    code = (T < a[..., None]).sum(-1)
    tie = (T == a[..., None]).any(-1)
    return code + (tie & (code % 2 == 1))


def signed_code(x, mag):
    return mag.astype(np.uint8) | np.where(np.signbit(x), 8, 0).astype(np.uint8)


def gsweep():
    """Per-tensor decode scales g = RN32(amax / 2688) over tensor maxima from the bf16
    minimum subnormal to the bf16 maximum (fp32 subnormal g included)."""
    amax_bits = [0x0001, 0x0005, 0x0040, 0x0080, 0x0230, 0x0400, 0x0C2A, 0x1000, 0x1191, 0x1880, 0x2000,
                 0x2ABC, 0x3000, 0x3A83, 0x3F80, 0x4528, 0x4B37, 0x5A5A, 0x6000, 0x6F00, 0x7F7F]
    a = synth.bits_to_float(np.array(amax_bits, dtype=np.uint16))
    return a, np.float32(a) / np.float32(2688.0)


def test_nearest_e2m1_search_is_the_nearest():
    """The threshold search equals an argmin over the eight magnitudes (ties to even) on a
    fine grid that holds every midpoint."""
    a = np.arange(0, 8 * 64 + 1) / 64.0
    dist = np.abs(a[:, None] - E2M1_MAG[None, :])
    best = dist.min(1, keepdims=True)
    cand = dist == best
    want = cand.argmax(1)
    for i in np.nonzero(cand.sum(1) > 1)[0]:                   # a tie: the even code
        c = np.nonzero(cand[i])[0]
        want[i] = c[c % 2 == 0][0]
    assert np.array_equal(nearest_e2m1(a), want)


def _readings(g, sb, x):
    """Codes of the positive magnitudes x (float64, bf16-exact) under readings S, R, X."""
    d = np.float32(UE4M3[sb]) * np.float32(g)
    x32 = x.astype(np.float32)
    S = nearest_e2m1(np.abs(x32 / d))
    with np.errstate(over="ignore"):
        R = nearest_e2m1(np.abs(x32 * (np.float32(1.0) / d)))
    X = nearest_e2m1(np.abs(x), float(UE4M3[sb]) * float(g))
    return d, S, R, X


def test_readings_side_by_side():
    """S, R and X over every UE4M3 code, the g sweep and every finite bf16 magnitude whose
    quotient lies in [1/16, 8] (outside it all three give 0 or the saturated 6).  A
    difference is always one code step, and only where the exact quotient x / D lies
    within the readings' rounding of an E2M1 midpoint: for S against X the rounding of d
    (2^-24 relative when d is a normal fp32, more when g is subnormal) plus the quotient's
    own (2^-24); for R two more roundings of 2^-24.  R is undefined where RN(1/d)
    overflows (d < 2^-128): it then saturates, and those cases are counted apart."""
    mags = np.sort(synth.bits_to_float(np.arange(0, 0x7F80, dtype=np.uint16)).astype(np.float64))
    _, gs = gsweep()
    n = s_x = s_r = r_inf = 0
    for g in gs:
        if g == 0:
            continue
        for sb in range(1, 0x7F):
            D = float(UE4M3[sb]) * float(g)
            lo, hi = np.searchsorted(mags, [D / 16, D * 8])
            x = mags[lo:hi]
            if x.size == 0:
                continue
            d, S, R, X = _readings(g, sb, x)
            if d == 0:
                continue
            n += x.size
            q = x / D                                   # exact quotient, rounded once in fp64
            rel_d = abs(float(d) - D) / D
            dx = np.nonzero(S != X)[0]
            s_x += dx.size
            assert np.all(np.abs(S[dx] - X[dx]) == 1)
            mid = MIDPOINTS[np.minimum(S[dx], X[dx])]
            assert np.all(np.abs(q[dx] - mid) <= mid * (rel_d + 2.0 ** -24) * (1 + 2.0 ** -20)), (g, sb)
            if float(d) < 2.0 ** -128:                  # RN(1/d) overflows
                r_inf += x.size
                continue
            dr = np.nonzero(S != R)[0]
            s_r += dr.size
            assert np.all(np.abs(S[dr] - R[dr]) == 1)
            mid = MIDPOINTS[np.minimum(S[dr], R[dr])]
            assert np.all(np.abs(q[dr] - mid) <= mid * (rel_d + 3 * 2.0 ** -24) * (1 + 2.0 ** -20)), (g, sb)
    assert n > 1_000_000
    print(f"\nNVFP4 element readings over {n} (g, sb, x) cases: S != X in {s_x}, S != R in {s_r} "
          f"(R undefined, 1/d overflows, in {r_inf})")


@pytest.mark.parametrize("amax_bits", [0x4528, 0x3C23, 0x0F00, 0x0088])
def test_oracle_elements_are_rounded_fp32_quotients(oracle, amax_bits):
    """Every NVFP4 code of the oracle on the quotient grid (all UE4M3 codes, every bf16
    magnitude within five binades of each block maximum, random signs) equals the nearest
    E2M1 to numpy's IEEE fp32 quotient x / d; every scale equals the nearest UE4M3 (ties
    even) to RN32(amax_b / RN32(6 g)); g = RN32(amax / 2688)."""
    x = synth.nvfp4_quotient_grid(amax_bits, seed=amax_bits)
    e, s, g = oracle.quantize_nvfp4(x)
    xf = synth.bits_to_float(x).astype(np.float32)
    assert g == np.float32(synth.bits_to_float(np.array([amax_bits], dtype=np.uint16))[0]) / np.float32(2688.0)
    blocks = xf.reshape(-1, 16)
    t = np.abs(blocks).max(1) / (np.float32(6.0) * np.float32(g))
    dist = np.abs(UE4M3[None, :] - t.astype(np.float64)[:, None])
    best = dist == dist.min(1, keepdims=True)
    want_sb = np.where(best.sum(1) == 1, best.argmax(1), np.argmax(best & (np.arange(0x7F) % 2 == 0), axis=1))
    assert np.array_equal(s.reshape(-1), want_sb)
    assert np.unique(want_sb).size >= (120 if amax_bits >= 0x0F00 else 20)
    d = UE4M3[want_sb].astype(np.float32) * np.float32(g)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = blocks / d[:, None]
    want = signed_code(blocks, nearest_e2m1(np.abs(np.where(d[:, None] == 0, 0.0, q))))
    want[d == 0] = 0
    got = unpack_fp4(e.reshape(-1), blocks.size).reshape(-1, 16)
    assert np.array_equal(got, want)


def test_oracle_zero_keeps_its_sign(oracle):
    x = synth.normal(2, 32, seed=5)
    x[0, 3] = 0x8000
    x[1, 20] = 0x0000
    e, _, _ = oracle.quantize_nvfp4(x)
    codes = unpack_fp4(e.reshape(-1), 64).reshape(2, 32)
    assert codes[0, 3] == 0x8 and codes[1, 20] == 0x0
