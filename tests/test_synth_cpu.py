"""The seeded input recipes: each generator draws what its docstring and the workload
descriptions state (distributions, outlier and zero fractions, per-row / per-column
scales), deterministically per seed, rounded to bf16 by round-to-nearest-even."""
import numpy as np

import synth


def vals(bits):
    return synth.bits_to_float(bits).astype(np.float64)


def test_deterministic_per_seed_and_seed_sensitive():
    a, b, c = synth.weight_fp4(64, 128, seed=3), synth.weight_fp4(64, 128, seed=3), synth.weight_fp4(64, 128, seed=4)
    assert a.dtype == np.uint16 and a.shape == (64, 128)
    assert np.array_equal(a, b) and not np.array_equal(a, c)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -8 + 2.0 ** -20, -3.0e38], dtype=np.float32)
    got = vals(synth.to_bf16_bits(x))
    # ties go to the even significand; above the tie rounds up; magnitudes keep their sign
    assert got[0] == 1.0 and got[1] == 1.0 + 2.0 ** -6 and got[2] == 1.0 + 2.0 ** -7
    assert got[3] < 0 and abs(got[3] / -3.0e38 - 1) < 2.0 ** -8


def test_weight_recipe():
    x = vals(synth.weight_fp4(1024, 1024, seed=0))
    big = np.abs(x) > 0.2                       # 10 sigma of the bulk: only the N(0, 1) replacements
    frac = big.mean()
    assert 0.0004 < frac < 0.0012               # 0.1% replaced, about 2/3 of them beyond 0.2
    assert abs(x[~big].std() / 0.02 - 1) < 0.02


def test_mx8_recipe():
    x = vals(synth.mx8_rowwise(256, 1024, seed=0))
    # per-row scale 2^u with u in [-8, 8]: log2 of a row's median |x| spans about 16 binades
    med = np.log2(np.median(np.abs(x), axis=1))
    assert med.max() - med.min() > 14 and med.max() - med.min() < 17
    # 1% outliers x100: relative to their row, about 1% of entries exceed 10 row-sigmas
    rel = np.abs(x) / np.median(np.abs(x), axis=1, keepdims=True)
    assert 0.005 < (rel > 15).mean() < 0.012


def test_activation_recipe():
    x = vals(synth.activations(2048, 256, seed=0))
    col = np.log2(x.std(axis=0))
    assert col.min() > -4.2 and col.max() < 4.2 and col.max() - col.min() > 7   # 2^v, v ~ U[-4, 4]
    z = x / x.std(axis=0)                                                        # scales are per column:
    assert abs(z.std(axis=1).mean() - 1) < 0.02                                  # removing them leaves N(0, 1) rows


def test_gradient_recipe():
    x = vals(synth.gradients(1024, 1024, seed=1))
    zero = x == 0
    assert 0.045 < zero.mean() < 0.055
    assert abs(x[~zero].std() / 1e-3 - 1) < 0.02


def test_special_values_cover_the_edges():
    v = vals(synth.special_values_block())
    assert np.any(v == 0) and np.any(np.signbit(v) & (v == 0))                    # +0 and -0
    assert np.any((np.abs(v) > 0) & (np.abs(v) < 2.0 ** -126))                     # subnormals
    assert np.any(np.abs(v) > 3e38)                                                # bf16 extremes
    assert np.any(v == 448.0) and np.any(v == 57344.0)                             # the FP8 maxima
