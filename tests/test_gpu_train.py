"""GPU parity of the training-side quantiser (16 x 16 random Hadamard transform and
stochastic rounding, row-wise MX and NVFP4) against the oracle's composition of its
pinned transform and its pinned rounding, bit for bit."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import microscaling_precision_number_b200 as mx

FMT = {"e4m3": 0, "e5m2": 1, "e2m1": 2, "nvfp4": 3}


@pytest.fixture(autouse=True)
def _no_watchdog():
    yield
    assert mx.watchdog_status(clear=True) == 0


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def with_specials(x, seed):
    x = x.copy()
    rng = np.random.default_rng(seed)
    sp = synth.special_values_block()
    idx = rng.choice(x.size, size=min(x.size // 9, 40), replace=False)
    x.reshape(-1)[idx] = sp[rng.integers(0, sp.size, size=idx.size)]
    return x


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2", "e2m1", "nvfp4"])
@pytest.mark.parametrize("rht,sr", [(True, False), (False, True), (True, True), (False, False)])
@pytest.mark.parametrize("shape", [(64, 256), (130, 512)])
def test_train_quantiser_matches_oracle(oracle, fmt, rht, sr, shape):
    x = with_specials(synth.gradients(*shape, seed=shape[0] + 3), seed=shape[1])
    rounding = "floor" if fmt == "e2m1" else "ceil"
    rnd = np.random.default_rng(shape[0]).integers(0, 256, size=shape, dtype=np.uint8) if sr else None
    signs = 0xA53C if rht else None
    q = mx.quantize_train(to_dev(x), fmt, rounding, rht_signs=signs,
                          sr_random=None if rnd is None else torch.from_numpy(rnd).cuda(), layout="both")
    xt = oracle.rht16(x, signs) if rht else x
    f = FMT[fmt]
    rnd_o = oracle.CEIL if rounding == "ceil" else oracle.FLOOR
    if fmt == "nvfp4":
        e, s, g = oracle.quantize_nvfp4_sr(xt, rnd) if sr else oracle.quantize_nvfp4(xt)
        assert q.global_scale.cpu().numpy()[0] == np.float32(g)
    else:
        e, s = oracle.quantize_mx_sr(xt, f, rnd_o, rnd) if sr else oracle.quantize_mx(xt, f, oracle.ROW, rnd_o)
    assert np.array_equal(q.elems.cpu().numpy(), e.reshape(-1))
    assert np.array_equal(q.scales.cpu().numpy(), s.reshape(-1))
    assert np.array_equal(q.scales_alt.cpu().numpy(), oracle.to_tcgen05_layout(s))


@pytest.mark.parametrize("rht,sr", [(True, True), (False, True), (True, False)])
@pytest.mark.parametrize("shape", [(33, 208), (1, 16), (3, 48)])
def test_train_nvfp4_odd_block_count(oracle, rht, sr, shape):
    """NVFP4 with an odd number of 16-element blocks (the quantisation pass takes two blocks
    per thread; the last thread has one), row-major and tcgen05 scales."""
    x = with_specials(synth.gradients(*shape, seed=shape[0] + 11), seed=shape[1] + 1)
    rnd = np.random.default_rng(shape[1]).integers(0, 256, size=shape, dtype=np.uint8) if sr else None
    signs = 0x5AC3 if rht else None
    q = mx.quantize_train(to_dev(x), "nvfp4", "ceil", rht_signs=signs,
                          sr_random=None if rnd is None else torch.from_numpy(rnd).cuda(), layout="both")
    xt = oracle.rht16(x, signs) if rht else x
    e, s, g = oracle.quantize_nvfp4_sr(xt, rnd) if sr else oracle.quantize_nvfp4(xt)
    assert q.global_scale.cpu().numpy()[0] == np.float32(g)
    assert np.array_equal(q.elems.cpu().numpy(), e.reshape(-1))
    assert np.array_equal(q.scales.cpu().numpy(), s.reshape(-1))
    assert np.array_equal(q.scales_alt.cpu().numpy(), oracle.to_tcgen05_layout(s))


@pytest.mark.parametrize("fmt", ["nvfp4", "e2m1", "e4m3"])
@pytest.mark.parametrize("sr", [False, True])
def test_train_transform_nonfinite(oracle, fmt, sr):
    """The transform meets Inf, NaN and fp32 overflow: groups holding +Inf, -Inf or NaN, two
    largest-finite bf16 values whose butterfly sums overflow to Inf, and a pair whose sum
    cancels while the difference overflows.  The tensor maximum (NVFP4) is taken over the
    finite transformed values only; bit for bit against the oracle."""
    x = synth.gradients(64, 256, seed=91)
    big, nbig = 0x7F7F, 0xFF7F
    plants = {(0, 3): 0x7F80, (1, 20): 0xFF80, (2, 40): 0x7FC0,          # +Inf, -Inf, NaN
              (3, 64): big, (3, 65): big,                                   # sums overflow
              (4, 96): big, (4, 104): nbig,                                 # cancel / overflow
              (5, 130): big, (6, 200): nbig}                                # lone extremes
    for (r, c), v in plants.items():
        x[r, c] = v
    shape = x.shape
    rnd = np.random.default_rng(92).integers(0, 256, size=shape, dtype=np.uint8) if sr else None
    rounding = "floor" if fmt == "e2m1" else "ceil"
    q = mx.quantize_train(to_dev(x), fmt, rounding, rht_signs=0x9E37,
                          sr_random=None if rnd is None else torch.from_numpy(rnd).cuda(), layout="both")
    xt = oracle.rht16(x, 0x9E37)
    if fmt == "nvfp4":
        e, s, g = oracle.quantize_nvfp4_sr(xt, rnd) if sr else oracle.quantize_nvfp4(xt)
        assert q.global_scale.cpu().numpy()[0] == np.float32(g)
    else:
        rnd_o = oracle.CEIL if rounding == "ceil" else oracle.FLOOR
        e, s = oracle.quantize_mx_sr(xt, FMT[fmt], rnd_o, rnd) if sr else oracle.quantize_mx(xt, FMT[fmt], oracle.ROW, rnd_o)
    assert np.array_equal(q.elems.cpu().numpy(), e.reshape(-1))
    assert np.array_equal(q.scales.cpu().numpy(), s.reshape(-1))
    assert np.array_equal(q.scales_alt.cpu().numpy(), oracle.to_tcgen05_layout(s))


def test_oracle_transform_overflows_where_planted(oracle):
    """CPU-side check that the planted pairs above do drive the fp32 butterfly to Inf (so
    the test reaches the kernels' non-finite path)."""
    x = synth.gradients(64, 256, seed=91)
    x[3, 64] = x[3, 65] = 0x7F7F
    xt = oracle.rht16(x, 0x9E37)
    assert np.any((xt[3, 64:80] & 0x7FFF) == 0x7F80)


@pytest.mark.parametrize("fmt", ["e2m1", "nvfp4"])
def test_train_quantiser_multi_cta(oracle, fmt):
    """A gradient of the benchmark's width (1024 x 14336) with the transform and stochastic
    rounding: the grid is capped, so every CTA walks several blocks (grid-stride loops) and
    NVFP4's tensor maximum comes from many partial maxima -- bit for bit as above."""
    shape = (1024, 14336)
    x = synth.gradients(*shape, seed=77)
    rnd = np.random.default_rng(78).integers(0, 256, size=shape, dtype=np.uint8)
    rounding = "floor" if fmt == "e2m1" else "ceil"
    q = mx.quantize_train(to_dev(x), fmt, rounding, rht_signs=0xB5C3, sr_random=torch.from_numpy(rnd).cuda(),
                          layout="tcgen05")
    xt = oracle.rht16(x, 0xB5C3)
    if fmt == "nvfp4":
        e, s, g = oracle.quantize_nvfp4_sr(xt, rnd)
        assert q.global_scale.cpu().numpy()[0] == np.float32(g)
    else:
        e, s = oracle.quantize_mx_sr(xt, FMT[fmt], oracle.FLOOR, rnd)
    assert np.array_equal(q.elems.cpu().numpy(), e.reshape(-1))
    assert np.array_equal(q.scales.cpu().numpy(), oracle.to_tcgen05_layout(s))


def test_rht_keeps_the_matmul(oracle):
    """The same transform on both operands along K leaves A * B^T unchanged up to the
    quantisation (the property that makes it usable on weight-gradient inputs)."""
    M, N, K = 256, 256, 512
    a = synth.normal(M, K, seed=1)
    b = synth.normal(N, K, seed=2)
    ref = mx.gemm(mx.quantize(to_dev(a), "e4m3", "row", "ceil", layout="tcgen05"),
                  mx.quantize(to_dev(b), "e4m3", "row", "ceil", layout="tcgen05")).float()
    got = mx.gemm(mx.quantize_train(to_dev(a), "e4m3", "ceil", rht_signs=0x5A0F),
                  mx.quantize_train(to_dev(b), "e4m3", "ceil", rht_signs=0x5A0F)).float()
    exact = to_dev(a).float() @ to_dev(b).float().T
    rel_ref = ((ref - exact).norm() / exact.norm()).item()
    rel_got = ((got - exact).norm() / exact.norm()).item()
    assert rel_got < 3 * rel_ref + 1e-3, (rel_got, rel_ref)
