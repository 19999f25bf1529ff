"""GPU parity of the NVFP4 element step on the quotient grid: every UE4M3 block-scale
code, every bf16 magnitude within five binades of each block maximum (random signs),
for per-tensor scales from fp32-subnormal to the bf16 maximum.  The kernels form the
correctly rounded fp32 quotient x / d (Markstein's corrected quotient when d >= 2^-100,
the IEEE division below); the oracle divides.  Codes, scales and g must match bit for
bit, for the streaming quantiser, the training quantiser (round to nearest and
stochastic rounding) and the 16 x 16 weight-block quantiser."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import microscaling_precision_number_b200 as mx

# tensor maxima (bf16 patterns): g = amax / 2688 from fp32-subnormal (first four) through
# the band where d = dec(sb) g crosses 2^-100 (0x0E80 .. 0x1780) up to the bf16 maximum
AMAX = [0x0001, 0x0040, 0x0088, 0x0400, 0x0C2A, 0x0E80, 0x0F00, 0x1000, 0x1191, 0x1400, 0x1600, 0x1780,
        0x1880, 0x2000, 0x2ABC, 0x3A83, 0x3C23, 0x3F80, 0x4528, 0x4B37, 0x5A5A, 0x6F00, 0x7F7F]


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host(t):
    return t.cpu().numpy()


@pytest.fixture(autouse=True)
def _no_watchdog():
    yield
    assert mx.watchdog_status(clear=True) == 0


@pytest.mark.parametrize("amax_bits", AMAX)
def test_nvfp4_quotient_grid(oracle, amax_bits):
    x = synth.nvfp4_quotient_grid(amax_bits, seed=amax_bits)
    q = mx.quantize(to_dev(x), "nvfp4", "row", "ceil", layout="both")
    e, s, g = oracle.quantize_nvfp4(x)
    assert host(q.global_scale)[0] == np.float32(g)
    assert np.array_equal(host(q.scales), s.reshape(-1))
    assert np.array_equal(host(q.elems), e.reshape(-1))
    assert np.array_equal(host(q.scales_alt), oracle.to_tcgen05_layout(s))


@pytest.mark.parametrize("amax_bits", [0x0088, 0x0F00, 0x1191, 0x1600, 0x3C23, 0x4528, 0x7F7F])
def test_nvfp4_train_quotient_grid(oracle, amax_bits):
    """The training quantiser without transform: round to nearest equals the streaming
    path's codes; stochastic rounding equals the oracle's (the quotients are formed with
    the opposite sign in the kernel, so this also checks that the rounding is symmetric)."""
    x = synth.nvfp4_quotient_grid(amax_bits, seed=amax_bits + 1)
    xd = to_dev(x)
    e, s, g = oracle.quantize_nvfp4(x)
    q = mx.quantize_train(xd, "nvfp4", "ceil", layout="rowmajor")
    assert host(q.global_scale)[0] == np.float32(g)
    assert np.array_equal(host(q.scales), s.reshape(-1))
    assert np.array_equal(host(q.elems), e.reshape(-1))
    rnd = np.random.default_rng(amax_bits).integers(0, 256, x.shape, dtype=np.uint8)
    es, ss, gs = oracle.quantize_nvfp4_sr(x, rnd)
    q = mx.quantize_train(xd, "nvfp4", "ceil", sr_random=torch.from_numpy(rnd).cuda(), layout="rowmajor")
    assert host(q.global_scale)[0] == np.float32(gs)
    assert np.array_equal(host(q.scales), ss.reshape(-1))
    assert np.array_equal(host(q.elems), es.reshape(-1))


@pytest.mark.parametrize("amax_bits", [0x0088, 0x1191, 0x3C23, 0x4528])
def test_nvfp4_2d_quotient_grid(oracle, amax_bits):
    x = synth.nvfp4_quotient_grid(amax_bits, seed=amax_bits + 2)
    x = x[: x.shape[0] // 16 * 16]
    q = mx.quantize_nvfp4_2d(to_dev(x), layout="rowmajor")
    e, s, g = oracle.quantize_nvfp4_2d(x)
    assert host(q.global_scale)[0] == np.float32(g)
    assert np.array_equal(host(q.scales), s.reshape(-1))
    assert np.array_equal(host(q.elems), e.reshape(-1))
