"""Full-size parity: every output byte of the benchmark-size quantisations, and whole
output tiles plus a point in every tile of the benchmark-size matmuls, against the CPU
oracle (run in row slabs on all host cores).

Quantisation: bit-exact codes and scales.  Matmul: the tolerance of test_gpu_gemm
(1e-3 * sum_k |a b| for the fp32 accumulation plus half a bf16 ulp for the output)."""
import numpy as np
import pytest
import torch

import synth
from oracle_par import (gemm_ref_pairs, gemm_ref_tile, quantize_mx_both, quantize_mx_rows, quantize_mx_sr_rows,
                        quantize_nvfp4_sr_rows, rht16_rows)
from test_gpu_gemm import gemm_tolerance

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import microscaling_precision_number_b200 as mx

FMT_NAMES = {0: "e4m3", 1: "e5m2", 2: "e2m1", 4: "e2m3", 5: "e3m2", 6: "int8"}


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host(t):
    return t.cpu().numpy()


@pytest.fixture(autouse=True)
def _no_watchdog():
    yield
    assert mx.watchdog_status(clear=True) == 0
    torch.cuda.empty_cache()


@pytest.mark.parametrize("which", ["activations", "gradients"])
def test_dual_full_size_every_byte(oracle, which):
    """Dual-orientation MXFP8 of the 16384 x 4096 activations (E4M3) and the 16384 x 14336
    gradients (E5M2), no-clip scales in the tcgen05 tiling -- the benchmark's launch --
    against the oracle's row-wise and column-wise quantisation of the whole tensor."""
    x, fmt = (synth.activations(), 0) if which == "activations" else (synth.gradients(), 1)
    R, C = x.shape
    xd = to_dev(x)
    qr, qc = mx.quantize_dual(xd, FMT_NAMES[fmt], "ceil", "tcgen05")
    re_, rs, ce, cs = quantize_mx_both(oracle, x, fmt, oracle.CEIL)
    assert np.array_equal(host(qr.elems).reshape(R, C), re_)
    assert np.array_equal(host(qc.elems).reshape(C, R), ce)
    assert np.array_equal(host(qr.scales), oracle.to_tcgen05_layout(rs))
    assert np.array_equal(host(qc.scales), oracle.to_tcgen05_layout(cs))
    del qr, qc
    # both scale layouts from the same single pass
    qr, qc = mx.quantize_dual(xd, FMT_NAMES[fmt], "ceil", "both")
    assert np.array_equal(host(qr.scales).reshape(R, C // 32), rs)
    assert np.array_equal(host(qc.scales).reshape(C, R // 32), cs)
    assert np.array_equal(host(qr.scales_alt), oracle.to_tcgen05_layout(rs))
    assert np.array_equal(host(qc.scales_alt), oracle.to_tcgen05_layout(cs))
    assert np.array_equal(host(qc.elems).reshape(C, R), ce)


@pytest.mark.parametrize("fmt", ["nvfp4", "e2m1"])
def test_train_16384x14336_every_byte(oracle, fmt):
    """The training quantiser in the benchmark's launch: the 16384 x 14336 gradient shape
    (N(0, 1e-3) values), the 16 x 16 transform with signs 0xB5C3 and stochastic rounding
    from one random byte per element, tcgen05 scales -- every code and scale byte against
    the oracle's transform followed by its quantisation, in row slabs."""
    R, C = 16384, 14336
    x = synth.normal(R, C, sigma=1e-3, seed=70)
    rnd = np.random.default_rng(71).integers(0, 256, size=(R, C), dtype=np.uint8)
    rounding = "ceil" if fmt == "nvfp4" else "floor"
    q = mx.quantize_train(to_dev(x), fmt, rounding, rht_signs=0xB5C3, sr_random=torch.from_numpy(rnd).cuda(),
                          layout="tcgen05")
    xt = rht16_rows(oracle, x, 0xB5C3)
    if fmt == "nvfp4":
        e, s, g = quantize_nvfp4_sr_rows(oracle, xt, rnd)
        assert host(q.global_scale)[0] == np.float32(g)
    else:
        e, s = quantize_mx_sr_rows(oracle, xt, 2, oracle.FLOOR, rnd)
    assert np.array_equal(host(q.elems).reshape(R, -1), e)
    assert np.array_equal(host(q.scales), oracle.to_tcgen05_layout(s))


@pytest.mark.parametrize("fmt", [4, 5, 6])
def test_rowwise_mxfp6_mxint8_16384x4096_every_byte(oracle, fmt):
    """MXFP6 (E2M3, E3M2; packed 6-bit codes) and MXINT8 row-wise quantisation of the
    16384 x 4096 activations, both scale layouts."""
    x = synth.activations()
    R, C = x.shape
    q = mx.quantize(to_dev(x), FMT_NAMES[fmt], "row", "ceil", layout="both")
    e, s = quantize_mx_rows(oracle, x, fmt, oracle.CEIL)
    assert np.array_equal(host(q.elems), e.reshape(-1))
    assert np.array_equal(host(q.scales), s.reshape(-1))
    assert np.array_equal(host(q.scales_alt), oracle.to_tcgen05_layout(s))


@pytest.mark.parametrize("fmt,rounding", [(0, "ceil"), (2, "floor")])
def test_colwise_16384x4096_every_byte(oracle, fmt, rounding):
    """Column-wise only (mx_quantize with axis = COL), both scale layouts."""
    x = synth.activations()
    R, C = x.shape
    q = mx.quantize(to_dev(x), FMT_NAMES[fmt], "col", rounding, layout="both")
    e, s = quantize_mx_rows(oracle, np.ascontiguousarray(x.T), fmt, oracle.CEIL if rounding == "ceil" else oracle.FLOOR)
    assert np.array_equal(host(q.elems), e.reshape(-1))
    assert np.array_equal(host(q.scales), s.reshape(-1))
    assert np.array_equal(host(q.scales_alt), oracle.to_tcgen05_layout(s))


def test_colwise_gradients_back_to_back(oracle):
    """Column-wise only on the 16384 x 14336 gradients (E5M2, tcgen05 scales), launched 12
    times back to back into separate outputs: the two consumer warp groups take alternate
    ring tiles there, so each launch must equal the oracle (launch-to-launch timing must not
    change a byte)."""
    x = synth.gradients()
    xd = to_dev(x)
    outs = [mx.quantize(xd, "e5m2", "col", "ceil", layout="tcgen05") for _ in range(12)]
    torch.cuda.synchronize()
    e, s = quantize_mx_rows(oracle, np.ascontiguousarray(x.T), 1, oracle.CEIL)
    assert np.array_equal(host(outs[0].elems), e.reshape(-1))
    assert np.array_equal(host(outs[0].scales), oracle.to_tcgen05_layout(s))
    for q in outs[1:]:
        assert torch.equal(q.elems, outs[0].elems)
        assert torch.equal(q.scales, outs[0].scales)


def _check(got, ref, mag, where):
    err = np.abs(got - ref)
    bad = np.nonzero(~(err <= gemm_tolerance(ref, mag)))
    assert bad[0].size == 0, f"{where}: {bad[0].size} entries out of tolerance"
    rounded = torch.from_numpy(ref).to(torch.float32).to(torch.bfloat16).double().numpy()
    assert np.mean(got == rounded) >= 0.95, where


@pytest.mark.parametrize("case", ["e4m3_8192", "e4m3_x_e2m1_8192x14336x4096"])
def test_gemm_full_tiles_and_every_tile(oracle, case):
    """The benchmark's matmuls: the first and the last 256 x 256 output tile complete, one
    random point inside every 128 x 256 tile, the four corners of a grid of tile edges,
    and 2,000 random entries."""
    if case == "e4m3_8192":
        (M, N, K), b_fmt, sig, seeds = (8192, 8192, 8192), 0, 1.0, (40, 41)
    else:
        (M, N, K), b_fmt, sig, seeds = (8192, 14336, 4096), 2, 0.02, (50, 51)
    a_bits = synth.normal(M, K, seed=seeds[0])
    b_bits = synth.normal(N, K, sigma=sig, seed=seeds[1])
    a = mx.quantize(to_dev(a_bits), "e4m3", "row", "ceil", layout="tcgen05")
    b = mx.quantize(to_dev(b_bits), FMT_NAMES[b_fmt], "row", "floor" if b_fmt == 2 else "ceil", layout="tcgen05")
    c = mx.gemm(a, b).float().cpu().numpy().astype(np.float64)
    del a, b
    ae, as_ = quantize_mx_rows(oracle, a_bits, 0, oracle.CEIL)
    be, bs = quantize_mx_rows(oracle, b_bits, b_fmt, oracle.FLOOR if b_fmt == 2 else oracle.CEIL)
    for m0, n0 in ((0, 0), (M - 256, N - 256)):
        ref, mag = gemm_ref_tile(oracle, ae, as_, 0, be, bs, b_fmt, M, N, K, m0, m0 + 256, n0, n0 + 256)
        _check(c[m0:m0 + 256, n0:n0 + 256], ref, mag, f"tile ({m0}, {n0})")
    rng = np.random.default_rng(7)
    tm, tn = np.meshgrid(np.arange(M // 128), np.arange(N // 256), indexing="ij")
    every = np.stack([tm.reshape(-1) * 128 + rng.integers(0, 128, tm.size),
                      tn.reshape(-1) * 256 + rng.integers(0, 256, tn.size)], axis=1)
    edges = np.array([(m, n) for m in (127, 128, M // 2 - 1, M // 2, M - 129, M - 128)
                      for n in (255, 256, N // 2 - 1, N // 2, N - 257, N - 256)])
    rand = np.stack([rng.integers(0, M, 2000), rng.integers(0, N, 2000)], axis=1)
    pairs = np.concatenate([every, edges, rand]).astype(np.int64)
    ref, mag = gemm_ref_pairs(oracle, ae, as_, 0, be, bs, b_fmt, M, N, K, pairs)
    _check(c[pairs[:, 0], pairs[:, 1]], ref, mag, "sampled entries")
