"""GPU parity of the tcgen05 block-scaled matmul against the oracle's fp64 reference over
its own dequantised operands.

Tolerance: the fp32 accumulation may differ from the fp64 sum by 1e-3 * sum_k |a_mk b_nk|
(the bound the MX matmul is specified to), and the bf16 output then rounds that fp32
value once more, by at most half a bf16 ulp.  So every checked entry must satisfy
    |C_gpu - C_ref| <= 1e-3 * sum_k |a b| + half_ulp_bf16(|C_ref| + 1e-3 * sum_k |a b|).
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import microscaling_precision_number_b200 as mx

TOL = 1e-3


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_to_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def half_ulp_bf16(x):
    """Half the spacing of bf16 numbers at magnitude x (8 significant bits)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -133)))
    return 2.0 ** (np.maximum(e, -126) - 8)


def gemm_tolerance(ref, mag):
    acc = TOL * mag
    return acc + half_ulp_bf16(np.abs(ref) + acc)


@pytest.fixture(autouse=True)
def _no_watchdog():
    yield
    assert mx.watchdog_status(clear=True) == 0


def run_case(oracle, a_bits, b_bits, b_fmt, pairs=None):
    M, K = a_bits.shape
    N = b_bits.shape[0]
    a_q = mx.quantize(to_dev(a_bits), "e4m3", "row", "ceil", layout="tcgen05")
    b_q = mx.quantize(to_dev(b_bits), "e2m1" if b_fmt == oracle.E2M1 else "e4m3", "row",
                      "floor" if b_fmt == oracle.E2M1 else "ceil", layout="tcgen05")
    c = bf16_to_f64(mx.gemm(a_q, b_q))
    if pairs is None:
        pairs = np.array([(m, n) for m in range(M) for n in range(N)], dtype=np.int64)
    # the oracle quantises the bf16 inputs itself; only the rows it needs
    rows_a = np.unique(pairs[:, 0])
    rows_b = np.unique(pairs[:, 1])
    ae, as_ = oracle.quantize_mx(a_bits[rows_a], oracle.E4M3, oracle.ROW, oracle.CEIL)
    be, bs = oracle.quantize_mx(b_bits[rows_b], b_fmt, oracle.ROW,
                                oracle.FLOOR if b_fmt == oracle.E2M1 else oracle.CEIL)
    ia = {int(r): i for i, r in enumerate(rows_a)}
    ib = {int(r): i for i, r in enumerate(rows_b)}
    local = np.array([(ia[int(m)], ib[int(n)]) for m, n in pairs], dtype=np.int64)
    ref, mag = oracle.gemm_ref(ae, as_, oracle.E4M3, be, bs, b_fmt, len(rows_a), len(rows_b), K, local)
    got = c[pairs[:, 0], pairs[:, 1]]
    err = np.abs(got - ref)
    bound = gemm_tolerance(ref, mag)
    bad = np.nonzero(~(err <= bound))[0]
    assert bad.size == 0, (f"{bad.size}/{len(pairs)} entries out of tolerance; first "
                           f"{[(tuple(pairs[i]), got[i], ref[i], mag[i]) for i in bad[:4]]}")
    # fp32 accumulation error is far below a bf16 ulp here: nearly every entry is the
    # correctly rounded bf16 of the fp64 reference
    rounded = torch.from_numpy(ref).to(torch.float32).to(torch.bfloat16).double().numpy()
    assert np.mean(got == rounded) >= 0.95, f"only {np.mean(got == rounded):.3f} of entries round-exact"
    return err, mag


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (128, 128, 128), (256, 512, 512), (384, 384, 256),
                                   (128, 256, 1024)])
def test_gemm_e4m3_small(oracle, M, N, K):
    a = synth.normal(M, K, seed=M + K)
    b = synth.normal(N, K, seed=N + 1)
    run_case(oracle, a, b, oracle.E4M3)


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (128, 128, 256), (256, 512, 512)])
def test_gemm_mixed_fp4_small(oracle, M, N, K):
    a = synth.normal(M, K, seed=M)
    b = synth.weight_fp4(N, K, seed=N)
    run_case(oracle, a, b, oracle.E2M1)


def test_gemm_exact_scaled_one_hot(oracle):
    """One nonzero per A row at a varying k: C is an exact scaled copy of B's column."""
    M, N, K = 128, 256, 256
    a = np.zeros((M, K), dtype=np.uint16)
    vals = [0x3F80, 0x4300, 0xC1C0, 0x3E00]              # 1, 128, -24, 0.125
    for m in range(M):
        a[m, (m * 37) % K] = vals[m % 4]
    b = synth.mx8_rowwise(N, K, seed=2)
    for b_fmt in (oracle.E4M3, oracle.E2M1):
        err, _ = run_case(oracle, a, b, b_fmt)


def test_gemm_wide_dynamic_range(oracle):
    """Rows spanning 2^-8 .. 2^8 with outliers (the MX8 row-wise workload's statistics)."""
    a = synth.mx8_rowwise(256, 512, seed=4)
    b = synth.mx8_rowwise(256, 512, seed=5)
    run_case(oracle, a, b, oracle.E4M3)


def sample_pairs(M, N, n, seed):
    rng = np.random.default_rng(seed)
    p = np.stack([rng.integers(0, M, n), rng.integers(0, N, n)], axis=1)
    corners = np.array([(0, 0), (0, N - 1), (M - 1, 0), (M - 1, N - 1), (127, 255), (128, 256)])
    return np.concatenate([p, corners]).astype(np.int64)


def test_config4_gemm_8192_sampled(oracle):
    M = N = K = 8192
    a = synth.normal(M, K, seed=40)
    b = synth.normal(N, K, seed=41)
    run_case(oracle, a, b, oracle.E4M3, sample_pairs(M, N, 192, 4))
    torch.cuda.empty_cache()


def test_config5_gemm_mixed_sampled(oracle):
    M, N, K = 8192, 14336, 4096
    a = synth.normal(M, K, seed=50)
    b = synth.normal(N, K, sigma=0.02, seed=51)
    run_case(oracle, a, b, oracle.E2M1, sample_pairs(M, N, 192, 5))
    torch.cuda.empty_cache()
