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


GPU_FMT = {0: "e4m3", 1: "e5m2", 2: "e2m1", 3: "nvfp4", 4: "e2m3", 5: "e3m2"}


def _gpu_quant(bits, fmt):
    rounding = "floor" if fmt == 2 else "ceil"      # MXFP4 weights: OCP floor; MXFP8: the recipe's
    return mx.quantize(to_dev(bits), GPU_FMT[fmt], "row", rounding, layout="tcgen05")


def _oracle_quant(oracle, bits, rows, fmt):
    """Oracle codes and scales of the given rows.  NVFP4's per-tensor scale depends on the
    whole tensor, so the row holding the tensor's largest finite |x| is quantised with the
    subset (block scales and codes are per row, so the other rows are unchanged)."""
    if fmt != oracle.NVFP4:
        e, s = oracle.quantize_mx(bits[rows], fmt, oracle.ROW, oracle.FLOOR if fmt == oracle.E2M1 else oracle.CEIL)
        return e, s, 1.0
    mag = (bits & 0x7FFF).astype(np.int64)
    mag[mag >= 0x7F80] = -1
    top = int(np.argmax(mag) // bits.shape[1])
    e, s, g = oracle.quantize_nvfp4(np.ascontiguousarray(np.concatenate([bits[rows], bits[top:top + 1]])))
    return e[:len(rows)], s[:len(rows)], g


def run_case(oracle, a_bits, b_bits, b_fmt, pairs=None, a_fmt=None):
    a_fmt = oracle.E4M3 if a_fmt is None else a_fmt
    M, K = a_bits.shape
    N = b_bits.shape[0]
    c = bf16_to_f64(mx.gemm(_gpu_quant(a_bits, a_fmt), _gpu_quant(b_bits, b_fmt)))
    if pairs is None:
        pairs = np.array([(m, n) for m in range(M) for n in range(N)], dtype=np.int64)
    # the oracle quantises the bf16 inputs itself; only the rows it needs
    rows_a = np.unique(pairs[:, 0])
    rows_b = np.unique(pairs[:, 1])
    ae, as_, ga = _oracle_quant(oracle, a_bits, rows_a, a_fmt)
    be, bs, gb = _oracle_quant(oracle, b_bits, rows_b, b_fmt)
    ia = {int(r): i for i, r in enumerate(rows_a)}
    ib = {int(r): i for i, r in enumerate(rows_b)}
    local = np.array([(ia[int(m)], ib[int(n)]) for m, n in pairs], dtype=np.int64)
    ref, mag = oracle.gemm_ref(ae, as_, a_fmt, be, bs, b_fmt, len(rows_a), len(rows_b), K, local, a_g=ga, b_g=gb)
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


def test_gemm_e4m3_8192_sampled(oracle):
    M = N = K = 8192
    a = synth.normal(M, K, seed=40)
    b = synth.normal(N, K, seed=41)
    run_case(oracle, a, b, oracle.E4M3, sample_pairs(M, N, 192, 4))
    torch.cuda.empty_cache()


def test_gemm_e4m3_x_e2m1_8192x14336x4096_sampled(oracle):
    M, N, K = 8192, 14336, 4096
    a = synth.normal(M, K, seed=50)
    b = synth.normal(N, K, sigma=0.02, seed=51)
    run_case(oracle, a, b, oracle.E2M1, sample_pairs(M, N, 192, 5))
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ FP4 x FP4 (kind::mxf4, kind::mxf4nvf4)
@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (128, 128, 256), (256, 512, 512), (384, 384, 768)])
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_gemm_fp4_x_fp4_small(oracle, M, N, K, fmt):
    f = oracle.E2M1 if fmt == "mxfp4" else oracle.NVFP4
    a = synth.normal(M, K, seed=M + 7)
    b = synth.weight_fp4(N, K, seed=N + 8)
    run_case(oracle, a, b, f, a_fmt=f)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_gemm_fp4_x_fp4_one_hot(oracle, fmt):
    """One nonzero per A row (exactly representable): C is a scaled copy of B's column,
    which checks the placement of every scale byte along K."""
    f = oracle.E2M1 if fmt == "mxfp4" else oracle.NVFP4
    M, N, K = 128, 256, 512
    a = np.zeros((M, K), dtype=np.uint16)
    vals = [0x3F80, 0x4040, 0xC0C0, 0x3F00]              # 1, 3, -6, 0.5
    for m in range(M):
        a[m, (m * 37) % K] = vals[m % 4]
    b = synth.mx8_rowwise(N, K, seed=3)
    run_case(oracle, a, b, f, a_fmt=f)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_gemm_fp4_x_fp4_8192_sampled(oracle, fmt):
    f = oracle.E2M1 if fmt == "mxfp4" else oracle.NVFP4
    M = N = K = 8192
    a = synth.normal(M, K, seed=60)
    b = synth.normal(N, K, sigma=0.02, seed=61)
    run_case(oracle, a, b, f, sample_pairs(M, N, 128, 6), a_fmt=f)
    torch.cuda.empty_cache()


def test_gemm_rejects_unsupported_pairs():
    x = to_dev(synth.normal(128, 256, seed=1))
    e4 = mx.quantize(x, "e4m3", "row", "ceil", layout="tcgen05")
    n4 = mx.quantize(x, "nvfp4", "row", "ceil", layout="tcgen05")
    f4 = mx.quantize(x, "e2m1", "row", "floor", layout="tcgen05")
    for a, b in ((f4, e4), (n4, f4), (e4, n4)):
        with pytest.raises(mx.MxError):
            mx.gemm(a, b)


# ------------------------------------------------------------------ FP6 and E5M2 operands (kind::mxf8f6f4)
@pytest.mark.parametrize("a_fmt,b_fmt", [(4, 4), (5, 2), (1, 0), (0, 5), (4, 1)])
@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (128, 384, 256)])
def test_gemm_fp6_fp8_operand_pairs(oracle, a_fmt, b_fmt, M, N, K):
    """MXFP6 (E2M3, E3M2) and E5M2 operands run on the same tensor-core kind as MXFP8 (the
    first shape uses CTA pairs, the second single CTAs)."""
    a = synth.normal(M, K, seed=M + a_fmt)
    b = synth.weight_fp4(N, K, seed=N + b_fmt) if b_fmt == 2 else synth.normal(N, K, seed=N + b_fmt)
    run_case(oracle, a, b, b_fmt, a_fmt=a_fmt)


# ------------------------------------------------------------------ an outside check of the scale tiling
def _scaled_mm(a, b, M, N, K):
    return torch._scaled_mm(a.elems.view(torch.float8_e4m3fn).view(M, K),
                            b.elems.view(torch.float8_e4m3fn).view(N, K).t(),
                            scale_a=a.scales.view(torch.float8_e8m0fnu),
                            scale_b=b.scales.view(torch.float8_e8m0fnu), out_dtype=torch.bfloat16)


def exact_operand(rows, K, seed):
    """bf16 entries k * 2^e with k in {-2 .. 2} and one exponent e in {-1, 0, 1} per 32-block:
    they quantise to E4M3 exactly under varied E8M0 scales, every partial sum of the
    matmul is a multiple of 2^-2 below 2^14 (an exact fp32 in any summation order), and a
    product with a misplaced scale byte lands elsewhere."""
    rng = np.random.default_rng(seed)
    k = rng.integers(-2, 3, (rows, K)).astype(np.float32)
    e = np.repeat(rng.integers(-1, 2, (rows, K // 32)), 32, axis=1).astype(np.float32)
    v = k * np.exp2(e)
    return synth.to_bf16_bits(v), v.astype(np.float64)


@pytest.mark.parametrize("M,N,K", [(256, 256, 512), (512, 384, 1024), (1024, 1024, 1024)])
def test_scale_tiling_exact_against_cublaslt(M, N, K):
    """The tcgen05 scale tiling is not defined by the pages; cuBLASLt's MXFP8 block-scaled
    matmul (through torch._scaled_mm) takes its E8M0 scales in the same 128 x 4 atom
    layout.  On operands whose products and sums are exact in fp32, both matmuls, fed the
    very bytes this library's quantiser writes, must give exactly the bf16 of the exact
    product -- bit for bit, whatever their accumulation order.  Skipped when this torch /
    cuBLAS lacks the call."""
    ab, av = exact_operand(M, K, M + K)
    bb, bv = exact_operand(N, K, N + 2 * K)
    ref = torch.from_numpy(av @ bv.T).to(torch.float32).to(torch.bfloat16)
    a = mx.quantize(to_dev(ab), "e4m3", "row", "ceil", layout="tcgen05")
    b = mx.quantize(to_dev(bb), "e4m3", "row", "ceil", layout="tcgen05")
    ours = mx.gemm(a, b).cpu()
    assert torch.equal(ours, ref)
    try:
        lib = _scaled_mm(a, b, M, N, K).cpu()
    except (RuntimeError, TypeError, AttributeError) as e:      # the library call itself is unavailable
        pytest.skip(f"torch._scaled_mm MXFP8 unavailable: {e}")
    assert torch.equal(lib, ref)


def test_scale_tiling_agrees_with_cublaslt_8192():
    """The benchmark's 8192^3 E4M3 operands (N(0, 1)): cuBLASLt's MXFP8 matmul, fed this
    library's tcgen05-tiled scales, gives a bit-identical product (the two kernels
    accumulate each output in the same K order)."""
    M = N = K = 8192
    a = mx.quantize(to_dev(synth.normal(M, K, seed=40)), "e4m3", "row", "ceil", layout="tcgen05")
    b = mx.quantize(to_dev(synth.normal(N, K, seed=41)), "e4m3", "row", "ceil", layout="tcgen05")
    ours = mx.gemm(a, b)
    try:
        lib = _scaled_mm(a, b, M, N, K)
    except (RuntimeError, TypeError, AttributeError) as e:
        pytest.skip(f"torch._scaled_mm MXFP8 unavailable: {e}")
    assert torch.equal(ours, lib)
    del a, b, ours, lib
    torch.cuda.empty_cache()
