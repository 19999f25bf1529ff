"""GPU parity of the quantisers, dequantisers and the direct cast against the CPU oracle,
through the C ABI.  Element codes and scales must match bit for bit; dequantised values
bit for bit (NaN matched as NaN)."""
import numpy as np
import pytest
import torch

import synth
from conftest import pack_codes

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import microscaling_precision_number_b200 as mx
    from microscaling_precision_number_b200 import _lib as L

FMT_NAMES = {0: "e4m3", 1: "e5m2", 2: "e2m1", 4: "e2m3", 5: "e3m2", 6: "int8"}


def to_dev(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def nan_aware_equal(a_bits: np.ndarray, b_bits: np.ndarray) -> bool:
    a_nan = ((a_bits & 0x7F80) == 0x7F80) & ((a_bits & 0x7F) != 0)
    b_nan = ((b_bits & 0x7F80) == 0x7F80) & ((b_bits & 0x7F) != 0)
    return bool(np.array_equal(a_nan, b_nan) and np.array_equal(a_bits[~a_nan], b_bits[~b_nan]))


def with_specials(x: np.ndarray, seed: int) -> np.ndarray:
    """Sprinkle edge values (zeros, subnormals, huge, Inf, NaN) and an all-zero block."""
    x = x.copy()
    rng = np.random.default_rng(seed)
    sp = synth.special_values_block()
    idx = rng.choice(x.size, size=min(x.size // 7, 64), replace=False)
    x.reshape(-1)[idx] = sp[rng.integers(0, sp.size, size=idx.size)]
    if x.shape[1] >= 32:
        x[0, :32] = 0
        x[0, 5] = 0x8000      # -0 in an otherwise zero block
    return x


SHAPES = [(1, 32), (3, 64), (37, 96), (130, 160), (257, 1024)]


@pytest.fixture(autouse=True)
def _no_watchdog():
    yield
    assert mx.watchdog_status(clear=True) == 0


# ------------------------------------------------------------------ direct cast
@pytest.mark.parametrize("fmt", [0, 1, 2, 4, 5])
def test_cast_exhaustive_bf16(oracle, fmt):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = host(mx.cast(to_dev(bits), FMT_NAMES[fmt]))
    ref = oracle.cast(bits, fmt)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatching bytes, first at {bad[:8]}"


@pytest.mark.parametrize("n", [2, 4, 10, 28, 1000, 4097 * 8 + 4, 4097 * 8 + 6])
def test_cast_tail(oracle, n):
    rng = np.random.default_rng(n)
    bits = rng.integers(0, 65536, size=n, dtype=np.uint32).astype(np.uint16)
    for fmt in (0, 2, 4, 5):
        if fmt in (4, 5) and n % 4:                     # FP6: whole bytes of packed codes only
            with pytest.raises(mx.MxError):
                mx.cast(to_dev(bits), FMT_NAMES[fmt])
            continue
        assert np.array_equal(host(mx.cast(to_dev(bits), FMT_NAMES[fmt])), oracle.cast(bits, fmt))


# ------------------------------------------------------------------ row-wise MX
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("fmt,rounding", [(0, "ceil"), (0, "floor"), (1, "ceil"), (1, "floor"), (2, "floor"), (2, "ceil"),
                                          (4, "floor"), (4, "ceil"), (5, "floor"), (5, "ceil"), (6, "floor"),
                                          (6, "ceil")])
def test_quantize_rowwise_matches_oracle(oracle, shape, fmt, rounding):
    x = with_specials(synth.mx8_rowwise(*shape, seed=shape[0]), seed=shape[1])
    q = mx.quantize(to_dev(x), FMT_NAMES[fmt], "row", rounding, layout="both")
    e_ref, s_ref = oracle.quantize_mx(x, fmt, oracle.ROW, oracle.CEIL if rounding == "ceil" else oracle.FLOOR)
    assert np.array_equal(host(q.elems), e_ref.reshape(-1))
    assert np.array_equal(host(q.scales), s_ref.reshape(-1))
    assert np.array_equal(host(q.scales_alt), oracle.to_tcgen05_layout(s_ref))


@pytest.mark.parametrize("layout", ["rowmajor", "tcgen05"])
def test_quantize_single_layout(oracle, layout):
    x = synth.weight_fp4(130, 96, seed=3)
    q = mx.quantize(to_dev(x), "e2m1", "row", "floor", layout=layout)
    _, s_ref = oracle.quantize_mx(x, oracle.E2M1, oracle.ROW, oracle.FLOOR)
    want = s_ref.reshape(-1) if layout == "rowmajor" else oracle.to_tcgen05_layout(s_ref)
    assert np.array_equal(host(q.scales), want)


def test_tcgen05_padding_is_zeroed(oracle):
    x = synth.normal(5, 64, seed=2)
    dev = to_dev(x)
    rows, cols = x.shape
    sc = torch.full((mx.scale_bytes(rows, cols // 32, "tcgen05"),), 0xAB, dtype=torch.uint8, device="cuda")
    el = torch.empty(rows * cols, dtype=torch.uint8, device="cuda")
    st = L.lib.mx_quantize(dev.data_ptr(), rows, cols, 0, 0, 1, el.data_ptr(), sc.data_ptr(), 2, None, None,
                           torch.cuda.current_stream().cuda_stream)
    assert st == 0
    _, s_ref = oracle.quantize_mx(x, 0, 0, 1)
    assert np.array_equal(host(sc), oracle.to_tcgen05_layout(s_ref))


# ------------------------------------------------------------------ column-wise and dual
@pytest.mark.parametrize("shape", [(32, 32), (64, 96), (96, 200), (160, 384)])
@pytest.mark.parametrize("fmt,rounding", [(0, "ceil"), (1, "ceil"), (2, "floor"), (4, "ceil"), (5, "floor"),
                                          (6, "ceil")])
def test_quantize_colwise_matches_oracle(oracle, shape, fmt, rounding):
    x = with_specials(synth.activations(*shape, seed=shape[1]), seed=shape[0])
    rnd = oracle.CEIL if rounding == "ceil" else oracle.FLOOR
    q = mx.quantize(to_dev(x), FMT_NAMES[fmt], "col", rounding, layout="both")
    e_ref, s_ref = oracle.quantize_mx(x, fmt, oracle.COL, rnd)
    assert np.array_equal(host(q.elems), e_ref.reshape(-1))
    assert np.array_equal(host(q.scales), s_ref.reshape(-1))
    assert np.array_equal(host(q.scales_alt), oracle.to_tcgen05_layout(s_ref))


@pytest.mark.parametrize("fmt,rounding", [(0, "ceil"), (1, "floor"), (2, "floor"), (4, "ceil"), (5, "floor"),
                                          (6, "ceil")])
def test_colwise_and_dual_many_tiles_per_cta(oracle, fmt, rounding):
    """The TMA-staged kernel on shapes with several ring tiles per CTA and a ragged last
    column tile inside a narrower last band: column-only (two warp groups on alternate
    tiles, 2048 x 2312: a last tile 8 columns wide) and both orientations (2048 x 2336: a
    last tile 32 columns wide), both scale layouts."""
    rnd = oracle.CEIL if rounding == "ceil" else oracle.FLOOR
    x = with_specials(synth.gradients(2048, 2312, seed=40 + fmt), seed=fmt)
    q = mx.quantize(to_dev(x), FMT_NAMES[fmt], "col", rounding, layout="both")
    e_ref, s_ref = oracle.quantize_mx(x, fmt, oracle.COL, rnd)
    assert np.array_equal(host(q.elems), e_ref.reshape(-1))
    assert np.array_equal(host(q.scales), s_ref.reshape(-1))
    assert np.array_equal(host(q.scales_alt), oracle.to_tcgen05_layout(s_ref))
    x = with_specials(synth.gradients(2048, 2336, seed=50 + fmt), seed=fmt)
    qr, qc = mx.quantize_dual(to_dev(x), FMT_NAMES[fmt], rounding, "both")
    er, sr = oracle.quantize_mx(x, fmt, oracle.ROW, rnd)
    ec, sc = oracle.quantize_mx(x, fmt, oracle.COL, rnd)
    assert np.array_equal(host(qr.elems), er.reshape(-1))
    assert np.array_equal(host(qr.scales), sr.reshape(-1))
    assert np.array_equal(host(qr.scales_alt), oracle.to_tcgen05_layout(sr))
    assert np.array_equal(host(qc.elems), ec.reshape(-1))
    assert np.array_equal(host(qc.scales), sc.reshape(-1))
    assert np.array_equal(host(qc.scales_alt), oracle.to_tcgen05_layout(sc))


@pytest.mark.parametrize("shape", [(32, 32), (64, 160), (160, 384), (256, 1024)])
@pytest.mark.parametrize("fmt,rounding", [(0, "ceil"), (1, "ceil"), (1, "floor"), (2, "floor"), (4, "floor"),
                                          (5, "ceil"), (6, "floor"), (6, "ceil")])
@pytest.mark.parametrize("layout", ["rowmajor", "tcgen05", "both"])
def test_quantize_dual_matches_oracle(oracle, shape, fmt, rounding, layout):
    x = with_specials(synth.gradients(*shape, seed=shape[0] + fmt), seed=shape[1])
    rnd = oracle.CEIL if rounding == "ceil" else oracle.FLOOR
    qr, qc = mx.quantize_dual(to_dev(x), FMT_NAMES[fmt], rounding, layout)
    er, sr = oracle.quantize_mx(x, fmt, oracle.ROW, rnd)
    ec, sc = oracle.quantize_mx(x, fmt, oracle.COL, rnd)
    tr = oracle.to_tcgen05_layout if layout == "tcgen05" else (lambda s: s.reshape(-1))
    assert np.array_equal(host(qr.elems), er.reshape(-1))
    assert np.array_equal(host(qr.scales), tr(sr))
    assert np.array_equal(host(qc.elems), ec.reshape(-1))
    assert np.array_equal(host(qc.scales), tr(sc))
    if layout == "both":                                  # the tcgen05 copies from the same pass
        assert np.array_equal(host(qr.scales_alt), oracle.to_tcgen05_layout(sr))
        assert np.array_equal(host(qc.scales_alt), oracle.to_tcgen05_layout(sc))


# ------------------------------------------------------------------ NVFP4
@pytest.mark.parametrize("shape", [(1, 16), (5, 48), (130, 256), (64, 4096)])
@pytest.mark.parametrize("specials", [False, True])
def test_nvfp4_matches_oracle(oracle, shape, specials):
    x = synth.weight_fp4(*shape, seed=shape[0])
    if specials:
        x = with_specials(x, seed=7)
    q = mx.quantize(to_dev(x), "nvfp4", "row", "ceil", layout="both")
    e_ref, s_ref, g_ref = oracle.quantize_nvfp4(x)
    assert host(q.global_scale)[0] == np.float32(g_ref)
    assert np.array_equal(host(q.elems), e_ref.reshape(-1))
    assert np.array_equal(host(q.scales), s_ref.reshape(-1))
    assert np.array_equal(host(q.scales_alt), oracle.to_tcgen05_layout(s_ref))
    d = bf16_bits(mx.dequantize(q, "tcgen05"))
    assert nan_aware_equal(d.reshape(-1), oracle.dequantize_nvfp4(e_ref, s_ref, g_ref, *shape).reshape(-1))


def test_nvfp4_degenerate_tensors(oracle):
    for x in (np.zeros((4, 32), dtype=np.uint16),                          # all zero: g = 1
              np.full((2, 16), 0x0001, dtype=np.uint16),                   # smallest subnormals
              np.full((2, 32), 0x7FC0, dtype=np.uint16)):                  # all NaN
        q = mx.quantize(to_dev(x), "nvfp4", "row", "ceil", layout="rowmajor")
        e_ref, s_ref, g_ref = oracle.quantize_nvfp4(x)
        assert host(q.global_scale)[0] == np.float32(g_ref)
        assert np.array_equal(host(q.elems), e_ref.reshape(-1))
        assert np.array_equal(host(q.scales), s_ref.reshape(-1))


# ------------------------------------------------------------------ dequantisation
@pytest.mark.parametrize("fmt", [0, 1, 2, 4, 5, 6])
@pytest.mark.parametrize("layout", ["rowmajor", "tcgen05"])
def test_dequantize_matches_oracle(oracle, fmt, layout):
    x = with_specials(synth.mx8_rowwise(67, 256, seed=fmt), seed=3)
    q = mx.quantize(to_dev(x), FMT_NAMES[fmt], "row", "ceil", layout="both")
    e_ref, s_ref = oracle.quantize_mx(x, fmt, oracle.ROW, oracle.CEIL)
    d = bf16_bits(mx.dequantize(q, layout))
    assert nan_aware_equal(d.reshape(-1), oracle.dequantize_mx(e_ref, s_ref, 67, 256, fmt).reshape(-1))


def test_dequantize_all_scale_codes(oracle):
    """Every E8M0 code (incl. 2^-127 and NaN) against every element code."""
    for fmt in (0, 1, 2, 4, 5, 6):
        ncode = {2: 16, 4: 64, 5: 64}.get(fmt, 256)         # FP6: the 64 six-bit codes
        codes = np.tile(np.arange(ncode, dtype=np.uint8), 256 * 32 // ncode)[: 256 * 32].reshape(256, 32)
        scales = np.arange(256, dtype=np.uint8).reshape(256, 1)
        if fmt == 2:
            elems = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
        elif fmt in (4, 5):
            elems = pack_codes(codes, 6)                  # 24 bytes per 32 codes
        else:
            elems = codes
        q = mx.Quantized(torch.from_numpy(np.ascontiguousarray(elems).reshape(-1)).cuda(),
                         torch.from_numpy(scales.reshape(-1).copy()).cuda(), None, None, 256, 32, fmt)
        d = bf16_bits(mx.dequantize(q, "rowmajor"))
        assert nan_aware_equal(d.reshape(-1), oracle.dequantize_mx(elems, scales, 256, 32, fmt).reshape(-1))


@pytest.mark.parametrize("fmt", [0, 1, 2, 4, 5, 6, "nvfp4"])
@pytest.mark.parametrize("layout", ["rowmajor", "tcgen05"])
def test_dequantize_many_tiles_per_cta(oracle, fmt, layout):
    """Shapes with more ring tiles than resident CTAs (each CTA walks several tiles and
    loads the next tile's block scales ahead), an odd block count (FP6 and NVFP4 read the
    last block from global memory) and a ragged last tile."""
    rows, cols = (12289, 496) if fmt == "nvfp4" else (12289, 480)
    x = with_specials(synth.mx8_rowwise(rows, cols, seed=11), seed=5)
    if fmt == "nvfp4":
        q = mx.quantize(to_dev(x), "nvfp4", "row", "ceil", layout="both")
        e_ref, s_ref, g_ref = oracle.quantize_nvfp4(x)
        assert np.array_equal(host(q.elems), e_ref.reshape(-1))
        ref = oracle.dequantize_nvfp4(e_ref, s_ref, g_ref, rows, cols)
    else:
        q = mx.quantize(to_dev(x), FMT_NAMES[fmt], "row", "ceil", layout="both")
        e_ref, s_ref = oracle.quantize_mx(x, fmt, oracle.ROW, oracle.CEIL)
        assert np.array_equal(host(q.elems), e_ref.reshape(-1))
        ref = oracle.dequantize_mx(e_ref, s_ref, rows, cols, fmt)
    d = bf16_bits(mx.dequantize(q, layout))
    assert nan_aware_equal(d.reshape(-1), ref.reshape(-1))


# ------------------------------------------------------------------ full-size workloads
def test_mx8_rowwise_1024x1024_full(oracle):
    x = synth.mx8_rowwise()
    q = mx.quantize(to_dev(x), "e4m3", "row", "ceil", layout="rowmajor")
    e_ref, s_ref = oracle.quantize_mx(x, oracle.E4M3, oracle.ROW, oracle.CEIL)
    assert np.array_equal(host(q.elems), e_ref.reshape(-1))
    assert np.array_equal(host(q.scales), s_ref.reshape(-1))
    d = bf16_bits(mx.dequantize(q, "rowmajor"))
    assert np.array_equal(d.reshape(-1), oracle.dequantize_mx(e_ref, s_ref, 1024, 1024, oracle.E4M3).reshape(-1))


def test_weight_4096x4096_full(oracle):
    x = synth.weight_fp4()
    dev = to_dev(x)
    q4 = mx.quantize(dev, "e2m1", "row", "floor", layout="both")
    e_ref, s_ref = oracle.quantize_mx(x, oracle.E2M1, oracle.ROW, oracle.FLOOR)
    assert np.array_equal(host(q4.elems), e_ref.reshape(-1))
    assert np.array_equal(host(q4.scales), s_ref.reshape(-1))
    assert np.array_equal(host(q4.scales_alt), oracle.to_tcgen05_layout(s_ref))
    qn = mx.quantize(dev, "nvfp4", "row", "ceil", layout="both")
    e_ref, s_ref, g_ref = oracle.quantize_nvfp4(x)
    assert host(qn.global_scale)[0] == np.float32(g_ref)
    assert np.array_equal(host(qn.elems), e_ref.reshape(-1))
    assert np.array_equal(host(qn.scales), s_ref.reshape(-1))
    assert np.array_equal(host(qn.scales_alt), oracle.to_tcgen05_layout(s_ref))


def test_empty_inputs_launch_nothing():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    q = mx.quantize(x, "e4m3", "row", "ceil")
    assert q.elems.numel() == 0
    assert mx.cast(torch.empty(0, dtype=torch.bfloat16, device="cuda"), "e2m1").numel() == 0


@pytest.mark.parametrize("shape", [(5, 48), (130, 256), (512, 4096), (1024, 8192)])
def test_nvfp4_multi_cta_matches_oracle(oracle, shape):
    """Shapes from one partial maximum to hundreds (the maximum pass's CTA count grows
    with the tile count up to 3 per SM): codes, scales and tensor scale match the oracle."""
    x = synth.weight_fp4(*shape, seed=shape[0])
    q = mx.quantize(to_dev(x), "nvfp4", "row", "ceil", layout="both")
    e, s, g = oracle.quantize_nvfp4(x)
    assert host(q.global_scale)[0] == np.float32(g)
    assert np.array_equal(host(q.elems), e.reshape(-1))
    assert np.array_equal(host(q.scales), s.reshape(-1))
    assert np.array_equal(host(q.scales_alt), oracle.to_tcgen05_layout(s))


@pytest.mark.parametrize("offset", [1, 2, 3])
def test_nvfp4_unaligned_scale_buffers(oracle, offset):
    """Scale buffers at byte offsets 1-3 (no 4-byte vector stores possible): same bytes as
    the oracle, and nothing written outside the buffers."""
    rows, cols = 96, 512
    x = synth.weight_fp4(rows, cols, seed=offset)
    e, s, g = oracle.quantize_nvfp4(x)
    src = to_dev(x)
    elems = torch.empty(rows * cols // 2, dtype=torch.uint8, device="cuda")
    n_rm, n_tc = rows * cols // 16, mx.scale_bytes(rows, cols // 16, "tcgen05")
    rm = torch.full((n_rm + 8,), 0xA5, dtype=torch.uint8, device="cuda")
    tc = torch.full((n_tc + 8,), 0xA5, dtype=torch.uint8, device="cuda")
    gs = torch.empty(1, dtype=torch.float32, device="cuda")
    st = L.lib.mx_quantize(src.data_ptr(), rows, cols, L.MX_FMT_NVFP4, L.MX_AXIS_ROW, L.MX_SCALE_CEIL_RECIPE,
                           elems.data_ptr(), rm.data_ptr() + offset, 3, tc.data_ptr() + offset, gs.data_ptr(),
                           torch.cuda.current_stream().cuda_stream)
    assert st == L.MX_OK
    assert np.array_equal(host(elems), e.reshape(-1))
    rm_h, tc_h = host(rm), host(tc)
    assert np.array_equal(rm_h[offset:offset + n_rm], s.reshape(-1))
    assert np.array_equal(tc_h[offset:offset + n_tc], oracle.to_tcgen05_layout(s))
    assert np.all(rm_h[:offset] == 0xA5) and np.all(rm_h[offset + n_rm:] == 0xA5)
    assert np.all(tc_h[:offset] == 0xA5) and np.all(tc_h[offset + n_tc:] == 0xA5)


@pytest.mark.parametrize("sigma_log2", [-60, -72, -78, -84, -95, -110])
def test_nvfp4_tiny_tensor_scales(oracle, sigma_log2):
    """Tensors whose per-tensor scale puts 6g on either side of 2^-80 (where the block
    scale's quotient switches between the multiply-and-correct form and the IEEE divide)."""
    x = synth.normal(64, 512, sigma=2.0 ** sigma_log2, seed=-sigma_log2)
    q = mx.quantize(to_dev(x), "nvfp4", "row", "ceil", layout="rowmajor")
    e_ref, s_ref, g_ref = oracle.quantize_nvfp4(x)
    assert host(q.global_scale)[0] == np.float32(g_ref)
    assert np.array_equal(host(q.elems), e_ref.reshape(-1))
    assert np.array_equal(host(q.scales), s_ref.reshape(-1))


def test_output_buffers_are_reused(oracle):
    """`out=` writes into the caller's buffers (same pointers, same results)."""
    x = to_dev(synth.activations(64, 256, seed=5))
    q = mx.quantize(x, "e4m3", "row", "ceil", layout="both")
    q.elems.zero_(); q.scales.zero_(); q.scales_alt.zero_()
    q2 = mx.quantize(x, "e4m3", "row", "ceil", layout="both", out=q)
    assert q2.elems.data_ptr() == q.elems.data_ptr() and q2.scales_alt.data_ptr() == q.scales_alt.data_ptr()
    ref = mx.quantize(x, "e4m3", "row", "ceil", layout="both")
    assert torch.equal(q2.elems, ref.elems) and torch.equal(q2.scales, ref.scales)
    assert torch.equal(q2.scales_alt, ref.scales_alt)
    d = mx.quantize_dual(x, "e5m2", "floor", "rowmajor")
    d2 = mx.quantize_dual(x, "e5m2", "floor", "rowmajor", out=d)
    assert d2[1].elems.data_ptr() == d[1].elems.data_ptr()
    y = torch.empty_like(x)
    assert mx.dequantize(q, "tcgen05", out=y).data_ptr() == y.data_ptr()
    assert torch.equal(y, mx.dequantize(q, "rowmajor"))
    with pytest.raises(ValueError):
        mx.quantize(x, "e4m3", "row", "ceil", layout="both", out=mx.Quantized(q.elems[:10], q.scales, q.scales_alt,
                                                                             None, 64, 256, q.fmt))


# ------------------------------------------------------------------ NVFP4 16 x 16 weight blocks
@pytest.mark.parametrize("shape", [(16, 16), (48, 96), (160, 256), (1024, 4096)])
def test_nvfp4_2d_matches_oracle(oracle, shape):
    x = with_specials(synth.weight_fp4(*shape, seed=shape[0] + 1), seed=shape[1] + 1)
    q = mx.quantize_nvfp4_2d(to_dev(x), layout="both")
    e, s, g = oracle.quantize_nvfp4_2d(x)
    assert host(q.global_scale)[0] == np.float32(g)
    assert np.array_equal(host(q.elems), e.reshape(-1))
    assert np.array_equal(host(q.scales), s.reshape(-1))
    assert np.array_equal(host(q.scales_alt), oracle.to_tcgen05_layout(s))


def test_nvfp4_2d_weight_transposes(oracle):
    """The weight and its transpose quantise to transposed codes and block scales on the GPU."""
    x = synth.weight_fp4(256, 512, seed=9)
    q = mx.quantize_nvfp4_2d(to_dev(x), layout="rowmajor")
    qt = mx.quantize_nvfp4_2d(to_dev(np.ascontiguousarray(x.T)), layout="rowmajor")
    e = host(q.elems).reshape(256, 256)
    et = host(qt.elems).reshape(512, 128)
    codes = np.stack([np.stack([r & 0xF, r >> 4], axis=1).reshape(-1) for r in e])
    codes_t = np.stack([np.stack([r & 0xF, r >> 4], axis=1).reshape(-1) for r in et])
    assert np.array_equal(codes_t, codes.T)
    assert np.array_equal(host(q.scales).reshape(256, 32)[::16], host(qt.scales).reshape(512, 16)[::16].T)


# ------------------------------------------------------------------ MX and NVFP4 of one tensor
@pytest.mark.parametrize("shape", [(1, 32), (37, 96), (130, 256), (512, 4096), (4096, 4096)])
@pytest.mark.parametrize("fmt,rounding", [(2, "floor"), (0, "ceil"), (6, "ceil")])
@pytest.mark.parametrize("specials", [False, True])
def test_mx_nvfp4_pair_matches_oracle(oracle, shape, fmt, rounding, specials):
    """One call quantising the same weight to an MX format and to NVFP4 (the MX pass supplies
    the NVFP4 tensor maximum, Inf / NaN excluded) equals the oracle for both."""
    x = synth.weight_fp4(*shape, seed=shape[0] + fmt)
    if specials:
        x = with_specials(x, seed=shape[1])
    qm, qn = mx.quantize_mx_nvfp4(to_dev(x), FMT_NAMES[fmt], rounding)
    e, s = oracle.quantize_mx(x, fmt, oracle.ROW, oracle.CEIL if rounding == "ceil" else oracle.FLOOR)
    assert np.array_equal(host(qm.elems), e.reshape(-1))
    assert np.array_equal(host(qm.scales), s.reshape(-1))
    assert np.array_equal(host(qm.scales_alt), oracle.to_tcgen05_layout(s))
    e, s, g = oracle.quantize_nvfp4(x)
    assert host(qn.global_scale)[0] == np.float32(g)
    assert np.array_equal(host(qn.elems), e.reshape(-1))
    assert np.array_equal(host(qn.scales), s.reshape(-1))
    assert np.array_equal(host(qn.scales_alt), oracle.to_tcgen05_layout(s))
