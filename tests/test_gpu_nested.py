"""GPU parity of the nested-block conversion (MXFP4 1 x 32 tiles -> FP8 E4M3 with 128 x 128
block scales) against the oracle, through the C ABI: codes, block scales and exactness
flags bit for bit."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import microscaling_precision_number_b200 as mx
    from microscaling_precision_number_b200 import _lib as L


@pytest.fixture(autouse=True)
def _no_watchdog():
    yield
    assert mx.watchdog_status(clear=True) == 0


def run(elems, scales, rows, cols, offsets=(0, 0, 0)):
    """offsets: byte offsets of the codes, the scales and the output inside larger buffers
    (16 / 1 / 16 break the 32-byte and 2-byte alignment of the wide loads and stores)."""
    eo, so, oo = offsets
    e = torch.zeros(eo + elems.size, dtype=torch.uint8, device="cuda")[eo:]
    e.copy_(torch.from_numpy(np.ascontiguousarray(elems).reshape(-1)))
    s = torch.zeros(so + scales.size, dtype=torch.uint8, device="cuda")[so:]
    s.copy_(torch.from_numpy(np.ascontiguousarray(scales).reshape(-1)))
    out = torch.empty(oo + rows * cols, dtype=torch.uint8, device="cuda")[oo:]
    bs = torch.empty((rows // 128) * (cols // 128), dtype=torch.float32, device="cuda")
    ok = torch.empty((rows // 128) * (cols // 128), dtype=torch.uint8, device="cuda")
    st = L.lib.mx_mxfp4_to_fp8_blocks(e.data_ptr(), s.data_ptr(), rows, cols, out.data_ptr(), bs.data_ptr(),
                                      ok.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == L.MX_OK
    return out.cpu().numpy().reshape(rows, cols), bs.cpu().numpy().reshape(rows // 128, cols // 128), \
        ok.cpu().numpy().reshape(rows // 128, cols // 128)


def check(oracle, elems, scales, rows, cols, offsets=(0, 0, 0)):
    got = run(elems, scales, rows, cols, offsets)
    ref = oracle.mxfp4_to_fp8_blocks(elems, scales, rows, cols)
    for g, r, what in zip(got, ref, ("codes", "block scales", "exact flags")):
        assert np.array_equal(g, r), what
    return ref


@pytest.mark.parametrize("shape", [(128, 128), (256, 512), (384, 1024)])
def test_quantised_weights(oracle, shape):
    x = synth.weight_fp4(*shape, seed=shape[1])
    e, s = oracle.quantize_mx(x, oracle.E2M1, oracle.ROW, oracle.FLOOR)
    _, _, ok = check(oracle, e, s, *shape)
    assert np.all(ok == 1)


@pytest.mark.parametrize("offsets", [(16, 0, 0), (0, 1, 0), (0, 0, 16), (16, 1, 16)])
def test_unaligned_buffers(oracle, offsets):
    """Buffers that are 16-byte (codes, output) or 1-byte (scales) aligned only: the kernel
    takes its narrow-access form; same results."""
    rng = np.random.default_rng(5)
    rows, cols = 256, 384
    x = synth.weight_fp4(rows, cols, seed=17)
    e, s = oracle.quantize_mx(x, oracle.E2M1, oracle.ROW, oracle.FLOOR)
    s = s.copy()
    s[128:, :2] = rng.integers(100, 140, size=(128, 2), dtype=np.uint8)
    check(oracle, e, s, rows, cols, offsets)


def test_arbitrary_codes_and_scales(oracle):
    """Random code bytes with random scales (every E8M0 code incl. NaN, wide gaps inside a
    block, all-zero tiles with large scales): every path of the kernel."""
    rng = np.random.default_rng(3)
    rows, cols = 512, 512
    e = rng.integers(0, 256, size=(rows, cols // 2), dtype=np.uint8)
    s = rng.integers(0, 256, size=(rows, cols // 32), dtype=np.uint8)
    e[0:16] = 0                                   # zero tiles in the first block
    s[256:384, 4:8] = rng.integers(120, 135, size=(128, 4), dtype=np.uint8)   # narrow spread in block (2, 1)
    _, _, ok = check(oracle, e, s, rows, cols)
    assert 0 in ok and 1 in ok


@pytest.mark.parametrize("gap,low", [(14, 0.5), (15, 0.5), (15, 1.0), (16, 1.0), (15, 1.5), (40, 1.0), (140, 1.0)])
def test_scale_gap_edges(oracle, gap, low):
    x = np.zeros((128, 256), dtype=np.float32)
    x[0, 0] = 6.0
    x[5, 32] = low * 2.0 ** -gap if gap < 130 else 0.0
    x[9, 200] = 3.0 * 2.0 ** -(gap % 64)
    bits = (torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    e, s = oracle.quantize_mx(bits, oracle.E2M1, oracle.ROW, oracle.FLOOR)
    if gap >= 130:                                 # a tile far below via its scale byte only
        s[5, 1] = 3
        e[5, 16] = 0x02
    check(oracle, e, s, 128, 256)


def test_single_tile_offsets_and_magnitudes(oracle):
    """One 128 x 128 block per (tile offset d, E2M1 magnitude): every other tile of the block
    sits at d >= -8 (always exact) and one tile holds a single code of the given magnitude
    at d in -8 .. -13, so the block flag is that code's exactness alone -- the boundary
    cases of the kernel's closed-form rule against the oracle's round trip."""
    offsets, mags = list(range(-8, -14, -1)), list(range(1, 8))
    cases = [(d, m, sign) for d in offsets for m in mags for sign in (0, 8)]
    rows, cols = 128, 128 * len(cases)
    e = np.zeros((rows, cols // 2), dtype=np.uint8)
    s = np.full((rows, cols // 32), 127, dtype=np.uint8)          # tile exponent 0
    for j, (d, m, sign) in enumerate(cases):
        e[0, 64 * j] = 0x07                                       # 6.0 * 2^0: s_max = 0
        s[7, 4 * j + 2] = 127 + d - 6                             # tile exponent d - 6: offset d
        e[7, 64 * j + 32] = (m | sign) << 4                       # its second code (odd index)
    _, _, ok = check(oracle, e, s, rows, cols)
    flags = {c: int(f) for c, f in zip(cases, ok.reshape(-1))}
    assert flags[(-8, 1, 0)] == 1 and flags[(-9, 1, 0)] == 0 and flags[(-9, 2, 8)] == 1
    assert flags[(-11, 6, 0)] == 1 and flags[(-11, 7, 0)] == 0 and flags[(-12, 6, 0)] == 0


def test_weight_14336x4096(oracle):
    """The mixed-GEMM weight shape (14336 x 4096, N(0, 0.02)) end to end."""
    x = synth.normal(14336, 4096, sigma=0.02, seed=51)
    e, s = oracle.quantize_mx(x, oracle.E2M1, oracle.ROW, oracle.FLOOR)
    _, _, ok = check(oracle, e, s, 14336, 4096)
    assert np.all(ok == 1)
