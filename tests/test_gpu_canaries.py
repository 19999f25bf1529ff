"""Out-of-bounds write checks for every entry point of the C ABI (in place of a memory
sanitizer): each output buffer sits between two 256-byte guard regions filled with a
canary byte; after the call on odd shapes (partial tcgen05 atoms, ragged last tiles,
single blocks) every guard byte must be unchanged and the output must equal the same
call into ordinary buffers."""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import microscaling_precision_number_b200 as mx
    from microscaling_precision_number_b200 import _lib as L

G = 256
CANARY = 0xA5


class Guarded:
    """n bytes of device memory with G canary bytes on each side (16-byte aligned)."""

    def __init__(self, n):
        self.n = n
        self.full = torch.full((n + 2 * G,), CANARY, dtype=torch.uint8, device="cuda")
        self.view = self.full[G:G + n]

    def ptr(self):
        return self.view.data_ptr()

    def intact(self):
        f = self.full.cpu().numpy()
        return bool(np.all(f[:G] == CANARY) and np.all(f[G + self.n:] == CANARY))


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def stream():
    return torch.cuda.current_stream().cuda_stream


@pytest.fixture(autouse=True)
def _no_watchdog():
    yield
    assert mx.watchdog_status(clear=True) == 0


SHAPES = [(1, 32), (37, 96), (130, 160), (257, 288)]
FMTS = [(0, "e4m3"), (1, "e5m2"), (2, "e2m1"), (4, "e2m3"), (5, "e3m2"), (6, "int8")]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("fmt,name", FMTS)
def test_quantize_rowwise_guards(shape, fmt, name):
    R, C = shape
    x = to_dev(synth.mx8_rowwise(R, C, seed=R + fmt))
    e = Guarded(mx.elem_bytes(R, C, fmt))
    rm = Guarded(R * C // 32)
    tc = Guarded(mx.scale_bytes(R, C // 32, "tcgen05"))
    assert L.lib.mx_quantize(x.data_ptr(), R, C, fmt, L.MX_AXIS_ROW, L.MX_SCALE_CEIL_RECIPE, e.ptr(), rm.ptr(), 3,
                             tc.ptr(), None, stream()) == L.MX_OK
    ref = mx.quantize(x, name, "row", "ceil", layout="both")
    assert e.intact() and rm.intact() and tc.intact()
    assert torch.equal(e.view, ref.elems) and torch.equal(rm.view, ref.scales) and torch.equal(tc.view, ref.scales_alt)


@pytest.mark.parametrize("shape", [(32, 40), (96, 200), (160, 384)])
@pytest.mark.parametrize("fmt,name", [(0, "e4m3"), (2, "e2m1"), (4, "e2m3")])
def test_quantize_colwise_and_dual_guards(shape, fmt, name):
    R, C = shape
    x = to_dev(synth.activations(R, C, seed=C + fmt))
    ce = Guarded(mx.elem_bytes(C, R, fmt))
    crm, ctc = Guarded(C * R // 32), Guarded(mx.scale_bytes(C, R // 32, "tcgen05"))
    assert L.lib.mx_quantize(x.data_ptr(), R, C, fmt, L.MX_AXIS_COL, L.MX_SCALE_CEIL_RECIPE, ce.ptr(), crm.ptr(), 3,
                             ctc.ptr(), None, stream()) == L.MX_OK
    ref = mx.quantize(x, name, "col", "ceil", layout="both")
    assert ce.intact() and crm.intact() and ctc.intact()
    assert torch.equal(ce.view, ref.elems) and torch.equal(crm.view, ref.scales) and torch.equal(ctc.view, ref.scales_alt)
    if C % 32:
        return
    re_ = Guarded(mx.elem_bytes(R, C, fmt))
    rrm, rtc = Guarded(R * C // 32), Guarded(mx.scale_bytes(R, C // 32, "tcgen05"))
    for g in (ce, crm, ctc):
        g.full.fill_(CANARY)
    assert L.lib.mx_quantize_dual(x.data_ptr(), R, C, fmt, L.MX_SCALE_CEIL_RECIPE, re_.ptr(), rrm.ptr(), ce.ptr(),
                                  crm.ptr(), 3, rtc.ptr(), ctc.ptr(), stream()) == L.MX_OK
    qr, qc = mx.quantize_dual(x, name, "ceil", "both")
    assert all(g.intact() for g in (re_, rrm, rtc, ce, crm, ctc))
    assert torch.equal(re_.view, qr.elems) and torch.equal(rrm.view, qr.scales) and torch.equal(rtc.view, qr.scales_alt)
    assert torch.equal(ce.view, qc.elems) and torch.equal(crm.view, qc.scales) and torch.equal(ctc.view, qc.scales_alt)


@pytest.mark.parametrize("shape", [(1, 16), (37, 48), (130, 160), (257, 272)])
def test_nvfp4_and_noalloc_guards(shape):
    R, C = shape
    x = to_dev(synth.weight_fp4(R, C, seed=R))
    ref = mx.quantize(x, "nvfp4", "row", "ceil", layout="both")
    for fn in ("mx_quantize", "mx_quantize_nvfp4_noalloc"):
        e, rm, tc, g = Guarded(R * C // 2), Guarded(R * C // 16), Guarded(mx.scale_bytes(R, C // 16, "tcgen05")), \
            Guarded(4)
        if fn == "mx_quantize":
            st = L.lib.mx_quantize(x.data_ptr(), R, C, L.MX_FMT_NVFP4, L.MX_AXIS_ROW, L.MX_SCALE_CEIL_RECIPE,
                                   e.ptr(), rm.ptr(), 3, tc.ptr(), g.ptr(), stream())
        else:
            st = L.lib.mx_quantize_nvfp4_noalloc(x.data_ptr(), R, C, e.ptr(), rm.ptr(), 3, tc.ptr(), g.ptr(),
                                                 stream())
        assert st == L.MX_OK
        assert all(b.intact() for b in (e, rm, tc, g)), fn
        assert torch.equal(e.view, ref.elems) and torch.equal(rm.view, ref.scales)
        assert torch.equal(tc.view, ref.scales_alt) and torch.equal(g.view, ref.global_scale.view(torch.uint8))


@pytest.mark.parametrize("shape", [(16, 16), (48, 96), (160, 272)])
def test_nvfp4_2d_and_train_guards(shape):
    R, C = shape
    x = to_dev(synth.weight_fp4(R, C, seed=C))
    e, rm, tc, g = Guarded(R * C // 2), Guarded(R * C // 16), Guarded(mx.scale_bytes(R, C // 16, "tcgen05")), \
        Guarded(4)
    assert L.lib.mx_quantize_nvfp4_2d(x.data_ptr(), R, C, e.ptr(), rm.ptr(), 3, tc.ptr(), g.ptr(), stream()) == L.MX_OK
    ref = mx.quantize_nvfp4_2d(x, layout="both")
    assert all(b.intact() for b in (e, rm, tc, g))
    assert torch.equal(e.view, ref.elems) and torch.equal(rm.view, ref.scales) and torch.equal(tc.view, ref.scales_alt)
    rnd = torch.from_numpy(np.random.default_rng(R).integers(0, 256, R * C, dtype=np.uint8)).cuda()
    for fmt, B in ((L.MX_FMT_NVFP4, 16), (L.MX_FMT_E2M1, 32), (L.MX_FMT_E4M3, 32)):
        if C % B:
            continue
        eb = mx.elem_bytes(R, C, fmt)
        e, rm, tc = Guarded(eb), Guarded(R * C // B), Guarded(mx.scale_bytes(R, C // B, "tcgen05"))
        g = Guarded(4) if fmt == L.MX_FMT_NVFP4 else None
        assert L.lib.mx_quantize_train(x.data_ptr(), R, C, fmt, L.MX_SCALE_CEIL_RECIPE, 1, 0x5A3C, rnd.data_ptr(),
                                       e.ptr(), rm.ptr(), 3, tc.ptr(), g.ptr() if g else None, stream()) == L.MX_OK
        ref = mx.quantize_train(x, fmt, "ceil", rht_signs=0x5A3C, sr_random=rnd, layout="both")
        assert all(b.intact() for b in (e, rm, tc) + ((g,) if g else ()))
        assert torch.equal(e.view, ref.elems) and torch.equal(tc.view, ref.scales_alt)


@pytest.mark.parametrize("shape", [(1, 32), (37, 96), (130, 160)])
@pytest.mark.parametrize("fmt,name", FMTS + [(3, "nvfp4")])
@pytest.mark.parametrize("layout", ["rowmajor", "tcgen05"])
def test_dequantize_guards(shape, fmt, name, layout):
    R, C = shape
    x = to_dev(synth.mx8_rowwise(R, C, seed=fmt))
    q = mx.quantize(x, name, "row", "ceil", layout="both")
    out = Guarded(R * C * 2)
    sc = q.scales if layout == "rowmajor" else q.scales_alt
    assert L.lib.mx_dequantize(q.elems.data_ptr(), sc.data_ptr(),
                               q.global_scale.data_ptr() if q.global_scale is not None else None, R, C, fmt,
                               1 if layout == "rowmajor" else 2, out.ptr(), stream()) == L.MX_OK
    ref = mx.dequantize(q, layout)
    assert out.intact()
    assert torch.equal(out.view.view(torch.int16), ref.view(torch.int16).reshape(-1))


@pytest.mark.parametrize("n", [4, 28, 1000, 8 * 4097 + 4])
@pytest.mark.parametrize("fmt,name", [(0, "e4m3"), (2, "e2m1"), (4, "e2m3")])
def test_cast_guards(n, fmt, name):
    x = to_dev(synth.normal(1, n, seed=n))
    out = Guarded(mx.elem_bytes(1, n, fmt))
    assert L.lib.mx_cast(x.data_ptr(), n, fmt, out.ptr(), stream()) == L.MX_OK
    assert out.intact()
    assert torch.equal(out.view, mx.cast(x.reshape(-1), name))


@pytest.mark.parametrize("M,N,K,bfmt", [(128, 128, 128, "e4m3"), (128, 384, 256, "e2m1"), (256, 512, 256, "e4m3"),
                                        (384, 256, 512, "nvfp4"), (256, 256, 256, "e2m1x")])
def test_gemm_guards(M, N, K, bfmt):
    afmt = {"e2m1x": "e2m1", "nvfp4": "nvfp4"}.get(bfmt, "e4m3")
    bname = "e2m1" if bfmt == "e2m1x" else bfmt
    a = mx.quantize(to_dev(synth.normal(M, K, seed=M)), afmt, "row", "floor", layout="tcgen05")
    b = mx.quantize(to_dev(synth.normal(N, K, seed=N)), bname, "row", "floor", layout="tcgen05")
    out = Guarded(M * N * 2)
    A = L.MxOperand(a.elems.data_ptr(), a.scales.data_ptr(), a.fmt,
                    a.global_scale.data_ptr() if a.global_scale is not None else None)
    B = L.MxOperand(b.elems.data_ptr(), b.scales.data_ptr(), b.fmt,
                    b.global_scale.data_ptr() if b.global_scale is not None else None)
    assert L.lib.mx_gemm(A, B, out.ptr(), M, N, K, stream()) == L.MX_OK
    ref = mx.gemm(a, b)
    assert out.intact()
    assert torch.equal(out.view.view(torch.int16), ref.view(torch.int16).reshape(-1))


def test_nested_guards():
    R, C = 256, 384
    q = mx.quantize(to_dev(synth.weight_fp4(R, C, seed=3)), "e2m1", "row", "floor", layout="rowmajor")
    o8, bs, ok = Guarded(R * C), Guarded(4 * (R // 128) * (C // 128)), Guarded((R // 128) * (C // 128))
    assert L.lib.mx_mxfp4_to_fp8_blocks(q.elems.data_ptr(), q.scales.data_ptr(), R, C, o8.ptr(), bs.ptr(), ok.ptr(),
                                        stream()) == L.MX_OK
    assert o8.intact() and bs.intact() and ok.intact()
    o2 = torch.empty(R * C, dtype=torch.uint8, device="cuda")
    bs2 = torch.empty((R // 128) * (C // 128), dtype=torch.float32, device="cuda")
    ok2 = torch.empty((R // 128) * (C // 128), dtype=torch.uint8, device="cuda")
    assert L.lib.mx_mxfp4_to_fp8_blocks(q.elems.data_ptr(), q.scales.data_ptr(), R, C, o2.data_ptr(), bs2.data_ptr(),
                                        ok2.data_ptr(), stream()) == L.MX_OK
    assert torch.equal(o8.view, o2) and torch.equal(bs.view, bs2.view(torch.uint8)) and torch.equal(ok.view, ok2)
