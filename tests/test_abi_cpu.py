"""The C-ABI library loads, exports every function include/mx.h declares, and rejects
invalid arguments on the host before any CUDA call (runs without a GPU)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT


@pytest.fixture(scope="module")
def L():
    from microscaling_precision_number_b200 import build
    build.build()
    from microscaling_precision_number_b200 import _lib
    return _lib


def declared_functions():
    text = open(os.path.join(ROOT, "include", "mx.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mx_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("mx_quantize", "mx_quantize_dual", "mx_dequantize", "mx_gemm", "mx_cast",
                     "mx_status_string", "mx_last_cuda_error"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    raw = ctypes.CDLL(L.LIB_PATH)
    for name in declared_functions():
        assert hasattr(raw, name), f"libmx.so does not export {name}"
    assert set(L.EXPORTS) == set(declared_functions())


def test_status_strings(L):
    for s in range(7):
        assert L.lib.mx_status_string(s).startswith(b"MX_")
    assert b"unknown" in L.lib.mx_status_string(99)


def test_scale_bytes(L):
    assert L.lib.mx_scale_bytes(4096, 128, L.MX_LAYOUT_ROWMAJOR) == 4096 * 128
    assert L.lib.mx_scale_bytes(4096, 128, L.MX_LAYOUT_TCGEN05) == 32 * 32 * 512
    assert L.lib.mx_scale_bytes(130, 5, L.MX_LAYOUT_TCGEN05) == 2 * 2 * 512
    assert L.lib.mx_scale_bytes(-1, 5, L.MX_LAYOUT_TCGEN05) == -1
    assert L.lib.mx_scale_bytes(1, 1, 3) == -1


FAKE = 0x10000   # a 16-byte-aligned non-null address; never dereferenced (rejected first)


@pytest.mark.parametrize("args,status", [
    # bad enum values
    (dict(fmt=7), "MX_ERR_ARG"), (dict(axis=2), "MX_ERR_ARG"), (dict(rounding=5), "MX_ERR_ARG"),
    # NVFP4 column-wise unsupported; NVFP4 needs global_scale, MX must not get one
    (dict(fmt=3, axis=1, g=FAKE), "MX_ERR_ARG"), (dict(fmt=3), "MX_ERR_ARG"), (dict(g=FAKE), "MX_ERR_ARG"),
    # layouts
    (dict(layout=0), "MX_ERR_LAYOUT"), (dict(layout=4), "MX_ERR_LAYOUT"), (dict(layout=3), "MX_ERR_LAYOUT"),
    (dict(layout=1, alt=FAKE), "MX_ERR_LAYOUT"),
    # shapes
    (dict(rows=-1), "MX_ERR_SHAPE"), (dict(cols=48), "MX_ERR_SHAPE"), (dict(axis=1, rows=40), "MX_ERR_SHAPE"),
    (dict(fmt=3, cols=24, g=FAKE), "MX_ERR_SHAPE"),
    # null / misaligned pointers
    (dict(src=0), "MX_ERR_ARG"), (dict(out=0), "MX_ERR_ARG"), (dict(sc=0), "MX_ERR_ARG"),
    (dict(src=FAKE + 8), "MX_ERR_ALIGN"), (dict(out=FAKE + 4), "MX_ERR_ALIGN"),
    # empty input is valid and launches nothing
    (dict(rows=0), "MX_OK"), (dict(cols=0), "MX_OK"),
])
def test_quantize_validation(L, args, status):
    a = dict(src=FAKE, rows=64, cols=64, fmt=0, axis=0, rounding=1, out=FAKE, sc=FAKE, layout=1, alt=0, g=0)
    a.update(args)
    st = L.lib.mx_quantize(a["src"] or None, a["rows"], a["cols"], a["fmt"], a["axis"], a["rounding"],
                           a["out"] or None, a["sc"] or None, a["layout"], a["alt"] or None, a["g"] or None, None)
    assert st == getattr(L, status), L.lib.mx_status_string(st)


def test_dual_dequant_cast_gemm_validation(L):
    lib = L.lib
    assert lib.mx_quantize_dual(FAKE, 64, 64, 3, 1, FAKE, FAKE, FAKE, FAKE, 1, None, None, None) == L.MX_ERR_ARG
    # both layouts need both alternate buffers; a single layout takes none
    assert lib.mx_quantize_dual(FAKE, 64, 64, 0, 1, FAKE, FAKE, FAKE, FAKE, 3, None, None, None) == L.MX_ERR_LAYOUT
    assert lib.mx_quantize_dual(FAKE, 64, 64, 0, 1, FAKE, FAKE, FAKE, FAKE, 3, FAKE, None, None) == L.MX_ERR_LAYOUT
    assert lib.mx_quantize_dual(FAKE, 64, 64, 0, 1, FAKE, FAKE, FAKE, FAKE, 1, FAKE, FAKE, None) == L.MX_ERR_LAYOUT
    assert lib.mx_quantize_dual(FAKE, 64, 64, 0, 1, FAKE, FAKE, FAKE, FAKE, 4, None, None, None) == L.MX_ERR_LAYOUT
    assert lib.mx_quantize_dual(FAKE, 48, 64, 0, 1, FAKE, FAKE, FAKE, FAKE, 1, None, None, None) == L.MX_ERR_SHAPE
    assert lib.mx_quantize_dual(FAKE, 64, 64, 0, 1, FAKE, FAKE, None, FAKE, 1, None, None, None) == L.MX_ERR_ARG
    assert lib.mx_quantize_dual(FAKE, 0, 64, 0, 1, None, None, None, None, 1, None, None, None) == L.MX_OK
    assert lib.mx_quantize_dual(FAKE, 0, 64, 0, 1, None, None, None, None, 3, FAKE, FAKE, None) == L.MX_OK
    assert lib.mx_dequantize(FAKE, FAKE, None, 4, 48, 0, 1, FAKE, None) == L.MX_ERR_SHAPE
    assert lib.mx_dequantize(FAKE, FAKE, None, 4, 64, 3, 1, FAKE, None) == L.MX_ERR_ARG
    assert lib.mx_dequantize(FAKE, FAKE, None, 4, 64, 0, 3, FAKE, None) == L.MX_ERR_LAYOUT
    assert lib.mx_dequantize(FAKE + 2, FAKE, None, 4, 64, 0, 1, FAKE, None) == L.MX_ERR_ALIGN
    assert lib.mx_cast(FAKE, 7, 2, FAKE, None) == L.MX_ERR_SHAPE
    assert lib.mx_cast(FAKE, 8, 3, FAKE, None) == L.MX_ERR_ARG
    assert lib.mx_cast(FAKE, 8, 6, FAKE, None) == L.MX_ERR_ARG        # INT8 needs a scale
    assert lib.mx_cast(FAKE, 6, 4, FAKE, None) == L.MX_ERR_SHAPE      # FP6: whole bytes of packed codes
    assert lib.mx_cast(FAKE, 10, 5, FAKE, None) == L.MX_ERR_SHAPE
    assert lib.mx_quantize(FAKE, 4, 64, 7, 0, 1, FAKE, FAKE, 1, None, None, None) == L.MX_ERR_ARG
    assert lib.mx_quantize(FAKE, 4, 64, 6, 0, 1, FAKE, FAKE, 1, None, FAKE, None) == L.MX_ERR_ARG   # g is NVFP4 only
    assert lib.mx_cast(None, 8, 0, FAKE, None) == L.MX_ERR_ARG
    assert lib.mx_cast(FAKE, 0, 0, FAKE, None) == L.MX_OK
    op = lambda fmt, p=FAKE, g=None: L.MxOperand(p, FAKE, fmt, g)
    assert lib.mx_gemm(op(0), op(6), FAKE, 128, 128, 128, None) == L.MX_ERR_ARG      # INT8: no tensor-core form
    assert lib.mx_gemm(op(6), op(0), FAKE, 128, 128, 128, None) == L.MX_ERR_ARG
    assert lib.mx_gemm(op(4), op(7), FAKE, 128, 128, 128, None) == L.MX_ERR_ARG      # unknown format
    assert lib.mx_gemm(op(2), op(0), FAKE, 128, 128, 128, None) == L.MX_ERR_ARG      # E2M1 x E4M3 unsupported
    assert lib.mx_gemm(op(3, g=FAKE), op(2), FAKE, 128, 128, 256, None) == L.MX_ERR_ARG   # NVFP4 x MXFP4
    assert lib.mx_gemm(op(3), op(3, g=FAKE), FAKE, 128, 128, 256, None) == L.MX_ERR_ARG   # missing g
    assert lib.mx_gemm(op(2, g=FAKE), op(2), FAKE, 128, 128, 256, None) == L.MX_ERR_ARG   # g on MX
    assert lib.mx_gemm(op(2), op(2), FAKE, 128, 128, 128, None) == L.MX_ERR_SHAPE    # FP4 x FP4: K % 256
    assert lib.mx_gemm(op(3, g=FAKE), op(3, g=FAKE), FAKE, 128, 128, 384, None) == L.MX_ERR_SHAPE
    assert lib.mx_gemm(op(3, g=FAKE + 2), op(3, g=FAKE), FAKE, 128, 128, 256, None) == L.MX_ERR_ALIGN
    assert lib.mx_gemm(op(2), op(2), FAKE, 0, 128, 256, None) == L.MX_OK
    assert lib.mx_gemm(op(0), op(2), FAKE, 100, 128, 128, None) == L.MX_ERR_SHAPE
    assert lib.mx_gemm(op(0), op(0), FAKE, 128, 128, 96, None) == L.MX_ERR_SHAPE
    assert lib.mx_gemm(op(0, FAKE + 16), op(0), FAKE, 128, 128, 128, None) == L.MX_ERR_ALIGN
    assert lib.mx_gemm(op(0), op(0), None, 128, 128, 128, None) == L.MX_ERR_ARG
    assert lib.mx_gemm(op(0), op(0), FAKE, 0, 128, 128, None) == L.MX_OK


def test_product_package_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "microscaling_precision_number_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in text and "from oracle" not in text and "mx_oracle" not in text, f


# ------------------------------------------------------------------ newer entry points
@pytest.mark.parametrize("args,status", [
    (dict(fmt=4), "MX_ERR_ARG"), (dict(fmt=6), "MX_ERR_ARG"),              # FP6 / INT8: not training formats
    (dict(rounding=2), "MX_ERR_ARG"), (dict(rht=2), "MX_ERR_ARG"),
    (dict(fmt=3), "MX_ERR_ARG"), (dict(g=FAKE), "MX_ERR_ARG"),             # g exactly for NVFP4
    (dict(layout=0), "MX_ERR_LAYOUT"), (dict(layout=3), "MX_ERR_LAYOUT"),
    (dict(rows=-1), "MX_ERR_SHAPE"), (dict(cols=48), "MX_ERR_SHAPE"), (dict(fmt=3, cols=40, g=FAKE), "MX_ERR_SHAPE"),
    (dict(src=0), "MX_ERR_ARG"), (dict(out=0), "MX_ERR_ARG"), (dict(sc=0), "MX_ERR_ARG"),
    (dict(src=FAKE + 8), "MX_ERR_ALIGN"), (dict(rnd=FAKE + 8), "MX_ERR_ALIGN"),
    (dict(fmt=3, g=FAKE + 2), "MX_ERR_ALIGN"),
    (dict(rows=0), "MX_OK"),
])
def test_quantize_train_validation(L, args, status):
    a = dict(src=FAKE, rows=64, cols=64, fmt=2, rounding=0, rht=1, signs=0xB5C3, rnd=FAKE, out=FAKE, sc=FAKE,
             layout=2, alt=0, g=0)
    a.update(args)
    got = L.lib.mx_quantize_train(a["src"], a["rows"], a["cols"], a["fmt"], a["rounding"], a["rht"], a["signs"],
                                  a["rnd"] or None, a["out"] or None, a["sc"] or None, a["layout"], a["alt"] or None,
                                  a["g"] or None, None)
    assert got == getattr(L, status), (args, got)


@pytest.mark.parametrize("args,status", [
    (dict(layout=0), "MX_ERR_LAYOUT"), (dict(layout=1, alt=FAKE), "MX_ERR_LAYOUT"),
    (dict(rows=24), "MX_ERR_SHAPE"), (dict(cols=40), "MX_ERR_SHAPE"), (dict(rows=-16), "MX_ERR_SHAPE"),
    (dict(src=0), "MX_ERR_ARG"), (dict(g=0), "MX_ERR_ARG"),
    (dict(out=FAKE + 4), "MX_ERR_ALIGN"), (dict(g=FAKE + 1), "MX_ERR_ALIGN"),
    (dict(cols=0), "MX_OK"),
])
def test_quantize_nvfp4_2d_validation(L, args, status):
    a = dict(src=FAKE, rows=32, cols=64, out=FAKE, sc=FAKE, layout=2, alt=0, g=FAKE)
    a.update(args)
    got = L.lib.mx_quantize_nvfp4_2d(a["src"], a["rows"], a["cols"], a["out"] or None, a["sc"] or None, a["layout"],
                                     a["alt"] or None, a["g"] or None, None)
    assert got == getattr(L, status), (args, got)


@pytest.mark.parametrize("args,status", [
    (dict(rows=64), "MX_ERR_SHAPE"), (dict(cols=192), "MX_ERR_SHAPE"), (dict(rows=-128), "MX_ERR_SHAPE"),
    (dict(elems=0), "MX_ERR_ARG"), (dict(scales=0), "MX_ERR_ARG"), (dict(ok=0), "MX_ERR_ARG"),
    (dict(elems=FAKE + 8), "MX_ERR_ALIGN"), (dict(out=FAKE + 8), "MX_ERR_ALIGN"), (dict(bs=FAKE + 2), "MX_ERR_ALIGN"),
    (dict(rows=0), "MX_OK"),
])
def test_nested_blocks_validation(L, args, status):
    a = dict(elems=FAKE, scales=FAKE, rows=128, cols=256, out=FAKE, bs=FAKE, ok=FAKE)
    a.update(args)
    got = L.lib.mx_mxfp4_to_fp8_blocks(a["elems"] or None, a["scales"] or None, a["rows"], a["cols"],
                                       a["out"] or None, a["bs"] or None, a["ok"] or None, None)
    assert got == getattr(L, status), (args, got)


def test_missing_library_fails_loudly(tmp_path):
    """No fallback of any kind: with the shared library absent, the first call raises
    ImportError, and a CPU tensor is refused rather than quantised on the host."""
    import subprocess
    import sys
    code = (
        "import torch, microscaling_precision_number_b200 as mx\n"
        "try:\n"
        "    mx._lib.lib.load()\n"
        "except ImportError as e:\n"
        "    print('import-error', e)\n"
        "try:\n"
        "    mx.quantize(torch.zeros(4, 32, dtype=torch.bfloat16), 'e4m3')\n"
        "except ValueError:\n"
        "    print('refused-cpu-tensor')\n")
    env = dict(os.environ, MX_LIB_PATH=str(tmp_path / "absent" / "libmx.so"))
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert "import-error" in out.stdout and "refused-cpu-tensor" in out.stdout, out.stdout + out.stderr


@pytest.mark.parametrize("limit_us", [0, 100001, 2 ** 32 - 1])
def test_watchdog_selftest_rejects_limits(L, limit_us):
    """The watchdog self-test takes a limit of 1 .. 100000 microseconds; anything else is
    rejected before any CUDA call."""
    assert L.lib.mx_watchdog_selftest(limit_us, None) == L.MX_ERR_ARG


def test_mx_nvfp4_pair_validation(L):
    """mx_quantize_mx_nvfp4 rejects bad formats, layouts, shapes and pointers on the host."""
    f = FAKE
    q = L.lib.mx_quantize_mx_nvfp4
    # (fmt, rounding, mx_layout, mx_alt, nv_layout, nv_alt, cols, g, src) -> status
    cases = [
        ((3, 1, 1, None, 1, None, 64, f, f), L.MX_ERR_ARG),        # NVFP4 is not an MX format
        ((2, 7, 1, None, 1, None, 64, f, f), L.MX_ERR_ARG),        # bad rounding
        ((2, 0, 3, None, 1, None, 64, f, f), L.MX_ERR_LAYOUT),     # both layouts need the second buffer
        ((2, 0, 1, None, 3, None, 64, f, f), L.MX_ERR_LAYOUT),
        ((2, 0, 1, f, 1, None, 64, f, f), L.MX_ERR_LAYOUT),        # one layout takes none
        ((2, 0, 0, None, 1, None, 64, f, f), L.MX_ERR_LAYOUT),
        ((2, 0, 1, None, 1, None, 48, f, f), L.MX_ERR_SHAPE),      # cols % 32
        ((2, 0, 1, None, 1, None, 64, None, f), L.MX_ERR_ARG),     # NVFP4 needs the tensor-scale slot
        ((2, 0, 1, None, 1, None, 64, f, f + 8), L.MX_ERR_ALIGN),
    ]
    for (fmt, rnd, ml, ma, nl, na, cols, g, src), want in cases:
        st = q(src, 64, cols, fmt, rnd, f, f, ml, ma, f, f, nl, na, g, None)
        assert st == want, (fmt, rnd, ml, nl, cols, L.lib.mx_status_string(st))
    assert q(None, 0, 64, 2, 0, None, None, 1, None, None, None, 1, None, None, None) == L.MX_OK
