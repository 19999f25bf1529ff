"""Runs a set of calls through the bounds-checked build (MX_LIB_PATH must name
libmx_checked.so; started as a subprocess by test_gpu_checked.py) and checks them against
the oracle.  Prints one JSON line: per case whether the outputs matched, and the
watchdog code after the case (64 = a store outside the registered output extents was
refused)."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle  # noqa: E402
import synth  # noqa: E402
import microscaling_precision_number_b200 as mx  # noqa: E402
from microscaling_precision_number_b200 import _lib as L  # noqa: E402


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host(t):
    return t.cpu().numpy()


def code():
    return mx.watchdog_status(clear=True)


def case_rows(R, C, fmt, name, rnd):
    x = synth.mx8_rowwise(R, C, seed=R)
    q = mx.quantize(dev(x), name, "row", rnd, layout="both")
    e, s = oracle.quantize_mx(x, fmt, oracle.ROW, oracle.CEIL if rnd == "ceil" else oracle.FLOOR)
    ok = np.array_equal(host(q.elems), e.reshape(-1)) and np.array_equal(host(q.scales), s.reshape(-1)) and \
        np.array_equal(host(q.scales_alt), oracle.to_tcgen05_layout(s))
    d = mx.dequantize(q, "tcgen05")
    ok = ok and np.array_equal(d.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1),
                               oracle.dequantize_mx(e, s, R, C, fmt).reshape(-1))
    return ok


def case_dual(R, C, fmt, name):
    x = synth.gradients(R, C, seed=C)
    qr, qc = mx.quantize_dual(dev(x), name, "ceil", "both")
    er, sr = oracle.quantize_mx(x, fmt, oracle.ROW, oracle.CEIL)
    ec, sc = oracle.quantize_mx(x, fmt, oracle.COL, oracle.CEIL)
    return (np.array_equal(host(qr.elems), er.reshape(-1)) and np.array_equal(host(qc.elems), ec.reshape(-1)) and
            np.array_equal(host(qr.scales), sr.reshape(-1)) and np.array_equal(host(qc.scales_alt),
                                                                                oracle.to_tcgen05_layout(sc)))


def case_nvfp4(R, C):
    x = synth.weight_fp4(R, C, seed=C)
    qm, qn = mx.quantize_mx_nvfp4(dev(x), "e2m1", "floor")
    e, s, g = oracle.quantize_nvfp4(x)
    ok = np.array_equal(host(qn.elems), e.reshape(-1)) and np.array_equal(host(qn.scales), s.reshape(-1))
    q2 = mx.quantize(dev(x), "nvfp4", "row", "ceil", layout="tcgen05")
    ok = ok and np.array_equal(host(q2.elems), e.reshape(-1)) and host(q2.global_scale)[0] == np.float32(g)
    q3 = mx.quantize_nvfp4_2d(dev(x), layout="both")
    e3, s3, g3 = oracle.quantize_nvfp4_2d(x)
    ok = ok and np.array_equal(host(q3.elems), e3.reshape(-1))
    rnd = np.random.default_rng(1).integers(0, 256, x.shape, dtype=np.uint8)
    q4 = mx.quantize_train(dev(x), "nvfp4", "ceil", sr_random=torch.from_numpy(rnd).cuda(), layout="both")
    e4, s4, g4 = oracle.quantize_nvfp4_sr(x, rnd)
    return ok and np.array_equal(host(q4.elems), e4.reshape(-1))


def case_gemm(M, N, K, bname, bfmt):
    a = synth.normal(M, K, seed=M)
    b = synth.normal(N, K, seed=N)
    qa = mx.quantize(dev(a), "e4m3", "row", "ceil", layout="tcgen05")
    qb = mx.quantize(dev(b), bname, "row", "floor" if bname == "e2m1" else "ceil", layout="tcgen05")
    c = mx.gemm(qa, qb).float().cpu().numpy().astype(np.float64)
    ae, as_ = oracle.quantize_mx(a, oracle.E4M3, oracle.ROW, oracle.CEIL)
    be, bs = oracle.quantize_mx(b, bfmt, oracle.ROW, oracle.FLOOR if bname == "e2m1" else oracle.CEIL)
    ref, mag = oracle.gemm_ref_block(ae, as_, oracle.E4M3, be, bs, bfmt, M, N, K, 0, M, 0, N)
    return bool(np.all(np.abs(c - ref) <= 1e-3 * mag + 2.0 ** (np.floor(np.log2(np.abs(ref) + 1e-3 * mag + 1e-30)) - 8)))


def case_misc():
    x = synth.normal(1, 1004, seed=3)
    out = mx.cast(dev(x).reshape(-1), "e2m1")
    ok = np.array_equal(host(out), oracle.cast(x, oracle.E2M1))
    w = synth.weight_fp4(256, 384, seed=4)
    q = mx.quantize(dev(w), "e2m1", "row", "floor", layout="rowmajor")
    o8 = torch.empty(256 * 384, dtype=torch.uint8, device="cuda")
    bsc = torch.empty(6, dtype=torch.float32, device="cuda")
    bok = torch.empty(6, dtype=torch.uint8, device="cuda")
    L.check(L.lib.mx_mxfp4_to_fp8_blocks(q.elems.data_ptr(), q.scales.data_ptr(), 256, 384, o8.data_ptr(),
                                         bsc.data_ptr(), bok.data_ptr(), torch.cuda.current_stream().cuda_stream),
            "nested")
    e, s = oracle.quantize_mx(w, oracle.E2M1, oracle.ROW, oracle.FLOOR)
    ref, _, _ = oracle.mxfp4_to_fp8_blocks(e, s, 256, 384)
    return ok and np.array_equal(host(o8), ref.reshape(-1))


CASES = {
    "rows_e4m3_37x96": lambda: case_rows(37, 96, 0, "e4m3", "ceil"),
    "rows_e2m1_130x160": lambda: case_rows(130, 160, 2, "e2m1", "floor"),
    "rows_e2m3_257x288": lambda: case_rows(257, 288, 4, "e2m3", "ceil"),
    "dual_e4m3_96x160": lambda: case_dual(96, 160, 0, "e4m3"),
    "dual_e2m1_160x384": lambda: case_dual(160, 384, 2, "e2m1"),
    "nvfp4_forms_144x288": lambda: case_nvfp4(144, 288),
    "gemm_e4m3_256x512x256": lambda: case_gemm(256, 512, 256, "e4m3", oracle.E4M3),
    "gemm_e2m1_128x384x256": lambda: case_gemm(128, 384, 256, "e2m1", oracle.E2M1),
    "cast_and_nested": case_misc,
}

if __name__ == "__main__":
    assert os.environ.get("MX_LIB_PATH", "").endswith("libmx_checked.so"), "run with the checked build"
    only = sys.argv[1:] or list(CASES)
    res = {}
    for name in only:
        ok = bool(CASES[name]())
        torch.cuda.synchronize()
        res[name] = {"match": ok, "watchdog": code()}
    print(json.dumps(res))
