"""The watchdog path of the bounded device waits, exercised without any fault: a
diagnostic kernel waits on a barrier that nothing arrives at, the wait gives up after
its short limit, records its code in the device flag and the kernel returns.  The flag
is then read and cleared through the C ABI, and ordinary calls afterwards are bit-exact
against the oracle (the context and the GPU stay usable)."""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import microscaling_precision_number_b200 as mx
    from microscaling_precision_number_b200 import _lib as L


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def status(clear):
    code = ctypes.c_int(-1)
    st = L.lib.mx_watchdog_status(ctypes.byref(code), 1 if clear else 0)
    return st, code.value


@pytest.mark.parametrize("limit_us", [1000, 20000])
def test_selftest_wait_gives_up_and_is_reported(oracle, limit_us):
    assert status(True)[0] in (L.MX_OK, L.MX_ERR_TIMEOUT)
    assert status(False) == (L.MX_OK, 0)
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    assert L.lib.mx_watchdog_selftest(limit_us, stream.cuda_stream) == L.MX_OK
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    assert limit_us * 1e-3 * 0.9 <= ms < limit_us * 1e-3 + 50.0          # it waited its limit, then returned
    assert status(False) == (L.MX_ERR_TIMEOUT, L.WD_SELFTEST)            # reported, still set
    assert status(True) == (L.MX_ERR_TIMEOUT, L.WD_SELFTEST)             # reported and cleared
    assert status(False) == (L.MX_OK, 0)
    # ordinary calls after the timeout: pipelined streaming, TMA-staged and matmul kernels
    x = synth.weight_fp4(256, 1024, seed=limit_us)
    q = mx.quantize(to_dev(x), "nvfp4", "row", "ceil", layout="rowmajor")
    e, s, g = oracle.quantize_nvfp4(x)
    assert np.array_equal(q.elems.cpu().numpy(), e.reshape(-1))
    assert np.array_equal(q.scales.cpu().numpy(), s.reshape(-1))
    qr, qc = mx.quantize_dual(to_dev(x), "e4m3", "ceil", "rowmajor")
    er, sr = oracle.quantize_mx(x, oracle.E4M3, oracle.ROW, oracle.CEIL)
    ec, sc = oracle.quantize_mx(x, oracle.E4M3, oracle.COL, oracle.CEIL)
    assert np.array_equal(qr.elems.cpu().numpy(), er.reshape(-1))
    assert np.array_equal(qc.elems.cpu().numpy(), ec.reshape(-1))
    a8 = mx.quantize(to_dev(x), "e4m3", "row", "ceil", layout="tcgen05")
    c = mx.gemm(a8, a8)
    torch.cuda.synchronize()
    assert torch.isfinite(c.float()).all()
    assert status(False) == (L.MX_OK, 0)
