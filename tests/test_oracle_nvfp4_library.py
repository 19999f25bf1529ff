"""CPU pin of the oracle's NVFP4 quantiser against an independent library routine:
vLLM's torch reference NVFP4 quantiser (the emulation path it checks its NVFP4 kernels
against).  It takes the per-tensor encode scale gs = 6 * 448 / amax (the reciprocal of the
oracle's decode scale g = amax / 2688), quantises each 16-block's scale
gs * amax_b / 6 to E4M3 and each element x * gs / dec(sb) to E2M1, ties to even.

The two differ only in where fp32 rounding happens (the library multiplies by rounded
reciprocals where the oracle divides once), so the test requires equal scale and element
codes everywhere except where the exact quotient lies within 2^-20 (relative) of a
rounding midpoint, and there only one code apart.  Where g is a power of two the scales
must agree exactly.  A dropped factor of 6 or 448, a transposed block, a wrong tie rule
or a scale rounded the wrong way would fail it."""
import ml_dtypes
import numpy as np
import pytest
import torch

import synth
from conftest import f32_to_bf16_bits
from test_oracle_formats import bf16_bits_to_f64, unpack_fp4

try:
    from vllm.model_executor.layers.quantization.utils.nvfp4_emulation_utils import ref_nvfp4_quant
except Exception:                                        # pragma: no cover - library absent
    ref_nvfp4_quant = None

E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E2M1_MID = (E2M1_MAG[1:] + E2M1_MAG[:-1]) / 2
UE4M3 = np.arange(0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
UE4M3_MID = (UE4M3[1:] + UE4M3[:-1]) / 2
NEAR = 2.0 ** -20


def near_midpoint(v, mids):
    v = np.abs(np.asarray(v, dtype=np.float64))
    return (np.abs(v[..., None] - mids) <= NEAR * np.maximum(v, 1e-300)[..., None]).any(-1)


def case(name):
    if name == "weight_pow2_g":
        x = synth.weight_fp4(256, 1024, seed=21)
        m = np.abs(bf16_bits_to_f64(x)).max()
        k = int(np.floor(np.log2(2688.0 / m)))
        x[17, 333] = f32_to_bf16_bits([2688.0 * 2.0 ** -k])[0]       # amax = 2688 * 2^-k: g = 2^-k
        return x, True
    if name == "activations_general_g":
        return synth.activations(128, 2048, seed=22), False
    if name == "wide_range_pow2_g":                      # most block scales land on subnormal or zero UE4M3
        x = synth.normal(128, 1024, sigma=1.0, seed=23)
        x[5, 40] = f32_to_bf16_bits([2688.0 * 2.0 ** 9])[0]
        return x, True
    raise ValueError(name)


@pytest.mark.skipif(ref_nvfp4_quant is None, reason="vllm's reference NVFP4 quantiser is not importable")
@pytest.mark.parametrize("name", ["weight_pow2_g", "activations_general_g", "wide_range_pow2_g"])
def test_nvfp4_matches_library_reference(oracle, name):
    x, pow2_g = case(name)
    rows, cols = x.shape
    xf = bf16_bits_to_f64(x)
    e, s, g = oracle.quantize_nvfp4(x)
    amax = np.abs(xf).max()
    assert g == float(np.float32(amax) / np.float32(2688.0))
    if pow2_g:
        assert g == 2.0 ** np.round(np.log2(g))

    gs = torch.tensor(np.float32(2688.0) / np.float32(amax), dtype=torch.float32)
    lib_vals, lib_scale = ref_nvfp4_quant(torch.from_numpy(xf.astype(np.float32)), gs, 16)
    lib_s = lib_scale.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    lib_v = lib_vals.numpy().astype(np.float64)

    # scales
    amax_b = np.abs(xf).reshape(rows, cols // 16, 16).max(-1)
    t = amax_b / (6.0 * g)
    bad_s = lib_s != s
    if pow2_g:
        assert not bad_s.any()
    else:
        assert near_midpoint(t[bad_s], UE4M3_MID).all()
        assert (np.abs(lib_s[bad_s].astype(int) - s[bad_s].astype(int)) == 1).all()

    # elements, in the blocks whose scales agree
    ours = np.stack([unpack_fp4(e[r], cols) for r in range(rows)])
    mag_ours = ours & 0x7
    mag_lib = np.searchsorted(E2M1_MAG, np.abs(lib_v))
    assert np.array_equal(E2M1_MAG[mag_lib], np.abs(lib_v))          # the library returned E2M1 values
    same_block = np.repeat(~bad_s, 16, axis=1)
    d = UE4M3[s.astype(int)].repeat(16, axis=1) * g
    q = np.divide(xf, d, out=np.zeros_like(xf), where=d > 0)
    bad_e = same_block & (mag_ours != mag_lib)
    assert near_midpoint(q[bad_e], E2M1_MID).all()
    assert (np.abs(mag_ours[bad_e].astype(int) - mag_lib[bad_e].astype(int)) == 1).all()
    nz = same_block & (mag_ours > 0) & (mag_lib > 0)
    assert np.array_equal((ours[nz] >> 3) == 1, lib_v[nz] < 0)
    # and the comparison is not vacuous: almost every element is compared and agrees
    agree = same_block & (mag_ours == mag_lib)
    assert agree.mean() > 0.999
    if name == "wide_range_pow2_g":
        assert (s == 0).mean() > 0.5 and ((s > 0) & (s < 8)).any()   # zero and subnormal scales reached
    else:
        assert (mag_ours[same_block] == 7).any() and (mag_ours[same_block] == 1).any()
