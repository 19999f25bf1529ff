import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name):
    """Parse a tests/golden/*.txt fixture: 'key: v1 v2 ...' lines, '#' comments."""
    out = {}
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split(":", 1)
            out[k.strip()] = [float(t) for t in v.split()]
    return out


def pack_codes(codes, bits):
    """Codes (one per entry, last axis along a row) -> the dense little-endian bit packing:
    code i at bits [bits*i, bits*i + bits) of the row.  numpy's bit routines, independent of
    the oracle's bit loop and the kernels' word arithmetic."""
    c = np.asarray(codes, dtype=np.uint8)
    b = np.unpackbits(c[..., None], axis=-1, bitorder="little")[..., :bits]
    return np.packbits(b.reshape(*c.shape[:-1], -1), axis=-1, bitorder="little")


def unpack_codes(packed, n, bits):
    """Inverse of pack_codes for rows of n codes."""
    p = np.asarray(packed, dtype=np.uint8)
    b = np.unpackbits(p, axis=-1, bitorder="little")[..., :n * bits].reshape(*p.shape[:-1], n, bits)
    return np.packbits(b, axis=-1, bitorder="little")[..., 0]


def f32_to_bf16_bits(values):
    """Exact fp32 values (already bf16-representable) -> bf16 bit patterns."""
    a = np.asarray(values, dtype=np.float32)
    bits = a.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0), "value not representable in bf16"
    return (bits >> 16).astype(np.uint16)


@pytest.fixture(scope="session")
def oracle():
    import oracle as o
    o.lib()
    return o
