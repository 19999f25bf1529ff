"""CPU pin of the oracle's tcgen05 scale tiling against an independent library routine:
vLLM's torch implementation of the block-scaling-factor layout that cuBLAS documents for
its block-scaled matmuls (128-row x 4-column atoms, 32 x 16-byte interleave), the layout
the Blackwell block-scaled MMA reads.  The routine needs its input zero-padded to whole
atoms; the oracle pads with zeros itself."""
import numpy as np
import pytest
import torch

import oracle

try:
    from vllm.model_executor.layers.quantization.qutlass_utils import to_blocked
except Exception:                                        # pragma: no cover - library absent
    to_blocked = None


@pytest.mark.skipif(to_blocked is None, reason="vllm's blocked-layout routine is not importable")
@pytest.mark.parametrize("rows,S", [(1, 1), (31, 3), (128, 4), (130, 5), (257, 33), (384, 64), (1000, 7),
                                    (4096, 256), (16384, 128)])
def test_tcgen05_tiling_matches_library_layout(rows, S):
    s = np.random.default_rng(rows * 131 + S).integers(0, 256, size=(rows, S), dtype=np.uint8)
    ours = oracle.to_tcgen05_layout(s).reshape(-1)
    R, C = -(-rows // 128) * 128, -(-S // 4) * 4
    padded = np.zeros((R, C), dtype=np.uint8)
    padded[:rows, :S] = s
    ref = to_blocked(torch.from_numpy(padded), backend="torch").numpy().reshape(-1)
    assert ours.shape == ref.shape
    assert np.array_equal(ours, ref)
    # and the inverse mapping recovers the rows-by-S array
    assert np.array_equal(oracle.from_tcgen05_layout(ours, rows, S), s)
