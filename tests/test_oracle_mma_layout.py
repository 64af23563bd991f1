"""Pins of the oracle's block-scaled MMA scale layout (oracle.c, "Scale-factor layout read by
the block-scaled tensor-core MMA"), against things other than itself:
- a library's rearrangement helper for the scales of cuBLAS's block-scaled GEMMs (`to_blocked`
  from torch's testing utilities, or the same helper shipped by the quack kernel library when
  torch's test dependencies are absent);
- hand-computed offsets of single entries;
- structure: a bijection of the real entries onto the non-padding bytes, padding zero.
The pages themselves do not define the layout ("Sonar: Online MXFP6", Current limits, only says
the converted weights feed block-scaled GEMMs with dimensions in multiples of 128)."""
import numpy as np
import pytest
import torch

import oracle
from synthetic import uniform_ints

try:
    from torch.testing._internal.common_quantized import to_blocked
except ImportError:
    to_blocked = pytest.importorskip("quack.mx_utils").to_blocked

SHAPES = [(1, 1), (1, 4), (3, 5), (127, 3), (128, 4), (129, 4), (128, 5), (200, 9), (256, 32), (300, 33), (513, 7)]


def random_scales(rows, kb, seed):
    return np.asarray(uniform_ints(seed, 11, rows * kb, 255), dtype=np.uint8).reshape(rows, kb)


@pytest.mark.parametrize("rows,kb", SHAPES)
def test_layout_equals_torch_to_blocked(rows, kb):
    s = random_scales(rows, kb, rows * 1000 + kb)
    want = to_blocked(torch.from_numpy(s)).numpy()
    got = oracle.swizzle_scales(s)
    assert got.shape == want.shape
    assert np.array_equal(got, want)


def test_single_offsets_by_hand():
    # kb = 8 -> 2 tiles per tile-row. (r=33, k=5): tile (0, 1) -> 512; r%32 = 1 -> +16; r/32 = 1 -> +4; k%4 = 1 -> +1
    assert oracle.mma_scale_index(33, 5, 8) == 533
    # last entry of the first tile
    assert oracle.mma_scale_index(127, 3, 8) == 31 * 16 + 3 * 4 + 3
    # (r=128, k=0) starts the second tile-row: tiles per row = ceil(5/4) = 2 -> tile 2
    assert oracle.mma_scale_index(128, 0, 5) == 2 * 512
    # rows 0, 32, 64, 96 of a tile share one 16-byte line
    assert [oracle.mma_scale_index(r, 0, 4) for r in (0, 32, 64, 96)] == [0, 4, 8, 12]
    assert oracle.mma_scales_bytes(129, 5) == 256 * 8
    assert oracle.mma_scales_bytes(0, 5) == 0


@pytest.mark.parametrize("rows,kb", [(1, 1), (130, 6), (257, 13)])
def test_bijection_and_zero_padding(rows, kb):
    idx = np.array([[oracle.mma_scale_index(r, k, kb) for k in range(kb)] for r in range(rows)])
    n = oracle.mma_scales_bytes(rows, kb)
    assert len(np.unique(idx)) == rows * kb and idx.min() >= 0 and idx.max() < n
    s = np.full((rows, kb), 0xA5, dtype=np.uint8)
    out = oracle.swizzle_scales(s)
    mask = np.zeros(n, dtype=bool)
    mask[idx.ravel()] = True
    assert np.all(out[mask] == 0xA5) and np.all(out[~mask] == 0)
