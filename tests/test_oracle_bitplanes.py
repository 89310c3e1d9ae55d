"""Pins for the oracle's bit-plane packing/decoding (CPU only)."""
import numpy as np
import pytest

from any_precision_expert_pw_b200.inputs import random_indices
from oracle.bitplanes import child_index, pack_bitplanes, unpack_bitplanes


def test_hand_built_ramp(golden):
    g = golden("bitplanes_ramp.json")
    idx = np.array(g["idx"], dtype=np.uint8)
    planes = pack_bitplanes(idx, g["n"])
    want = np.array([[int(h, 16) for h in row] for row in g["planes_hex"]], dtype=np.uint32)
    assert planes.shape == (8, 2, 1)
    assert np.array_equal(planes[:, :, 0], want)
    assert unpack_bitplanes(planes, 5)[0].tolist() == g["q5_row0"]
    assert unpack_bitplanes(planes, 3)[1].tolist() == g["q3_row1"]


@pytest.mark.parametrize("n", [4, 8])
def test_round_trip_and_top_bits(n):
    idx = random_indices(7, 96, n, seed=1)
    planes = pack_bitplanes(idx, n)
    assert np.array_equal(unpack_bitplanes(planes, n), idx.astype(np.int64))
    for q in range(1, n + 1):
        # the b-bit index is the top b bits of the parent index, for every b
        assert np.array_equal(unpack_bitplanes(planes, q), idx.astype(np.int64) >> (n - q))
        assert np.array_equal(child_index(idx, n, q), idx.astype(np.int64) >> (n - q))


@pytest.mark.parametrize("n", [4, 8])
def test_plane_major_nesting(n):
    # the top q planes of the n-bit parent are exactly the planes of the q-bit child model
    idx = random_indices(5, 64, n, seed=2)
    planes = pack_bitplanes(idx, n)
    for q in range(1, n + 1):
        child = (idx >> (n - q)).astype(np.uint8)
        assert np.array_equal(planes[:q], pack_bitplanes(child, q))


def test_single_bit_positions():
    # one set bit at (row, column) lands in exactly one word of the matching plane
    n = 8
    for (r, c, v) in [(0, 0, 128), (1, 37, 1), (2, 63, 16), (0, 95, 255)]:
        idx = np.zeros((3, 96), dtype=np.uint8)
        idx[r, c] = v
        planes = pack_bitplanes(idx, n)
        for p in range(n):
            expect = np.zeros((3, 3), dtype=np.uint32)
            if (v >> (n - 1 - p)) & 1:
                expect[r, c // 32] = np.uint32(1) << np.uint32(c % 32)
            assert np.array_equal(planes[p], expect)


def test_rejects_ragged_columns():
    with pytest.raises(ValueError):
        pack_bitplanes(np.zeros((2, 33), dtype=np.uint8), 4)
