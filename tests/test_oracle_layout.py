"""Pins of the oracle's scale-factor layouts: hand-worked offsets from the
cuBLAS block-scaling layout description and the linear formula printed on the
linear-SF epilogue page, bijection and padding properties, round trips."""
import numpy as np
import pytest

import oracle
from golden_io import rows


def test_swizzle_offsets_golden(olib):
    for kv, r, k, off in rows("swizzle_128x4.txt"):
        assert olib.qzo_sf_offset_swizzled(int(r), int(k), int(kv)) == int(off), (kv, r, k)


def test_linear_offsets_golden(olib):
    for kv, r, k, off in rows("sf_linear.txt"):
        assert olib.qzo_sf_offset_linear(int(r), int(k), int(kv)) == int(off)


@pytest.mark.parametrize("rows_,kv", [(1, 1), (64, 8), (128, 4), (129, 6), (300, 24), (1536, 64), (7, 448)])
def test_swizzle_bijection_and_size(olib, rows_, kv):
    n = olib.qzo_sf_region_bytes(rows_, kv, 1)
    assert n == (-(-rows_ // 128) * 128) * (-(-kv // 4) * 4)
    seen = np.zeros(n, dtype=np.int32)
    for r in range(rows_):
        for k in range(kv):
            off = olib.qzo_sf_offset_swizzled(r, k, kv)
            assert 0 <= off < n
            seen[off] += 1
    assert seen.max() == 1 and seen.sum() == rows_ * kv


@pytest.mark.parametrize("rows_,kv", [(1, 1), (129, 6), (300, 24)])
def test_swizzle_round_trip_and_zero_padding(olib, rows_, kv):
    rng = np.random.default_rng(rows_ * 31 + kv)
    lin = rng.integers(1, 255, rows_ * kv, dtype=np.uint8)
    swz = oracle.swizzle(lin, rows_, kv)
    assert np.array_equal(oracle.unswizzle(swz, rows_, kv), lin)
    assert np.count_nonzero(swz) == rows_ * kv           # every padding byte is 0x00


def test_region_bytes_empty_and_linear(olib):
    assert olib.qzo_sf_region_bytes(0, 8, 1) == 0
    assert olib.qzo_sf_region_bytes(0, 8, 0) == 0
    assert olib.qzo_sf_region_bytes(5, 7, 0) == 35
    assert olib.qzo_sf_region_bytes(5, 7, 1) == 128 * 8
