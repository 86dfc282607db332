"""Pins of the oracle's column-wise quantization: a matrix built so that each
column holds known MXFP8 / NVFP4 blocks gets exactly those blocks' codes and
scales in the transposed payload, and column-wise quantization of x agrees
with the (pinned) row-wise quantization of x's transpose element by element
at every position (the transpose is the only step between them)."""
import numpy as np
import pytest

import oracle
import synth


def test_mxfp8_columns_of_known_blocks():
    """Column j is 2^j times a fixed ramp: its single 32-element block gets
    scale exponent e0 + j and the ramp's codes."""
    rows, cols = 32, 8
    ramp = ((np.arange(rows) - 16) / 8.0).astype(np.float32)   # multiples of 1/8: exact in bf16
    x = np.stack([ramp * np.float32(2.0 ** j) for j in range(cols)], axis=1)   # exact in binary32
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((xb.astype(np.uint32) << 16).view(np.float32), x)
    q, sf = oracle.quantize_colwise(xb, oracle.MXFP8, oracle.LINEAR)
    q0, sf0 = oracle.quantize_mxfp8(xb[:, :1].T.copy(), oracle.LINEAR)
    assert q.shape == (cols, rows)
    for j in range(cols):
        assert np.array_equal(q[j], q0[0])                  # same codes
        assert int(sf[j]) == int(sf0[0]) + j                # scale exponent steps by one per column


@pytest.mark.parametrize("layout", [oracle.LINEAR, oracle.SWIZZLED])
def test_colwise_is_rowwise_of_the_transpose(layout):
    x = synth.bf16_bits(synth.blockwise_scaled((96, 160), 16, seed=41))
    q, sf = oracle.quantize_colwise(x, oracle.MXFP8, layout)
    for c in (0, 77, 159):
        qc, _ = oracle.quantize_mxfp8(np.ascontiguousarray(x[:, c][None, :]), oracle.LINEAR)
        assert np.array_equal(q[c], qc[0])
    q4, sf4, a4 = oracle.quantize_colwise(x, oracle.NVFP4, layout, oracle.NVFP4_PER_TENSOR_COMPUTE)
    assert q4.shape == (160, 48)
    full = np.abs((x.astype(np.uint32) << 16).view(np.float32)).max()
    assert a4[0] == np.float32(full)                        # the tensor amax does not depend on orientation
