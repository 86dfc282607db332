"""Pins of the oracle's gate|up split of a folded fused expert (R14).

Model-Optimizer "Fold fused experts' quantizers into their weights
shard-locally": the fused (2I, H) expert is quantized once, gate and up
sharing one per-tensor amax, and the folded payload and scales are later cut
by rows into gate and up.  The review on that page states the property that
pins the cut: quantizing the fused tensor and slicing its scales equals
slicing first and quantizing each part (with the shared amax for a
per-tensor scale), because a block scale depends only on its own rows.  So
the split is checked against the oracle's own quantizers applied to each
part, which write their scales through a separate path.  The cut rule for
scales that span 128 rows (FP8 with 128 x 128 block scales) is checked on
hand-built cases, the page's 2880-row gate among them.
"""
import numpy as np
import pytest

import oracle
import synth

LAYOUT_PAIRS = [(oracle.LINEAR, oracle.LINEAR), (oracle.LINEAR, oracle.SWIZZLED),
                (oracle.SWIZZLED, oracle.LINEAR), (oracle.SWIZZLED, oracle.SWIZZLED)]


def fused(rows, cols, seed):
    return synth.bf16_bits(synth.blockwise_scaled((rows, cols), 16, seed=seed, lo=-10, hi=10))


@pytest.mark.parametrize("src,dst", LAYOUT_PAIRS)
@pytest.mark.parametrize("cut", [0, 1, 72, 128, 143, 144])
def test_mxfp8_split_equals_quantizing_each_part(src, dst, cut):
    rows, cols = 144, 96
    x = fused(rows, cols, 11 + cut)
    q, sf = oracle.quantize_mxfp8(x, src)
    parts = oracle.split_fused(oracle.MXFP8, q, sf, None, oracle.AMAX_NONE, cols, cut, src, dst)
    for (qp, sp, ap), (a, b) in zip(parts, [(0, cut), (cut, rows)]):
        rq, rsf = oracle.quantize_mxfp8(np.ascontiguousarray(x[a:b]), dst)
        assert np.array_equal(qp, rq.reshape(qp.shape))
        assert np.array_equal(sp, rsf)
        assert ap.size == 0


@pytest.mark.parametrize("src,dst", LAYOUT_PAIRS)
@pytest.mark.parametrize("cut", [0, 5, 72, 128, 144])
def test_nvfp4_split_shares_the_tensor_amax(src, dst, cut):
    """Per-tensor NVFP4: the fused amax is the one weight_scale_2 of gate and
    up; each part equals its own rows quantized with that given amax."""
    rows, cols = 144, 64
    x = fused(rows, cols, 31 + cut)
    q, sf, A = oracle.quantize_nvfp4(x, src, oracle.NVFP4_PER_TENSOR_COMPUTE)
    parts = oracle.split_fused(oracle.NVFP4, q, sf, A, oracle.AMAX_PER_TENSOR, cols, cut, src, dst)
    for (qp, sp, ap), (a, b) in zip(parts, [(0, cut), (cut, rows)]):
        assert ap.shape == (1,) and ap[0] == A[0]
        if b == a:
            assert qp.size == 0 and sp.size == 0
            continue
        rq, rsf, _ = oracle.quantize_nvfp4(np.ascontiguousarray(x[a:b]), dst, oracle.NVFP4_PER_TENSOR_GIVEN, A[0])
        assert np.array_equal(qp, rq.reshape(qp.shape))
        assert np.array_equal(sp, rsf)
    # the parts' own amaxes differ from the shared one in general: the share is not a no-op
    own = [np.abs((x[a:b].astype(np.uint32) << 16).view(np.float32)).max() for a, b in [(0, 72), (72, 144)]]
    assert own[0] != own[1]


@pytest.mark.parametrize("src,dst", LAYOUT_PAIRS)
def test_nvfp4_per_row_amax_is_cut_with_the_rows(src, dst):
    rows, cols, cut = 200, 48, 77
    x = fused(rows, cols, 5)
    q, sf, A = oracle.quantize_nvfp4(x, src, oracle.NVFP4_PER_ROW)
    parts = oracle.split_fused(oracle.NVFP4, q, sf, A, oracle.AMAX_PER_ROW, cols, cut, src, dst)
    for (qp, sp, ap), (a, b) in zip(parts, [(0, cut), (cut, rows)]):
        rq, rsf, rA = oracle.quantize_nvfp4(np.ascontiguousarray(x[a:b]), dst, oracle.NVFP4_PER_ROW)
        assert np.array_equal(ap, rA)
        assert np.array_equal(qp, rq.reshape(qp.shape))
        assert np.array_equal(sp, rsf)


def test_hand_worked_relayout():
    """Three rows, one scale column: linear bytes [10, 20, 30] cut after row 0
    into swizzled parts.  Swizzled row r, column 0 sits at byte
    ((r % 32) * 4 + (r // 32) % 4) * 4 inside a 512-byte tile, padding 0x00."""
    q = np.arange(3 * 32, dtype=np.uint8).reshape(3, 32)
    sf = np.array([10, 20, 30], dtype=np.uint8)
    (q0, s0, _), (q1, s1, _) = oracle.split_fused(oracle.MXFP8, q, sf, None, oracle.AMAX_NONE, 32, 1,
                                                  oracle.LINEAR, oracle.SWIZZLED)
    e0 = np.zeros(512, np.uint8)
    e0[0] = 10
    e1 = np.zeros(512, np.uint8)
    e1[0], e1[16] = 20, 30
    assert np.array_equal(s0, e0) and np.array_equal(s1, e1)
    assert np.array_equal(q0, q[:1]) and np.array_equal(q1, q[1:])


def block128_case(rows, cols, seed):
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 256, (rows, cols), dtype=np.uint8)
    srows, scols = -(-rows // 128), -(-cols // 128)
    s = (rng.standard_normal((srows, scols)) ** 2 + 0.25).astype(np.float32)
    return q, s


@pytest.mark.parametrize("rows,cut", [(256, 128), (300, 256), (300, 0), (300, 300), (128, 128), (5760, 2816)])
def test_fp8_block128_cut_on_a_block_boundary(rows, cut):
    cols = 200
    q, s = block128_case(rows, cols, rows + cut)
    parts = oracle.split_fused(oracle.FP8_BLOCK128, q, s.view(np.uint8), None, oracle.AMAX_NONE, cols, cut,
                               oracle.LINEAR, oracle.LINEAR)
    b = cut // 128                        # first scale row of part 1 (cut is on a block boundary or = rows)
    srows = [(0, -(-cut // 128)), (b, b - (-(rows - cut) // 128))]
    for (qp, sp, _), (ra, rb), (sa, sb) in zip(parts, [(0, cut), (cut, rows)], srows):
        assert np.array_equal(qp, q[ra:rb])
        assert np.array_equal(sp.view(np.float32), s[sa:sb].reshape(-1))


@pytest.mark.parametrize("rows,cut", [(5760, 2880), (200, 100), (384, 192), (300, 1)])
def test_fp8_block128_cut_inside_a_block_is_refused(rows, cut):
    """(5760, 2880) is a 2880-row gate over 128-row blocks (the page's example).
    (200, 100): the proportional count 2 * 100 / 200 = 1 scale row is an
    integer, yet block 0 covers rows 0-127 of both parts, so it is refused."""
    q, s = block128_case(rows, 128, 3)
    with pytest.raises(oracle.CutRefused):
        oracle.split_fused(oracle.FP8_BLOCK128, q, s.view(np.uint8), None, oracle.AMAX_NONE, 128, cut,
                           oracle.LINEAR, oracle.LINEAR)


@pytest.mark.parametrize("fmt", [oracle.MXFP8, oracle.NVFP4])
def test_parts_reassemble_the_fused_scales(fmt):
    rows, cols, cut = 300, 128, 131
    x = fused(rows, cols, 77)
    if fmt == oracle.MXFP8:
        q, sf = oracle.quantize_mxfp8(x, oracle.LINEAR)
        A, kind = None, oracle.AMAX_NONE
    else:
        q, sf, A = oracle.quantize_nvfp4(x, oracle.LINEAR, oracle.NVFP4_PER_TENSOR_COMPUTE)
        kind = oracle.AMAX_PER_TENSOR
    kv = cols // (32 if fmt == oracle.MXFP8 else 16)
    parts = oracle.split_fused(fmt, q, sf, A, kind, cols, cut, oracle.LINEAR, oracle.SWIZZLED)
    lin = [oracle.unswizzle(sp, n, kv) for (_, sp, _), n in zip(parts, (cut, rows - cut))]
    assert np.array_equal(np.concatenate(lin), sf)
    assert np.array_equal(np.concatenate([p[0] for p in parts]), q.reshape(rows, -1))
    for (_, sp, _), n in zip(parts, (cut, rows - cut)):
        live = np.zeros(sp.size, bool)
        for r in range(n):
            for k in range(kv):
                live[oracle.load().qzo_sf_offset_swizzled(r, k, kv)] = True
        assert np.all(sp[~live] == 0), "padding of a part's swizzled region must be 0x00"
