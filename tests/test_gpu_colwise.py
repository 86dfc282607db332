"""GPU parity of the column-wise (transposed) grouped quantization
(qz_quantize_grouped_colwise) against the oracle (row-wise quantization of
the transpose): both formats, both layouts, ragged rows and columns (columns
not a multiple of 8 or 128 included), empty experts, strided inputs,
canary-guarded outputs, invalid entries, grid invariance and agreement with
the row-wise kernel on the explicitly transposed tensor."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import Guarded, assert_bytes_equal, host_bits

pytestmark = pytest.mark.gpu

qz = pytest.importorskip("nvfp4_quantization_moe_b200")
LAYOUTS = [qz.SF_LINEAR, qz.SF_SWIZZLED]


def run_colwise(xs, fmt, layout, amaxes=None, err=None, max_ctas=0):
    entries, keep = [], []
    for i, x in enumerate(xs):
        rows, cols = x.shape
        qb = rows * cols if fmt == qz.FMT_MXFP8 else rows * cols // 2
        q = Guarded(qb)
        sf = Guarded(qz.sf_bytes(cols, rows, fmt, layout) if rows else 0)
        a = None
        if fmt == qz.FMT_NVFP4:
            a = torch.tensor([amaxes[i]], dtype=torch.float32, device="cuda")
        entries.append(qz.Entry(x, q.view, sf.view, a))
        keep.append((q, sf))
    qz.quantize_grouped_colwise(qz.ExpertTable(entries, device=torch.device("cuda")), fmt, layout, err=err,
                                max_ctas=max_ctas)
    torch.cuda.synchronize()
    return keep


def check(xs, fmt, layout, keep, amaxes=None):
    for i, (x, (q, sf)) in enumerate(zip(xs, keep)):
        assert q.guards_intact() and sf.guards_intact(), f"expert {i}: write outside its buffers"
        if x.shape[0] == 0:
            continue
        xb = host_bits(x)
        if fmt == qz.FMT_MXFP8:
            rq, rsf = oracle.quantize_colwise(xb, oracle.MXFP8, layout)
        else:
            rq, rsf, _ = oracle.quantize_colwise(xb, oracle.NVFP4, layout, oracle.NVFP4_PER_TENSOR_GIVEN, amaxes[i])
        assert_bytes_equal(q.host(), rq.reshape(-1), f"expert {i} payload")
        assert_bytes_equal(sf.host(), rsf, f"expert {i} scales")


SHAPES = [(32, 8), (64, 130), (128, 128), (96, 37), (256, 257), (0, 64), (160, 1000), (512, 96)]


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("fmt", [qz.FMT_MXFP8, qz.FMT_NVFP4])
def test_shapes(fmt, layout):
    # blocks of 16 with their own scale running down the columns (the transpose of a
    # row-blocked matrix); rows are padded to a multiple of 8 elements (16-byte rows)
    xs = []
    for i, (r, c) in enumerate(SHAPES):
        base = torch.zeros((r, (c + 7) // 8 * 8), dtype=torch.bfloat16, device="cuda")
        if r:
            base[:, :c] = synth.blockwise_scaled((c, r), 16, seed=700 + i, lo=-12, hi=12).t().cuda()
        xs.append(base[:, :c])
    amaxes = [float(x.float().abs().max()) if x.numel() else 1.0 for x in xs]
    check(xs, fmt, layout, run_colwise(xs, fmt, layout, amaxes), amaxes)


@pytest.mark.parametrize("fmt", [qz.FMT_MXFP8, qz.FMT_NVFP4])
def test_strided_input_and_grid_invariance(fmt):
    base = synth.normal_bf16((192, 400), 1.0, seed=71).cuda()
    xs = [base[:, 16:272], base[:128, 8:40]]   # row stride 400, column offsets 16 and 8 elements
    amaxes = [float(x.float().abs().max()) * 1.5 for x in xs]
    for max_ctas in (1, 5, 0):
        check(xs, fmt, qz.SF_SWIZZLED, run_colwise(xs, fmt, qz.SF_SWIZZLED, amaxes, max_ctas=max_ctas), amaxes)


def test_same_bytes_as_rowwise_on_the_transpose():
    x = synth.blockwise_scaled((384, 256), 32, seed=72, lo=-8, hi=8).t().contiguous().cuda()
    keep = run_colwise([x], qz.FMT_MXFP8, qz.SF_SWIZZLED)
    xt = x.t().contiguous()
    ents = qz.alloc_outputs([xt], qz.FMT_MXFP8, qz.SF_SWIZZLED)
    qz.quantize_grouped_mxfp8(qz.ExpertTable(ents), qz.SF_SWIZZLED)
    torch.cuda.synchronize()
    q, sf = keep[0]
    assert_bytes_equal(q.host(), ents[0].q.cpu().numpy().reshape(-1), "payload vs row-wise of x^T")
    assert_bytes_equal(sf.host(), ents[0].sf.cpu().numpy(), "scales vs row-wise of x^T")


def test_invalid_entries_are_skipped_and_reported():
    x = synth.normal_bf16((64, 64), 1.0, seed=73).cuda()
    q = torch.zeros(64 * 64, dtype=torch.uint8, device="cuda")
    sf = torch.zeros(qz.sf_bytes(64, 64, qz.FMT_MXFP8, qz.SF_LINEAR), dtype=torch.uint8, device="cuda")
    bad_q = torch.zeros(64 * 64, dtype=torch.uint8, device="cuda")
    raw = [(x.data_ptr(), 64, 64, 64, q.data_ptr(), sf.data_ptr(), 0),
           (x.data_ptr(), 40, 64, 64, bad_q.data_ptr(), sf.data_ptr(), 0),         # rows % 32
           (x.data_ptr() + 2, 64, 64, 64, bad_q.data_ptr(), sf.data_ptr(), 0),     # x misaligned
           (x.data_ptr(), 64, 64, 64, 0, sf.data_ptr(), 0)]                        # q NULL
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    qz.quantize_grouped_colwise(qz.ExpertTable.from_raw(raw, "cuda"), qz.FMT_MXFP8, qz.SF_LINEAR, err=err)
    torch.cuda.synchronize()
    bits = int(err.item())
    assert bits & qz.DERR_SHAPE and bits & qz.DERR_ALIGN and bits & qz.DERR_NULL
    assert torch.count_nonzero(bad_q).item() == 0
    rq, rsf = oracle.quantize_colwise(host_bits(x), oracle.MXFP8, oracle.LINEAR)
    assert_bytes_equal(q.cpu().numpy(), rq.reshape(-1), "valid entry payload")
