"""GPU parity of the gate|up split of folded fused experts
(qz_split_fused_experts) against the oracle: MXFP8 and NVFP4 in every pair
of source and destination SF layouts (cuts on and off the 128-row tiles,
scale columns not a multiple of 4, empty parts), per-tensor and per-row
amax, FP8 with 128 x 128 FP32 block scales including the refused cut of a
2880-row gate, unaligned payload outputs, canary-guarded buffers, invalid
entries, grid invariance; and the fold itself done on the GPU: a fused
expert quantized once and split equals its parts quantized with the shared
amax, with gate and up entries sharing one amax slot."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import Guarded, assert_bytes_equal

pytestmark = pytest.mark.gpu

qz = pytest.importorskip("nvfp4_quantization_moe_b200")
LAYOUT_PAIRS = [(0, 0), (0, 1), (1, 0), (1, 1)]


def row_bytes(fmt, cols):
    return cols // 2 if fmt == qz.FMT_NVFP4 else cols


def folded(fmt, rows, cols, src, seed):
    """A folded expert as random bytes: payload, source SF region (padding
    bytes random too: nothing may read them) and amax slots."""
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 256, (rows, row_bytes(fmt, cols)), dtype=np.uint8)
    nsf = qz.sf_bytes(rows, cols, fmt, src)
    sf = rng.integers(0, 256, nsf, dtype=np.uint8)
    amax = (rng.random(max(rows, 1)) * 10 + 0.5).astype(np.float32)
    return q, sf, amax


def run_split(cases, fmt, amax_kind, src, dst, err=None, max_ctas=0, q_offset=0):
    """cases: [(q, sf, amax, rows, cols, cut)] host arrays.  Returns, per case,
    the guarded outputs [(q_p, sf_p, amax_p)] for p = 0, 1."""
    entries, outs, keep = [], [], []
    for q, sf, amax, rows, cols, cut in cases:
        dq = torch.from_numpy(q).cuda() if q.size else torch.empty(16, dtype=torch.uint8, device="cuda")
        dsf = Guarded(max(sf.size, 1))
        if sf.size:
            dsf.view.copy_(torch.from_numpy(sf))
        da = torch.from_numpy(amax).cuda()
        parts = []
        for n in (cut, rows - cut):
            qp = Guarded(n * row_bytes(fmt, cols) + q_offset)
            sp = Guarded(qz.sf_bytes(n, cols, fmt, dst))
            na = 1 if amax_kind == qz.AMAX_PER_TENSOR else (n if amax_kind == qz.AMAX_PER_ROW else 0)
            ap = Guarded(4 * na)
            parts.append((qp, sp, ap))
        keep.append((dq, dsf, da))
        outs.append(parts)
        entries.append(qz.SplitEntry(
            q=dq, sf=dsf.view, rows=rows, cols=cols, cut=cut,
            sf_out=tuple(p[1].view for p in parts),
            q_out=tuple(p[0].view[q_offset:] for p in parts),
            amax=da if amax_kind != qz.AMAX_NONE else None,
            amax_out=tuple(p[2].view.view(torch.float32) if amax_kind != qz.AMAX_NONE else None for p in parts)))
    qz.split_fused_experts(qz.SplitTable(entries, device=torch.device("cuda")), fmt, amax_kind, src, dst, err=err,
                           max_ctas=max_ctas)
    torch.cuda.synchronize()
    return outs


def check(cases, outs, fmt, amax_kind, src, dst, q_offset=0):
    for i, ((q, sf, amax, rows, cols, cut), parts) in enumerate(zip(cases, outs)):
        ref = oracle.split_fused(fmt, q, sf, amax if amax_kind else None, amax_kind, cols, cut, src, dst)
        for p, ((qp, sp, ap), (rq, rsf, ra)) in enumerate(zip(parts, ref)):
            assert qp.guards_intact() and sp.guards_intact() and ap.guards_intact(), f"case {i} part {p}: overrun"
            assert_bytes_equal(qp.host()[q_offset:], rq.reshape(-1), f"case {i} part {p} payload")
            assert_bytes_equal(sp.host(), rsf, f"case {i} part {p} scales")
            if amax_kind != qz.AMAX_NONE:
                assert_bytes_equal(ap.host().view(np.float32), ra, f"case {i} part {p} amax")


SHAPES = {
    qz.FMT_MXFP8: [(256, 64, 128), (144, 96, 72), (300, 128, 131), (1, 32, 0), (1, 32, 1), (0, 32, 0),
                   (200, 160, 200), (130, 256, 3), (512, 128, 256), (300, 256, 128)],
    qz.FMT_NVFP4: [(144, 64, 72), (300, 48, 77), (5760, 2880, 2880), (16, 16, 8), (0, 16, 0), (129, 208, 128)],
}


@pytest.mark.parametrize("src,dst", LAYOUT_PAIRS)
def test_mxfp8(src, dst):
    cases = [(*folded(qz.FMT_MXFP8, r, c, src, 10 + i), r, c, k) for i, (r, c, k) in enumerate(SHAPES[qz.FMT_MXFP8])]
    outs = run_split(cases, qz.FMT_MXFP8, qz.AMAX_NONE, src, dst)
    check(cases, outs, qz.FMT_MXFP8, qz.AMAX_NONE, src, dst)


@pytest.mark.parametrize("amax_kind", [qz.AMAX_PER_TENSOR, qz.AMAX_PER_ROW])
@pytest.mark.parametrize("src,dst", LAYOUT_PAIRS)
def test_nvfp4(src, dst, amax_kind):
    cases = [(*folded(qz.FMT_NVFP4, r, c, src, 40 + i), r, c, k) for i, (r, c, k) in enumerate(SHAPES[qz.FMT_NVFP4])]
    outs = run_split(cases, qz.FMT_NVFP4, amax_kind, src, dst)
    check(cases, outs, qz.FMT_NVFP4, amax_kind, src, dst)


def fp8_block128_case(rows, cols, cut, seed):
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 256, (rows, cols), dtype=np.uint8)
    s = (rng.random((-(-rows // 128)) * (-(-cols // 128))) + 0.5).astype(np.float32)
    return (q, s.view(np.uint8), np.zeros(1, np.float32), rows, cols, cut)


def test_fp8_block128_whole_blocks_and_the_refused_cut():
    ok = [fp8_block128_case(256, 200, 128, 1), fp8_block128_case(300, 130, 256, 2),
          fp8_block128_case(5760, 2880, 2816, 3), fp8_block128_case(300, 64, 300, 4)]
    bad = fp8_block128_case(5760, 2880, 2880, 5)        # a 2880-row gate over 128-row blocks
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = run_split(ok + [bad], qz.FMT_FP8_BLOCK128, qz.AMAX_NONE, 0, 0, err=err)
    check(ok, outs[:4], qz.FMT_FP8_BLOCK128, qz.AMAX_NONE, 0, 0)
    assert int(err.item()) == qz.DERR_CUT
    for qp, sp, ap in outs[4]:                           # the refused entry wrote nothing
        assert np.all(qp.host() == 0xA5) and np.all(sp.host() == 0xA5)
    with pytest.raises(oracle.CutRefused):
        oracle.split_fused(oracle.FP8_BLOCK128, bad[0], bad[1], None, 0, 2880, 2880, 0, 0)


@pytest.mark.parametrize("q_offset", [1, 4, 8, 16])
def test_unaligned_payload_outputs(q_offset):
    cases = [(*folded(qz.FMT_NVFP4, r, c, 1, 70 + i), r, c, k) for i, (r, c, k) in enumerate([(300, 48, 77),
                                                                                          (2048, 1024, 1000)])]
    outs = run_split(cases, qz.FMT_NVFP4, qz.AMAX_PER_TENSOR, 1, 1, q_offset=q_offset)
    check(cases, outs, qz.FMT_NVFP4, qz.AMAX_PER_TENSOR, 1, 1, q_offset=q_offset)


@pytest.mark.parametrize("max_ctas", [1, 7, 0])
def test_grid_invariance(max_ctas):
    cases = [(*folded(qz.FMT_MXFP8, r, c, 1, 90 + i), r, c, k) for i, (r, c, k) in enumerate(SHAPES[qz.FMT_MXFP8])]
    outs = run_split(cases, qz.FMT_MXFP8, qz.AMAX_NONE, 1, 1, max_ctas=max_ctas)
    check(cases, outs, qz.FMT_MXFP8, qz.AMAX_NONE, 1, 1)


def test_payload_not_copied_when_no_output_is_given():
    q, sf, amax = folded(qz.FMT_NVFP4, 256, 64, 1, 7)
    dq, dsf = torch.from_numpy(q).cuda(), torch.from_numpy(sf).cuda()
    sfo = [Guarded(qz.sf_bytes(n, 64, qz.FMT_NVFP4, 1)) for n in (100, 156)]
    e = qz.SplitEntry(q=dq, sf=dsf, rows=256, cols=64, cut=100, sf_out=(sfo[0].view, sfo[1].view))
    qz.split_fused_experts(qz.SplitTable([e]), qz.FMT_NVFP4, qz.AMAX_NONE, 1, 1)
    torch.cuda.synchronize()
    ref = oracle.split_fused(oracle.NVFP4, q, sf, None, 0, 64, 100, 1, 1)
    for p in range(2):
        assert_bytes_equal(sfo[p].host(), ref[p][1], f"part {p} scales")


def test_invalid_entries_are_skipped_and_reported():
    good = folded(qz.FMT_MXFP8, 128, 64, 1, 3)
    dq = torch.from_numpy(good[0]).cuda()
    dsf = torch.from_numpy(good[1]).cuda()
    o = [Guarded(128 * 64) for _ in range(2)]
    s = [Guarded(qz.sf_bytes(64, 64, qz.FMT_MXFP8, 1) + 16) for _ in range(2)]
    P2 = lambda a, b: (a, b)  # noqa: E731
    qo = P2(o[0].view.data_ptr(), o[1].view.data_ptr())
    so = P2(s[0].view.data_ptr(), s[1].view.data_ptr())
    raw = [
        (dq.data_ptr(), dsf.data_ptr(), 0, 128, 64, 129, qo, so, (0, 0)),          # cut past the end: shape
        (dq.data_ptr(), dsf.data_ptr(), 0, 128, 48, 64, qo, so, (0, 0)),           # cols not a multiple of 32
        (dq.data_ptr(), 0, 0, 128, 64, 64, qo, so, (0, 0)),                         # no source scales: null
        (dq.data_ptr(), dsf.data_ptr(), 0, 128, 64, 64, qo, (so[0] + 4, so[1]), (0, 0)),  # swizzled dst misaligned
    ]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    qz.split_fused_experts(qz.SplitTable.from_raw(raw, torch.device("cuda")), qz.FMT_MXFP8, qz.AMAX_NONE, 1, 1,
                           err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == qz.DERR_SHAPE | qz.DERR_NULL | qz.DERR_ALIGN
    for g in o + s:
        assert np.all(g.raw.cpu().numpy() == 0xA5), "a skipped entry wrote bytes"


@pytest.mark.parametrize("layout", [qz.SF_LINEAR, qz.SF_SWIZZLED])
def test_fold_on_the_gpu_then_split_equals_quantizing_the_parts(layout):
    """Fused NVFP4 experts [2I, H] quantized on the GPU as whole tensors
    (computed amax), then split on the GPU, equal (a) the oracle quantizing
    each part with the fused amax and (b) the GPU quantizer run on gate and
    up entries that share one amax slot (the one-pass fold)."""
    E, I, H = 3, 200, 256              # I = 200: the cut falls inside a 128-row tile
    W = synth.blockwise_scaled((E * 2 * I, H), 16, seed=5, lo=-6, hi=6).cuda().view(E, 2 * I, H)
    q = torch.empty((E, 2 * I, H // 2), dtype=torch.uint8, device="cuda")
    nsf = qz.sf_bytes(2 * I, H, qz.FMT_NVFP4, layout)
    sf = torch.empty((E, max(nsf, 16)), dtype=torch.uint8, device="cuda")
    A = torch.empty((E, 1), dtype=torch.float32, device="cuda")
    qz.quantize_grouped_nvfp4(qz.ExpertTable([qz.Entry(W[e], q[e], sf[e], A[e]) for e in range(E)]),
                              qz.NVFP4_PER_TENSOR_COMPUTE, layout)
    npart = qz.sf_bytes(I, H, qz.FMT_NVFP4, layout)
    qo = torch.empty((E, 2, I, H // 2), dtype=torch.uint8, device="cuda")
    so = torch.empty((E, 2, max(npart, 16)), dtype=torch.uint8, device="cuda")
    ao = torch.empty((E, 2, 1), dtype=torch.float32, device="cuda")
    qz.split_fused_experts(qz.SplitTable([qz.SplitEntry(q=q[e], sf=sf[e], rows=2 * I, cols=H, cut=I,
                                                        sf_out=(so[e, 0], so[e, 1]), q_out=(qo[e, 0], qo[e, 1]),
                                                        amax=A[e], amax_out=(ao[e, 0], ao[e, 1]))
                                          for e in range(E)]),
                           qz.FMT_NVFP4, qz.AMAX_PER_TENSOR, layout, layout)
    # (b) one pass: gate and up entries share the expert's amax slot
    q1 = torch.empty_like(qo)
    s1 = torch.empty_like(so)
    A1 = torch.empty((E, 1), dtype=torch.float32, device="cuda")
    parts = [qz.Entry(W[e, p * I:(p + 1) * I], q1[e, p], s1[e, p], A1[e]) for e in range(E) for p in range(2)]
    qz.quantize_grouped_nvfp4(qz.ExpertTable(parts), qz.NVFP4_PER_TENSOR_COMPUTE, layout)
    torch.cuda.synchronize()
    assert torch.equal(A1, A)
    assert torch.equal(qo, q1) and torch.equal(so[..., :npart], s1[..., :npart])
    assert torch.equal(ao[:, 0], A) and torch.equal(ao[:, 1], A)
    Wh = synth.bf16_bits(W.cpu())
    for e in range(E):
        for p in range(2):
            rq, rsf, _ = oracle.quantize_nvfp4(np.ascontiguousarray(Wh[e, p * I:(p + 1) * I]), layout,
                                               oracle.NVFP4_PER_TENSOR_GIVEN, float(A[e].item()))
            assert_bytes_equal(qo[e, p].cpu().numpy(), rq.reshape(I, -1), f"expert {e} part {p} payload")
            assert_bytes_equal(so[e, p, :npart].cpu().numpy(), rsf, f"expert {e} part {p} scales")


def test_qwen3_30b_gate_up_layer():
    """A whole Qwen3-30B-A3B gate_up projection (128 experts, fused [1536, 2048],
    gate|up cut at 768) folded to NVFP4 swizzled and split: every expert's
    payload equals the rows of its folded payload; the oracle checks the
    scales and amaxes of three experts completely."""
    E, R, H, cut = 128, 1536, 2048, 768
    W = synth.normal_bf16((E * R, H), 0.02, seed=2, device="cuda").view(E, R, H)
    q = torch.empty((E, R, H // 2), dtype=torch.uint8, device="cuda")
    nsf = qz.sf_bytes(R, H, qz.FMT_NVFP4, qz.SF_SWIZZLED)
    sf = torch.empty((E, nsf), dtype=torch.uint8, device="cuda")
    A = torch.empty((E, 1), dtype=torch.float32, device="cuda")
    qz.quantize_grouped_nvfp4(qz.ExpertTable([qz.Entry(W[e], q[e], sf[e], A[e]) for e in range(E)]),
                              qz.NVFP4_PER_TENSOR_COMPUTE, qz.SF_SWIZZLED)
    npart = qz.sf_bytes(cut, H, qz.FMT_NVFP4, qz.SF_SWIZZLED)
    qo = torch.empty((E, 2, cut, H // 2), dtype=torch.uint8, device="cuda")
    so = torch.full((E, 2, npart), 0xA5, dtype=torch.uint8, device="cuda")
    ao = torch.empty((E, 2, 1), dtype=torch.float32, device="cuda")
    table = qz.SplitTable([qz.SplitEntry(q=q[e], sf=sf[e], rows=R, cols=H, cut=cut, sf_out=(so[e, 0], so[e, 1]),
                                         q_out=(qo[e, 0], qo[e, 1]), amax=A[e], amax_out=(ao[e, 0], ao[e, 1]))
                           for e in range(E)])
    qz.split_fused_experts(table, qz.FMT_NVFP4, qz.AMAX_PER_TENSOR, qz.SF_SWIZZLED, qz.SF_SWIZZLED)
    torch.cuda.synchronize()
    assert torch.equal(qo.view(E, R, H // 2), q)
    assert torch.equal(ao[:, 0], A) and torch.equal(ao[:, 1], A)
    for e in (0, 77, 127):
        ref = oracle.split_fused(oracle.NVFP4, q[e].cpu().numpy(), sf[e].cpu().numpy(), A[e].cpu().numpy(),
                                 oracle.AMAX_PER_TENSOR, H, cut, oracle.SWIZZLED, oracle.SWIZZLED)
        for p in range(2):
            assert_bytes_equal(so[e, p].cpu().numpy(), ref[p][1], f"expert {e} part {p} scales")
