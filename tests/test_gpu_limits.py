"""GPU parity at the documented limits of the C ABI: tables of QZ_MAX_EXPERTS
(4096) entries for every grouped entry point, the largest row stride
(QZ_MAX_LD elements), the largest hidden size of the fused norm
(QZ_MAX_HIDDEN) and the most splits of the decode merge (QZ_MAX_SPLITS), each
against the oracle, with canary-guarded outputs where the outputs are small."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import assert_bytes_equal, guarded_entries, host_bits, oracle_threads

pytestmark = pytest.mark.gpu

qz = pytest.importorskip("nvfp4_quantization_moe_b200")
LAYOUTS = [qz.SF_LINEAR, qz.SF_SWIZZLED]


def max_table(block, seed):
    """QZ_MAX_EXPERTS small experts: 1-3 rows, 2 or 4 blocks per row, the
    narrower ones read with a row stride wider than the row."""
    n = qz.MAX_EXPERTS
    rows = [1 + i % 3 for i in range(n)]
    base = synth.blockwise_scaled((sum(rows), 4 * block), block, seed=seed, lo=-8, hi=8).cuda()
    xs, off = [], 0
    for i, r in enumerate(rows):
        cols = 4 * block if i % 2 else 2 * block
        xs.append(base[off:off + r, :cols])
        off += r
    return xs


def run_and_check(xs, fmt, layout, mode=qz.NVFP4_PER_ROW, amax_in=None, workspace=None):
    entries, keep = guarded_entries(xs, fmt, layout, mode, amax_in)
    table = qz.ExpertTable(entries)
    if fmt == qz.FMT_MXFP8:
        qz.quantize_grouped_mxfp8(table, layout)
    else:
        qz.quantize_grouped_nvfp4(table, mode, layout, workspace=workspace)
    torch.cuda.synchronize()
    hosts = [host_bits(x) for x in xs]
    ref = oracle.quantize_grouped(hosts, oracle.MXFP8 if fmt == qz.FMT_MXFP8 else oracle.NVFP4, layout, mode,
                                  amax_in, threads=oracle_threads())
    for i, ((q, sf, a), r) in enumerate(zip(keep, ref)):
        assert q.guards_intact() and sf.guards_intact(), f"expert {i}: write outside its buffers"
        assert_bytes_equal(q.host(), r[0].reshape(-1), f"expert {i} payload")
        assert_bytes_equal(sf.host(), r[1], f"expert {i} scales")
        if fmt == qz.FMT_NVFP4 and mode != qz.NVFP4_PER_TENSOR_GIVEN:
            got = a.view.view(torch.float32).cpu().numpy()[: r[2].size]
            assert np.array_equal(got.view(np.uint32), r[2].view(np.uint32)), f"expert {i} amax"
    return keep


@pytest.mark.parametrize("layout", LAYOUTS)
def test_mxfp8_max_table(layout):
    run_and_check(max_table(32, 11), qz.FMT_MXFP8, layout)


@pytest.mark.parametrize("mode", [qz.NVFP4_PER_TENSOR_GIVEN, qz.NVFP4_PER_TENSOR_COMPUTE, qz.NVFP4_PER_ROW])
@pytest.mark.parametrize("layout", LAYOUTS)
def test_nvfp4_max_table(layout, mode):
    xs = max_table(16, 12)
    amax_in = [float(x.float().abs().max()) * 1.25 for x in xs] if mode == qz.NVFP4_PER_TENSOR_GIVEN else None
    run_and_check(xs, qz.FMT_NVFP4, layout, mode, amax_in)


def test_nvfp4_computed_amax_single_launch_max_table():
    xs = max_table(16, 13)
    ws = qz.alloc_workspace(qz.MAX_EXPERTS)
    run_and_check(xs, qz.FMT_NVFP4, qz.SF_SWIZZLED, qz.NVFP4_PER_TENSOR_COMPUTE, workspace=ws)


@pytest.mark.parametrize("fmt", [qz.FMT_MXFP8, qz.FMT_NVFP4])
def test_dequant_colwise_and_split_max_tables(fmt):
    block = 32 if fmt == qz.FMT_MXFP8 else 16
    n = qz.MAX_EXPERTS
    # dequantize: the quantized max table back to bf16
    xs = max_table(block, 14)
    mode = qz.NVFP4_PER_TENSOR_COMPUTE
    keep = run_and_check(xs, fmt, qz.SF_SWIZZLED, mode) if fmt == qz.FMT_NVFP4 else \
        run_and_check(xs, fmt, qz.SF_SWIZZLED)
    ys = [torch.empty_like(x) for x in xs]
    dq = []
    for (q, sf, a), y, x in zip(keep, ys, xs):
        dq.append(qz.DqEntry(q.view, sf.view, y, a.view.view(torch.float32) if a is not None else None))
    qz.dequantize_grouped(qz.DqTable(dq), fmt, False, qz.SF_SWIZZLED)
    torch.cuda.synchronize()
    for i in range(0, n, 97):
        q, sf, a = keep[i]
        rows, cols = xs[i].shape
        qh = q.host().reshape(rows, -1)
        ref = oracle.dequantize_mxfp8(qh, sf.host(), oracle.SWIZZLED) if fmt == qz.FMT_MXFP8 else \
            oracle.dequantize_nvfp4(qh, sf.host(), a.view.view(torch.float32).cpu().numpy()[:1], False,
                                    oracle.SWIZZLED)
        assert_bytes_equal(host_bits(ys[i]), ref, f"dequantized expert {i}")
    # column-wise: 4096 experts of [block, 8..24] (rows a multiple of the block)
    cx = [synth.normal_bf16((block, 8 + 8 * (i % 3)), 1.0, seed=5000 + i).cuda() for i in range(n)]
    amax = [float(x.float().abs().max()) for x in cx]
    centries, ckeep = [], []
    for x, A in zip(cx, amax):
        rows, cols = x.shape
        q = torch.empty(rows * cols // (2 if fmt == qz.FMT_NVFP4 else 1), dtype=torch.uint8, device="cuda")
        sf = torch.empty(max(qz.sf_bytes(cols, rows, fmt, qz.SF_LINEAR), 16), dtype=torch.uint8, device="cuda")
        a = torch.tensor([A], dtype=torch.float32, device="cuda") if fmt == qz.FMT_NVFP4 else None
        centries.append(qz.Entry(x, q, sf, a))
        ckeep.append((q, sf))
    qz.quantize_grouped_colwise(qz.ExpertTable(centries), fmt, qz.SF_LINEAR)
    torch.cuda.synchronize()
    for i in range(0, n, 89):
        xh = host_bits(cx[i])
        rows, cols = xh.shape
        if fmt == qz.FMT_MXFP8:
            rq, rsf = oracle.quantize_colwise(xh, oracle.MXFP8, oracle.LINEAR)
        else:
            rq, rsf, _ = oracle.quantize_colwise(xh, oracle.NVFP4, oracle.LINEAR, oracle.NVFP4_PER_TENSOR_GIVEN,
                                                 amax[i])
        assert_bytes_equal(ckeep[i][0].cpu().numpy(), rq.reshape(-1), f"column-wise expert {i} payload")
        assert_bytes_equal(ckeep[i][1].cpu().numpy()[: rsf.size], rsf, f"column-wise expert {i} scales")
    # fused gate|up split of the quantized max table: each expert cut after its first row
    kind = qz.AMAX_PER_TENSOR if fmt == qz.FMT_NVFP4 else qz.AMAX_NONE
    sentries, skeep = [], []
    for (q, sf, a), x in zip(keep, xs):
        rows, cols = x.shape
        rb = cols // 2 if fmt == qz.FMT_NVFP4 else cols
        parts = [(torch.empty(max(nr * rb, 16), dtype=torch.uint8, device="cuda"),
                  torch.empty(max(qz.sf_bytes(nr, cols, fmt, qz.SF_LINEAR), 16), dtype=torch.uint8, device="cuda"),
                  torch.empty(1, dtype=torch.float32, device="cuda")) for nr in (1, rows - 1)]
        sentries.append(qz.SplitEntry(q=q.view, sf=sf.view, rows=rows, cols=cols, cut=1,
                                      sf_out=(parts[0][1], parts[1][1]), q_out=(parts[0][0], parts[1][0]),
                                      amax=a.view.view(torch.float32) if a is not None else None,
                                      amax_out=(parts[0][2], parts[1][2]) if a is not None else (None, None)))
        skeep.append(parts)
    qz.split_fused_experts(qz.SplitTable(sentries), fmt, kind, qz.SF_SWIZZLED, qz.SF_LINEAR)
    torch.cuda.synchronize()
    for i in range(0, n, 101):
        q, sf, a = keep[i]
        rows, cols = xs[i].shape
        amax_h = a.view.view(torch.float32).cpu().numpy()[:1] if a is not None else None
        ref = oracle.split_fused(oracle.MXFP8 if fmt == qz.FMT_MXFP8 else oracle.NVFP4, q.host().reshape(rows, -1),
                                 sf.host(), amax_h, kind, cols, 1, oracle.SWIZZLED, oracle.LINEAR)
        for p, ((pq, psf, pa), (rq, rsf, ra)) in enumerate(zip(skeep[i], ref)):
            assert_bytes_equal(pq.cpu().numpy()[: rq.size], rq.reshape(-1), f"split expert {i} part {p} payload")
            assert_bytes_equal(psf.cpu().numpy()[: rsf.size], rsf, f"split expert {i} part {p} scales")
            if kind == qz.AMAX_PER_TENSOR:
                assert pa.item() == float(ra[0])


@pytest.mark.parametrize("fmt", [qz.FMT_MXFP8, qz.FMT_NVFP4])
def test_largest_row_stride(fmt):
    """Two rows QZ_MAX_LD elements apart (64 MB of address range)."""
    ld = qz.binding.MAX_LD if hasattr(qz.binding, "MAX_LD") else 1 << 24
    base = torch.zeros(ld + 64, dtype=torch.bfloat16, device="cuda")
    vals = synth.blockwise_scaled((2, 64), 16, seed=77, lo=-6, hi=6).cuda()
    base[:64] = vals[0]
    base[ld:ld + 64] = vals[1]
    x = base.as_strided((2, 64), (ld, 1))
    amax_in = [float(vals.float().abs().max())]
    mode = qz.NVFP4_PER_TENSOR_GIVEN
    entries, keep = guarded_entries([x], fmt, qz.SF_SWIZZLED, mode, amax_in)
    table = qz.ExpertTable(entries)
    if fmt == qz.FMT_MXFP8:
        qz.quantize_grouped_mxfp8(table, qz.SF_SWIZZLED)
        rq, rsf = oracle.quantize_mxfp8(host_bits(vals), oracle.SWIZZLED)
    else:
        qz.quantize_grouped_nvfp4(table, mode, qz.SF_SWIZZLED)
        rq, rsf, _ = oracle.quantize_nvfp4(host_bits(vals), oracle.SWIZZLED, mode, amax_in[0])
    torch.cuda.synchronize()
    q, sf, _ = keep[0]
    assert q.guards_intact() and sf.guards_intact()
    assert_bytes_equal(q.host(), rq.reshape(-1), "payload")
    assert_bytes_equal(sf.host(), rsf, "scales")


@pytest.mark.parametrize("fmt,layout", [(qz.FMT_MXFP8, qz.SF_SWIZZLED), (qz.FMT_NVFP4, qz.SF_LINEAR)])
def test_fused_norm_largest_hidden(fmt, layout):
    T, H = 3, qz.MAX_HIDDEN
    g = torch.Generator().manual_seed(9)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    r = torch.randn(T, H, generator=g).to(torch.bfloat16)
    gamma = (torch.rand(H, generator=g) + 0.5).to(torch.bfloat16)
    y_ref, h_ref = oracle.residual_rmsnorm(host_bits(x), host_bits(r), host_bits(gamma), 1e-6)
    yd = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    hd = torch.empty_like(yd)
    q = torch.empty((T, H if fmt == qz.FMT_MXFP8 else H // 2), dtype=torch.uint8, device="cuda")
    sf = torch.empty(qz.sf_bytes(T, H, fmt, layout), dtype=torch.uint8, device="cuda")
    A = torch.tensor([float(np.abs((y_ref.astype(np.uint32) << 16).view(np.float32)).max())], device="cuda")
    qz.rmsnorm_quantize(x.cuda(), r.cuda(), gamma.cuda(), 1e-6, yd, hd, fmt, q, sf, layout,
                        A if fmt == qz.FMT_NVFP4 else None)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(hd), h_ref)
    gy = host_bits(yd)
    assert np.abs(gy.astype(np.int32) - y_ref.astype(np.int32)).max() <= 1
    if fmt == qz.FMT_MXFP8:
        rq, rsf = oracle.quantize_mxfp8(gy, layout)
    else:
        rq, rsf, _ = oracle.quantize_nvfp4(gy, layout, oracle.NVFP4_PER_TENSOR_GIVEN, float(A.item()))
    assert_bytes_equal(q.cpu().numpy(), rq.reshape(q.shape), "payload")
    assert_bytes_equal(sf.cpu().numpy(), rsf, "scales")


def test_merge_most_splits_and_largest_hidden():
    for S, T, H in ((4096, 2, 128), (2, 3, qz.MAX_HIDDEN)):
        O, lse = synth.merge_partials(S, T, H, seed=S + H)
        y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
        q = torch.empty((T, H), dtype=torch.uint8, device="cuda")
        sf = torch.empty(qz.sf_bytes(T, H, qz.FMT_MXFP8, qz.SF_SWIZZLED), dtype=torch.uint8, device="cuda")
        qz.attention_merge_quantize(torch.from_numpy(O).cuda(), torch.from_numpy(lse).cuda(), y, q, sf)
        torch.cuda.synchronize()
        gy = host_bits(y)
        assert np.abs(gy.astype(np.int32) - oracle.attention_merge(O, lse).astype(np.int32)).max() <= 1
        rq, rsf = oracle.quantize_mxfp8(gy, oracle.SWIZZLED)
        assert_bytes_equal(q.cpu().numpy(), rq, f"payload S={S} H={H}")
        assert_bytes_equal(sf.cpu().numpy(), rsf, f"scales S={S} H={H}")
