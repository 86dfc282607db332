"""GPU parity of the grouped NVFP4 kernels against the oracle: per-tensor
(given and computed amax) and per-row modes, both layouts, ragged shapes,
stress values, the row-scaled split activation of 16384 x 4096 over 64
Dirichlet-sized experts (empty splits included) at full size, split ==
per-expert, per-expert independence and the Qwen3-235B-A22B shapes."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import Guarded, assert_bytes_equal, guarded_entries, host_bits, oracle_threads

pytestmark = pytest.mark.gpu

qz = pytest.importorskip("nvfp4_quantization_moe_b200")
LAYOUTS = [qz.SF_LINEAR, qz.SF_SWIZZLED]
MODES = {"given": qz.NVFP4_PER_TENSOR_GIVEN, "compute": qz.NVFP4_PER_TENSOR_COMPUTE, "row": qz.NVFP4_PER_ROW}


def run_nvfp4(xs, layout, mode, amax_in=None, **kw):
    entries, keep = guarded_entries(xs, qz.FMT_NVFP4, layout, mode, amax_in)
    qz.quantize_grouped_nvfp4(qz.ExpertTable(entries), mode, layout, **kw)
    torch.cuda.synchronize()
    out = []
    for (q, sf, a), x in zip(keep, xs):
        assert q.guards_intact() and sf.guards_intact() and a.guards_intact()
        rows = x.shape[0]
        out.append((q.host().reshape(rows, -1) if rows else q.host(), sf.host(),
                    a.view.view(torch.float32).cpu().numpy()))
    return out


def check(xs, layout, mode, got, amax_in=None):
    hosts = [host_bits(x) for x in xs]
    ref = oracle.quantize_grouped(hosts, oracle.NVFP4, layout, mode, amax_in, threads=oracle_threads())
    for i, ((gq, gsf, ga), (rq, rsf, ra)) in enumerate(zip(got, ref)):
        assert_bytes_equal(gq, rq, f"expert {i} payload")
        assert_bytes_equal(gsf, rsf, f"expert {i} scales")
        if mode != qz.NVFP4_PER_TENSOR_GIVEN and xs[i].shape[0]:
            n = ra.size
            assert np.array_equal(ga[:n].view(np.uint32), ra.view(np.uint32)), f"expert {i} amax"


SHAPES = [(1, 16), (5, 48), (127, 80), (129, 144), (200, 400), (300, 4096), (17, 7168)]


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("layout", LAYOUTS)
def test_shapes_modes_layouts(mode, layout):
    m = MODES[mode]
    xs = [synth.blockwise_scaled(s, 16, seed=200 + i, lo=-20, hi=8).cuda() for i, s in enumerate(SHAPES)]
    amax_in = None
    if m == qz.NVFP4_PER_TENSOR_GIVEN:
        amax_in = [float(x.float().abs().max()) * f for x, f in zip(xs, (1.0, 0.5, 2.0, 1.0, 0.9, 1.3, 1.0))]
    check(xs, layout, m, run_nvfp4(xs, layout, m, amax_in), amax_in)


@pytest.mark.parametrize("mode", list(MODES))
def test_every_bf16_pattern(mode):
    m = MODES[mode]
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    exp = (bits >> 7) & 0xFF
    bits = bits[(exp != 0xFF) & (exp > 30)].astype(np.uint16)   # row/tensor amax stays >= 2^-100
    rng = np.random.default_rng(1)
    rng.shuffle(bits)
    n = bits.size // 128 * 128
    x = torch.from_numpy(bits[:n].view(np.int16).reshape(-1, 128).copy()).view(torch.bfloat16).cuda()
    amax_in = [float(x.float().abs().max())] if m == qz.NVFP4_PER_TENSOR_GIVEN else None
    check([x], qz.SF_SWIZZLED, m, run_nvfp4([x], qz.SF_SWIZZLED, m, amax_in), amax_in)


def test_long_rows_take_the_two_pass_path():
    xs = [synth.split_activation(tokens=40, hidden=8192, seed=7).cuda(),
          synth.split_activation(tokens=9, hidden=16384 + 48, seed=8).cuda()]
    for layout in LAYOUTS:
        check(xs, layout, qz.NVFP4_PER_ROW, run_nvfp4(xs, layout, qz.NVFP4_PER_ROW))


def split_entries(x, counts, layout):
    """Per-expert views of one concatenated activation and per-expert outputs
    (payload and row amax contiguous across experts, SF regions separate)."""
    T, K = x.shape
    q_all = torch.empty((T, K // 2), dtype=torch.uint8, device=x.device)
    a_all = torch.empty(T, dtype=torch.float32, device=x.device)
    entries, sfs = [], []
    off = 0
    for c in counts:
        c = int(c)
        sf = Guarded(qz.sf_bytes(c, K, qz.FMT_NVFP4, layout))
        entries.append(qz.Entry(x[off:off + c], q_all[off:off + c], sf.view, a_all[off:off + c]))
        sfs.append(sf)
        off += c
    return entries, sfs, q_all, a_all


@pytest.mark.parametrize("force_empty", [(), (0, 5, 63)])
def test_split_activation_full_size(force_empty):
    """The row-scaled NVFP4 workload at full size: [16384, 4096], 1% outliers
    x20, rows over 64 experts by multinomial(Dirichlet(0.3)), swizzled SF."""
    cfg = synth.SPLIT_ACT
    x = synth.split_activation(device="cuda")
    counts = synth.dirichlet_splits(force_empty=force_empty)
    entries, sfs, q_all, a_all = split_entries(x, counts, qz.SF_SWIZZLED)
    qz.quantize_grouped_nvfp4(qz.ExpertTable(entries), qz.NVFP4_PER_ROW, qz.SF_SWIZZLED)
    torch.cuda.synchronize()
    xh = host_bits(x)
    hosts, off = [], 0
    for c in counts:
        hosts.append(xh[off:off + c])
        off += c
    ref = oracle.quantize_grouped(hosts, oracle.NVFP4, oracle.SWIZZLED, oracle.NVFP4_PER_ROW,
                                  threads=oracle_threads())
    qa = q_all.cpu().numpy()
    aa = a_all.cpu().numpy()
    off = 0
    for i, (c, (rq, rsf, ra)) in enumerate(zip(counts, ref)):
        assert_bytes_equal(qa[off:off + c], rq, f"expert {i} payload")
        assert_bytes_equal(sfs[i].host(), rsf, f"expert {i} scales")
        assert sfs[i].guards_intact()
        assert np.array_equal(aa[off:off + c].view(np.uint32), ra.view(np.uint32))
        off += c
    assert any(c == 0 for c in counts) or not force_empty


def test_split_equals_concatenated_linear():
    """Quantizing the whole activation as one expert (linear SF) gives the same
    payload, amax and scale rows as the per-expert split."""
    x = synth.split_activation(tokens=3000, hidden=1024, seed=11).cuda()
    counts = synth.dirichlet_splits(tokens=3000, experts=16, seed=11, force_empty=(2,))
    entries, sfs, q_all, a_all = split_entries(x, counts, qz.SF_LINEAR)
    qz.quantize_grouped_nvfp4(qz.ExpertTable(entries), qz.NVFP4_PER_ROW, qz.SF_LINEAR)
    whole = run_nvfp4([x], qz.SF_LINEAR, qz.NVFP4_PER_ROW)[0]
    torch.cuda.synchronize()
    assert np.array_equal(q_all.cpu().numpy(), whole[0])
    assert np.array_equal(a_all.cpu().numpy().view(np.uint32), whole[2].view(np.uint32))
    lin = np.concatenate([s.host() for s in sfs])
    assert np.array_equal(lin, whole[1])


def test_requantize_one_split_expert():
    x = synth.split_activation(tokens=1000, hidden=512, seed=12).cuda()
    counts = synth.dirichlet_splits(tokens=1000, experts=6, seed=12)
    entries, sfs, q_all, a_all = split_entries(x, counts, qz.SF_SWIZZLED)
    qz.quantize_grouped_nvfp4(qz.ExpertTable(entries), qz.NVFP4_PER_ROW, qz.SF_SWIZZLED)
    torch.cuda.synchronize()
    snap = [s.raw.clone() for s in sfs]
    qsnap, asnap = q_all.clone(), a_all.clone()
    e = int(np.argmax(counts))
    off = int(np.sum(counts[:e]))
    c = int(counts[e])
    x[off:off + c] = synth.split_activation(tokens=c, hidden=512, seed=99).cuda()
    qz.quantize_grouped_nvfp4(qz.ExpertTable([entries[e]]), qz.NVFP4_PER_ROW, qz.SF_SWIZZLED)
    torch.cuda.synchronize()
    for i, s in enumerate(sfs):
        assert torch.equal(s.raw, snap[i]) == (i != e)
        assert s.guards_intact()
    rows = torch.ones(1000, dtype=torch.bool, device="cuda")
    rows[off:off + c] = False
    assert torch.equal(q_all[rows], qsnap[rows]) and torch.equal(a_all[rows], asnap[rows])
    got = [(q_all[off:off + c].cpu().numpy(), sfs[e].host(), a_all[off:off + c].cpu().numpy())]
    check([x[off:off + c]], qz.SF_SWIZZLED, qz.NVFP4_PER_ROW, got)


def test_grid_invariance_compute_mode():
    xs = [synth.normal_bf16((300, 640), std=0.02, seed=300 + i).cuda() for i in range(5)]
    base = run_nvfp4(xs, qz.SF_SWIZZLED, qz.NVFP4_PER_TENSOR_COMPUTE)
    for ctas in (1, 37, 148):
        other = run_nvfp4(xs, qz.SF_SWIZZLED, qz.NVFP4_PER_TENSOR_COMPUTE, max_ctas=ctas)
        for a, b in zip(base, other):
            assert all(np.array_equal(u, v) for u, v in zip(a, b))


@pytest.mark.parametrize("layout", LAYOUTS)
def test_per_row_grid_sizes_and_a_large_table(layout):
    """Per-row mode on rows staged through shared memory: a single CTA (the
    stage ring wraps many times), a few CTAs, the default grid, and a table
    of 1100 small experts (a prefix table past the small-table launch kind),
    each against the oracle."""
    shapes = [(1, 16), (37, 2064), (129, 4096), (64, 2048), (3, 6000), (200, 96), (0, 64)]
    xs = [synth.blockwise_scaled(s, 16, seed=400 + i, lo=-12, hi=12).cuda() for i, s in enumerate(shapes)]
    for ctas in (1, 3, 0):
        check(xs, layout, qz.NVFP4_PER_ROW, run_nvfp4(xs, layout, qz.NVFP4_PER_ROW, max_ctas=ctas))
    many = [synth.blockwise_scaled((1 + i % 3, 48), 16, seed=900 + i, lo=-8, hi=8).cuda() for i in range(1100)]
    check(many, layout, qz.NVFP4_PER_ROW, run_nvfp4(many, layout, qz.NVFP4_PER_ROW))


def test_qwen3_235b_sampled_both_projections():
    cfg = synth.QWEN3_235B
    for shape, seed in ((cfg["gate_up"], cfg["seed"]), (cfg["down"], cfg["seed"] + 1000)):
        stack = synth.expert_stack(128, shape, cfg["std"], seed=seed, device="cuda")
        xs = list(stack.unbind(0))
        entries = qz.alloc_outputs(xs, qz.FMT_NVFP4, qz.SF_SWIZZLED, qz.NVFP4_PER_TENSOR_COMPUTE)
        qz.quantize_grouped_nvfp4(qz.ExpertTable(entries), qz.NVFP4_PER_TENSOR_COMPUTE, qz.SF_SWIZZLED)
        torch.cuda.synchronize()
        nsf = qz.sf_bytes(shape[0], shape[1], qz.FMT_NVFP4, qz.SF_SWIZZLED)
        amax_all = torch.stack([e.amax[0] for e in entries])
        ref_amax = stack.float().abs().amax(dim=(1, 2))
        assert torch.equal(amax_all, ref_amax)
        sample = [0, 64, 127]
        got = [(entries[i].q.cpu().numpy(), entries[i].sf[:nsf].cpu().numpy(), entries[i].amax.cpu().numpy())
               for i in sample]
        check([xs[i] for i in sample], qz.SF_SWIZZLED, qz.NVFP4_PER_TENSOR_COMPUTE, got)
        del stack, xs, entries
        torch.cuda.empty_cache()


def _blocks_with_every_amax(block: int) -> torch.Tensor:
    bits = np.arange(1, 0x7F80, dtype=np.uint32)
    bits = bits[: bits.size // 8 * 8]
    v = torch.from_numpy((bits << 16).view(np.float32).copy())
    x = torch.zeros(v.numel(), block, dtype=torch.float32)
    x[:, 0] = v
    x[:, 1] = -0.7 * v
    x[:, 2] = 0.3 * v
    x[:, 3] = 0.55 * v
    return x.to(torch.bfloat16)


def test_every_bf16_value_as_block_amax_per_row():
    """Rows of one block: the row amax, the block amax and hence S and the
    block scale take every bf16 magnitude."""
    x = _blocks_with_every_amax(16)
    x = x[x.float().abs().amax(dim=1) >= 2.0 ** -100].cuda()   # the contract's smallest amax
    check([x], qz.SF_SWIZZLED, qz.NVFP4_PER_ROW, run_nvfp4([x], qz.SF_SWIZZLED, qz.NVFP4_PER_ROW))


@pytest.mark.parametrize("A", [2688.0, 1.0, 3.0e4])
def test_every_bf16_value_as_block_amax_given_scale(A):
    """One tensor of blocks with every bf16 magnitude under a fixed encode
    scale: the block scales span every e4m3 code, zero included."""
    x = _blocks_with_every_amax(16).reshape(-1, 128)
    x = x[x.float().abs().amax(dim=1) <= A].cuda()    # the given amax bounds the tensor
    check([x], qz.SF_LINEAR, qz.NVFP4_PER_TENSOR_GIVEN, run_nvfp4([x], qz.SF_LINEAR, qz.NVFP4_PER_TENSOR_GIVEN, [A]), [A])


@pytest.mark.parametrize("mode", list(MODES))
def test_strided_rows_all_modes(mode):
    m = MODES[mode]
    base = synth.normal_bf16((260, 1024 + 64), seed=21).cuda()
    odd = synth.normal_bf16((133, 1024 + 8), seed=22).cuda()
    xs = [base[:, :1024], odd[:, :1024], odd[:, 8:8 + 512]]
    amax_in = [float(x.float().abs().max()) for x in xs] if m == qz.NVFP4_PER_TENSOR_GIVEN else None
    got = run_nvfp4(xs, qz.SF_SWIZZLED, m, amax_in)
    check([x.contiguous() for x in xs], qz.SF_SWIZZLED, m, got, amax_in)


def run_compute_l2(xs, layout, **kw):
    """Computed per-tensor amax through the single cooperative launch."""
    entries, keep = guarded_entries(xs, qz.FMT_NVFP4, layout, qz.NVFP4_PER_TENSOR_COMPUTE)
    ws = qz.alloc_workspace(len(xs))
    ws.fill_(0xFF)                       # the call zeroes what it needs
    qz.quantize_grouped_nvfp4(qz.ExpertTable(entries), qz.NVFP4_PER_TENSOR_COMPUTE, layout, workspace=ws, **kw)
    torch.cuda.synchronize()
    out = []
    for (q, sf, a), x in zip(keep, xs):
        assert q.guards_intact() and sf.guards_intact() and a.guards_intact()
        rows = x.shape[0]
        out.append((q.host().reshape(rows, -1) if rows else q.host(), sf.host(),
                    a.view.view(torch.float32).cpu().numpy()))
    return out


@pytest.mark.parametrize("layout", LAYOUTS)
def test_compute_l2_path_parity(layout):
    xs = [synth.blockwise_scaled(s, 16, seed=400 + i, lo=-20, hi=8).cuda() for i, s in enumerate(SHAPES)]
    xs.insert(2, torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda"))      # an empty expert
    check(xs, layout, qz.NVFP4_PER_TENSOR_COMPUTE, run_compute_l2(xs, layout))


def test_compute_l2_many_chunks_and_grid_invariance():
    """3072 tiles -> three ~1024-tile chunks; one CTA, a few, and a full wave
    give the same bytes (a single CTA exercises every wait in order)."""
    xs = [synth.normal_bf16((1024, 1024), std=0.02, seed=500 + i).cuda() for i in range(48)]
    xs[7].zero_()
    base = run_compute_l2(xs, qz.SF_SWIZZLED)
    for ctas in (1, 37):
        other = run_compute_l2(xs, qz.SF_SWIZZLED, max_ctas=ctas)
        for a, b in zip(base, other):
            assert all(np.array_equal(u, v) for u, v in zip(a, b))
    sample = [0, 7, 23, 47]
    check([xs[i] for i in sample], qz.SF_SWIZZLED, qz.NVFP4_PER_TENSOR_COMPUTE, [base[i] for i in sample])
    # and the same as the three-launch path
    three = run_nvfp4(xs, qz.SF_SWIZZLED, qz.NVFP4_PER_TENSOR_COMPUTE)
    for a, b in zip(base, three):
        assert all(np.array_equal(u, v) for u, v in zip(a, b))


def test_compute_l2_workspace_too_small_is_rejected():
    xs = [synth.normal_bf16((64, 64), seed=1).cuda()]
    entries, keep = guarded_entries(xs, qz.FMT_NVFP4, qz.SF_SWIZZLED, qz.NVFP4_PER_TENSOR_COMPUTE)
    ws = torch.zeros(qz.workspace_bytes(1) - 4, dtype=torch.uint8, device="cuda")
    with pytest.raises(qz.QzError):
        qz.quantize_grouped_nvfp4(qz.ExpertTable(entries), qz.NVFP4_PER_TENSOR_COMPUTE, qz.SF_SWIZZLED, workspace=ws)
    assert torch.all(keep[0][0].raw == 0xA5)


@pytest.mark.parametrize("layout", LAYOUTS)
def test_compute_l2_wait_runs_out(layout):
    """The failure path of the single-launch pipeline, with no GPU fault: the
    amax warps withhold the counts that release the quantize warps, so every
    wait runs out after the 0.2 ms limit.  The launch must end on its own
    with QZ_DERR_TIMEOUT in the error word and no output byte written; the
    context stays usable and the next call on the same buffers is exact."""
    xs = [synth.normal_bf16((300, 1024), std=0.02, seed=700 + i).cuda() for i in range(24)]
    entries, keep = guarded_entries(xs, qz.FMT_NVFP4, layout, qz.NVFP4_PER_TENSOR_COMPUTE)
    for (_, _, a) in keep:
        a.view.fill_(0xA5)
    table = qz.ExpertTable(entries)
    ws = qz.alloc_workspace(len(xs))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    qz.quantize_grouped_nvfp4(table, qz.NVFP4_PER_TENSOR_COMPUTE, layout, err=err, workspace=ws,
                              wait_limit_ns=200_000, test_flags=qz.TEST_WITHHOLD_ARRIVALS)
    ev1.record()
    torch.cuda.synchronize()
    assert int(err.item()) & qz.DERR_TIMEOUT
    assert ev0.elapsed_time(ev1) < 1000.0, "the launch must end soon after its waits run out"
    for q, sf, a in keep:
        assert torch.all(q.raw == 0xA5) and torch.all(sf.raw == 0xA5) and torch.all(a.raw == 0xA5)
    # the same buffers, a normal call: exact against the oracle
    err.zero_()
    qz.quantize_grouped_nvfp4(table, qz.NVFP4_PER_TENSOR_COMPUTE, layout, err=err, workspace=ws)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = [(q.host().reshape(x.shape[0], -1), sf.host(), a.view.view(torch.float32).cpu().numpy())
           for (q, sf, a), x in zip(keep, xs)]
    check(xs, layout, qz.NVFP4_PER_TENSOR_COMPUTE, got)


def test_compute_l2_large_experts_one_per_chunk():
    """Experts larger than a chunk's minimum (each its own chunk) next to
    small ones that share a chunk, and a call smaller than one chunk."""
    shapes = [(3072, 512), (16, 64), (5, 4096), (1100, 1024), (1, 16), (2048, 2048)]
    xs = [synth.blockwise_scaled(s, 16, seed=800 + i, lo=-6, hi=6).cuda() for i, s in enumerate(shapes)]
    for layout in LAYOUTS:
        check(xs, layout, qz.NVFP4_PER_TENSOR_COMPUTE, run_compute_l2(xs, layout))
        check(xs[1:3], layout, qz.NVFP4_PER_TENSOR_COMPUTE, run_compute_l2(xs[1:3], layout))


def _order_cases():
    from golden_io import rows
    return rows("nvfp4_rounding_order.txt")


@pytest.mark.parametrize("path", ["compute", "compute_l2", "row", "given"])
def test_rounding_order_golden_on_gpu(path):
    """The hand-worked cases that fix the order of the binary32 roundings of
    the two-level scale (encode scale, block scale, element multiplier) give
    the golden bytes on every NVFP4 path of the kernels."""
    for case in _order_cases():
        elems = np.zeros((1, 32), dtype=np.uint16)
        elems[0, 0], elems[0, 16], elems[0, 17] = (int(v, 16) for v in case[1:4])
        x = torch.from_numpy(elems.view(np.int16).copy()).view(torch.bfloat16).cuda()
        for layout in LAYOUTS:
            mode = {"compute": qz.NVFP4_PER_TENSOR_COMPUTE, "compute_l2": qz.NVFP4_PER_TENSOR_COMPUTE,
                    "row": qz.NVFP4_PER_ROW, "given": qz.NVFP4_PER_TENSOR_GIVEN}[path]
            amax_in = [float.fromhex(case[4])] if path == "given" else None
            ws = qz.alloc_workspace(1, "cuda") if path == "compute_l2" else None
            (gq, gsf, ga), = run_nvfp4([x], layout, mode, amax_in, workspace=ws)
            lin = gsf if layout == qz.SF_LINEAR else oracle.unswizzle(gsf, 1, 2)
            assert float(ga[0]).hex() == case[4], case[0]
            assert list(lin[:2]) == [int(case[5], 16), int(case[6], 16)], (case[0], path, layout)
            assert gq[0].tobytes().hex().upper() == case[7], (case[0], path, layout)
