"""GPU parity of the grouped MXFP8 kernel against the oracle: bit-exact
payload and scale bytes, both layouts, ragged tiles, strided rows, batch-size
and grid-shape invariance, per-expert independence (canaries), empty and
invalid table entries, stream order and CUDA-graph replay, and the
Qwen3-30B-A3B / Qwen3-235B-A22B expert shapes at full size (sampled experts)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import Guarded, assert_bytes_equal, guarded_entries, host_bits, oracle_threads

pytestmark = pytest.mark.gpu

qz = pytest.importorskip("nvfp4_quantization_moe_b200")
LAYOUTS = [qz.SF_LINEAR, qz.SF_SWIZZLED]


def run_mxfp8(xs, layout, **kw):
    entries, keep = guarded_entries(xs, qz.FMT_MXFP8, layout)
    table = qz.ExpertTable(entries)
    qz.quantize_grouped_mxfp8(table, layout, **kw)
    torch.cuda.synchronize()
    for q, sf, _ in keep:
        assert q.guards_intact() and sf.guards_intact(), "write outside an expert's buffers"
    return [(q.host().reshape(x.shape[0], -1) if x.shape[0] else q.host(), sf.host()) for (q, sf, _), x in zip(keep, xs)]


def check_against_oracle(xs_dev, layout, got, threads=None):
    hosts = [host_bits(x) for x in xs_dev]
    ref = oracle.quantize_grouped(hosts, oracle.MXFP8, layout, threads=threads or oracle_threads())
    for i, ((gq, gsf), (rq, rsf)) in enumerate(zip(got, ref)):
        assert_bytes_equal(gq, rq, f"expert {i} payload")
        assert_bytes_equal(gsf, rsf, f"expert {i} scales")


@pytest.mark.parametrize("layout", LAYOUTS)
def test_tiny_group(layout):
    xs = [x.cuda() for x in synth.tiny_group()]
    check_against_oracle(xs, layout, run_mxfp8(xs, layout))


SHAPES = [(1, 32), (3, 64), (127, 96), (128, 128), (129, 160), (200, 416), (257, 2048), (64, 7168)]


@pytest.mark.parametrize("layout", LAYOUTS)
def test_ragged_shapes_stress_values(layout):
    xs = [synth.blockwise_scaled(s, 32, seed=100 + i).cuda() for i, s in enumerate(SHAPES)]
    check_against_oracle(xs, layout, run_mxfp8(xs, layout))


@pytest.mark.parametrize("layout", LAYOUTS)
def test_every_bf16_pattern(layout):
    """All finite bf16 bit patterns, 32 per block, shuffled so that block
    amaxes span the whole exponent range."""
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    rng = np.random.default_rng(0)
    rng.shuffle(bits)
    n = bits.size // 256 * 256
    x = torch.from_numpy(bits[:n].view(np.int16).reshape(-1, 256).copy()).view(torch.bfloat16).cuda()
    check_against_oracle([x], layout, run_mxfp8([x], layout))


def test_random_bit_patterns_and_zero_blocks():
    x = synth.random_finite_bf16((96, 512), seed=5)
    x[3, :] = 0
    x[4, 32:64] = -0.0
    xs = [x.cuda()]
    check_against_oracle(xs, qz.SF_SWIZZLED, run_mxfp8(xs, qz.SF_SWIZZLED))


def test_strided_rows():
    """Row strides and offsets that keep rows 32-byte aligned (256-bit loads)
    and ones that only keep them 16-byte aligned (paired 128-bit loads)."""
    base = synth.normal_bf16((300, 2048 + 64), seed=9).cuda()
    odd = synth.normal_bf16((140, 2048 + 8), seed=10).cuda()
    xs = [base[:, :2048], base[:150, 64:64 + 1024], odd[:, :2048], odd[:, 8:8 + 1536]]
    got = run_mxfp8(xs, qz.SF_SWIZZLED)
    check_against_oracle([x.contiguous() for x in xs], qz.SF_SWIZZLED, got)


def test_batch_size_and_grid_invariance():
    xs = [synth.normal_bf16((192, 256), std=0.02, seed=40 + i).cuda() for i in range(17)]
    whole = run_mxfp8(xs, qz.SF_SWIZZLED)
    for batch in (1, 16):
        parts = []
        for s in range(0, 17, batch):
            parts += run_mxfp8(xs[s:s + batch], qz.SF_SWIZZLED)
        for (a, b), (c, d) in zip(whole, parts):
            assert np.array_equal(a, c) and np.array_equal(b, d)
    for ctas in (1, 148, 4 * 148):
        other = run_mxfp8(xs, qz.SF_SWIZZLED, max_ctas=ctas)
        for (a, b), (c, d) in zip(whole, other):
            assert np.array_equal(a, c) and np.array_equal(b, d)
    check_against_oracle(xs, qz.SF_SWIZZLED, whole)


@pytest.mark.parametrize("hint", [1, 1 << 26, 1 << 40])
def test_grid_sized_by_the_element_hint(hint):
    """The element-count hint only sizes the grid (one wave up to 16 waves of
    short CTAs, most of them idle on a small table): the bytes stay the
    oracle's."""
    xs = [synth.blockwise_scaled(s, 32, seed=60 + i, lo=-10, hi=10).cuda()
          for i, s in enumerate([(130, 256), (1, 64), (300, 96), (0, 32), (64, 512)])]
    entries, keep = guarded_entries(xs, qz.FMT_MXFP8, qz.SF_SWIZZLED)
    table = qz.ExpertTable(entries)
    opts = qz.binding._opts(None, 0, elems_hint=hint)
    st = qz.load().qz_quantize_grouped_mxfp8(ctypes.c_void_p(table.ptr), table.n, qz.SF_SWIZZLED,
                                             qz.binding._stream_ptr(None), opts)
    assert st == qz.QZ_OK
    torch.cuda.synchronize()
    for q, sf, _ in keep:
        assert q.guards_intact() and sf.guards_intact()
    got = [(q.host().reshape(x.shape[0], -1) if x.shape[0] else q.host(), sf.host()) for (q, sf, _), x in zip(keep, xs)]
    check_against_oracle(xs, qz.SF_SWIZZLED, got)


def test_requantize_one_expert_touches_nothing_else():
    xs = [synth.normal_bf16((130, 320), seed=60 + i).cuda() for i in range(4)]
    entries, keep = guarded_entries(xs, qz.FMT_MXFP8, qz.SF_SWIZZLED)
    qz.quantize_grouped_mxfp8(qz.ExpertTable(entries), qz.SF_SWIZZLED)
    torch.cuda.synchronize()
    before = [(q.raw.clone(), sf.raw.clone()) for q, sf, _ in keep]
    xs[2].mul_(3.0)
    qz.quantize_grouped_mxfp8(qz.ExpertTable([entries[2]]), qz.SF_SWIZZLED)
    torch.cuda.synchronize()
    for i, ((q, sf, _), (bq, bsf)) in enumerate(zip(keep, before)):
        same = torch.equal(q.raw, bq) and torch.equal(sf.raw, bsf)
        assert same == (i != 2)
        assert q.guards_intact() and sf.guards_intact()
    check_against_oracle([xs[2]], qz.SF_SWIZZLED, [(keep[2][0].host().reshape(130, -1), keep[2][1].host())])


def test_empty_and_invalid_entries_are_skipped():
    dev = torch.device("cuda")
    good = synth.normal_bf16((64, 256), seed=3).cuda()
    q = Guarded(64 * 256)
    sf = Guarded(qz.sf_bytes(64, 256, qz.FMT_MXFP8, qz.SF_SWIZZLED))
    bad_q = Guarded(64 * 256)
    bad_sf = Guarded(4096)
    odd = torch.empty(64 * 256 + 8, dtype=torch.bfloat16, device=dev)
    raw = [
        (good.data_ptr(), 0, 256, 256, 0, 0, 0),                                           # empty split
        (good.data_ptr(), 64, 256, 256, q.view.data_ptr(), sf.view.data_ptr(), 0),          # valid
        (good.data_ptr(), 64, 250, 256, bad_q.view.data_ptr(), bad_sf.view.data_ptr(), 0),  # cols % 32
        (odd.data_ptr() + 2, 64, 256, 256, bad_q.view.data_ptr(), bad_sf.view.data_ptr(), 0),  # x misaligned
        (good.data_ptr(), 64, 256, 256, 0, bad_sf.view.data_ptr(), 0),                     # q null
        (good.data_ptr(), 64, 256, 200, bad_q.view.data_ptr(), bad_sf.view.data_ptr(), 0),  # ld < cols
        (good.data_ptr(), 64, 256, 256, bad_q.view.data_ptr(), bad_sf.view.data_ptr() + 4, 0),  # sf misaligned
    ]
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    qz.quantize_grouped_mxfp8(qz.ExpertTable.from_raw(raw, dev), qz.SF_SWIZZLED, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == (qz.DERR_SHAPE | qz.DERR_ALIGN | qz.DERR_NULL)
    assert torch.all(bad_q.raw == 0xA5) and torch.all(bad_sf.raw == 0xA5)
    rq, rsf = oracle.quantize_mxfp8(host_bits(good), oracle.SWIZZLED)
    assert_bytes_equal(q.host(), rq.reshape(-1), "payload")
    assert_bytes_equal(sf.host(), rsf, "scales")


def test_stream_order_and_graph_replay():
    side = torch.cuda.Stream()
    xs = [torch.zeros((256, 512), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    src = [synth.normal_bf16((256, 512), seed=80 + i).cuda() for i in range(3)]
    entries, keep = guarded_entries(xs, qz.FMT_MXFP8, qz.SF_SWIZZLED)
    table = qz.ExpertTable(entries)
    torch.cuda.synchronize()
    with torch.cuda.stream(side):
        torch.cuda._sleep(2_000_000)          # the producer is slow ...
        for x, s in zip(xs, src):
            x.copy_(s)
        qz.quantize_grouped_mxfp8(table, qz.SF_SWIZZLED, stream=side)   # ... and ordered on its stream
    torch.cuda.synchronize()
    got = [(q.host().reshape(256, -1), sf.host()) for q, sf, _ in keep]
    check_against_oracle(src, qz.SF_SWIZZLED, got)
    # graph capture of the same call, replayed on new inputs
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        qz.quantize_grouped_mxfp8(table, qz.SF_SWIZZLED, stream=s)   # warm-up outside capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            qz.quantize_grouped_mxfp8(table, qz.SF_SWIZZLED, stream=s)
    for x in xs:
        x.mul_(-0.5)
    g.replay()
    torch.cuda.synchronize()
    got = [(q.host().reshape(256, -1), sf.host()) for q, sf, _ in keep]
    check_against_oracle([x for x in xs], qz.SF_SWIZZLED, got)


def test_qwen3_30b_layer_full_parity():
    """One layer of the Qwen3-30B-A3B refit at full size, in the bench's call
    shape (16 experts per call): the first gate_up call and the first down
    call compared completely with the oracle."""
    cfg = synth.QWEN3_30B
    gate_up = synth.expert_stack(16, cfg["gate_up"], cfg["std"], seed=cfg["seed"], device="cuda")
    down = synth.expert_stack(16, cfg["down"], cfg["std"], seed=cfg["seed"] + 1000, device="cuda")
    for stack in (gate_up, down):
        xs = list(stack.unbind(0))
        check_against_oracle(xs, qz.SF_SWIZZLED, run_mxfp8(xs, qz.SF_SWIZZLED))


def test_qwen3_235b_experts_sampled():
    """Qwen3-235B-A22B expert shapes at full size: a 128-expert gate_up call,
    with experts 0, 77 and 127 compared completely with the oracle and every
    scale byte of the others checked against the block invariant."""
    cfg = synth.QWEN3_235B
    stack = synth.expert_stack(128, cfg["gate_up"], cfg["std"], seed=cfg["seed"], device="cuda")
    xs = list(stack.unbind(0))
    entries = qz.alloc_outputs(xs, qz.FMT_MXFP8, qz.SF_SWIZZLED)
    qz.quantize_grouped_mxfp8(qz.ExpertTable(entries), qz.SF_SWIZZLED)
    torch.cuda.synchronize()
    rows, cols = cfg["gate_up"]
    nsf = qz.sf_bytes(rows, cols, qz.FMT_MXFP8, qz.SF_SWIZZLED)
    sample = [0, 77, 127]
    got = [(entries[i].q.cpu().numpy(), entries[i].sf[:nsf].cpu().numpy()) for i in sample]
    check_against_oracle([xs[i] for i in sample], qz.SF_SWIZZLED, got)
    # all experts: the scale of each block is the least exponent keeping the
    # block's amax <= 448 (checked on the GPU in torch, from the input alone)
    for i in range(0, 128, 9):
        x = xs[i].float().abs().view(rows, cols // 32, 32).amax(dim=2)
        sfl = entries[i].sf[:nsf].view(rows // 128, cols // 128, 32, 4, 4)  # [rt, ct, r%32, r/32, k]
        sfl = sfl.permute(0, 3, 2, 1, 4).reshape(rows, cols // 32).to(torch.int32) - 127
        e = sfl.double()
        amax = x.double()
        assert torch.all(amax <= 448.0 * torch.exp2(e))
        assert torch.all((amax > 224.0 * torch.exp2(e)) | (amax == 0))


def _blocks_with_every_amax(block: int) -> torch.Tensor:
    """One block per positive finite bf16 value v: [v, -0.7 v, 0.3 v, 0, ...]."""
    bits = np.arange(1, 0x7F80, dtype=np.uint32)
    bits = bits[: bits.size // 8 * 8]
    v = torch.from_numpy((bits << 16).view(np.float32).copy())
    x = torch.zeros(v.numel(), block, dtype=torch.float32)
    x[:, 0] = v
    x[:, 1] = -0.7 * v
    x[:, 2] = 0.3 * v
    return x.to(torch.bfloat16).reshape(-1, 8 * block)


@pytest.mark.parametrize("layout", LAYOUTS)
def test_every_bf16_value_as_block_amax(layout):
    x = _blocks_with_every_amax(32).cuda()
    check_against_oracle([x], layout, run_mxfp8([x], layout))


def test_back_to_back_calls_on_one_stream():
    """Programmatic dependent launch between the tile kernels of consecutive
    calls: a call that is not declared independent still sees stream order
    (two calls writing the same outputs leave the second call's bytes; a
    call after a torch kernel that writes its input sees the new input);
    calls declared independent on disjoint experts give every call's bytes;
    both also inside a captured CUDA graph."""
    shape = (384, 1024)
    a = synth.normal_bf16(shape, seed=1).cuda()
    b = synth.blockwise_scaled(shape, 32, seed=2, lo=-20, hi=20).cuda()
    (q, sf, _), = guarded_entries([a], qz.FMT_MXFP8, qz.SF_SWIZZLED)[1]
    ta = qz.ExpertTable([qz.Entry(a, q.view.view(shape), sf.view)])
    tb = qz.ExpertTable([qz.Entry(b, q.view.view(shape), sf.view)])
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for _ in range(20):                        # write-after-write on the same outputs, in stream order
            qz.quantize_grouped_mxfp8(ta, qz.SF_SWIZZLED, stream=s)
            qz.quantize_grouped_mxfp8(tb, qz.SF_SWIZZLED, stream=s)
    torch.cuda.synchronize()
    check_against_oracle([b], qz.SF_SWIZZLED, [(q.host().reshape(shape), sf.host())])
    c = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    tc = qz.ExpertTable([qz.Entry(c, q.view.view(shape), sf.view)])
    with torch.cuda.stream(s):
        qz.quantize_grouped_mxfp8(ta, qz.SF_SWIZZLED, stream=s)
        c.copy_(b).mul_(3.0)                       # a torch kernel writes the next call's input
        qz.quantize_grouped_mxfp8(tc, qz.SF_SWIZZLED, stream=s)
    torch.cuda.synchronize()
    check_against_oracle([c], qz.SF_SWIZZLED, [(q.host().reshape(shape), sf.host())])
    # independent calls on disjoint experts, MXFP8 and NVFP4 given, and as a graph
    xs = [synth.blockwise_scaled((200 + 17 * i, 512), 32, seed=30 + i, lo=-8, hi=8).cuda() for i in range(12)]
    mx, mkeep = guarded_entries(xs, qz.FMT_MXFP8, qz.SF_SWIZZLED)
    amax_in = [float(x.float().abs().max()) for x in xs]
    nv, nkeep = guarded_entries(xs, qz.FMT_NVFP4, qz.SF_LINEAR, qz.NVFP4_PER_TENSOR_GIVEN, amax_in)
    mtabs = [qz.ExpertTable([e]) for e in mx]
    ntabs = [qz.ExpertTable([e]) for e in nv]

    def burst():
        for mt, nt in zip(mtabs, ntabs):
            qz.quantize_grouped_mxfp8(mt, qz.SF_SWIZZLED, stream=s, independent=True)
            qz.quantize_grouped_nvfp4(nt, qz.NVFP4_PER_TENSOR_GIVEN, qz.SF_LINEAR, stream=s, independent=True)

    def verify():
        got = [(qq.host().reshape(x.shape[0], -1), ss.host()) for (qq, ss, _), x in zip(mkeep, xs)]
        check_against_oracle(xs, qz.SF_SWIZZLED, got)
        ref = oracle.quantize_grouped([host_bits(x) for x in xs], oracle.NVFP4, oracle.LINEAR,
                                      oracle.NVFP4_PER_TENSOR_GIVEN, amax_in, threads=oracle_threads())
        for (qq, ss, aa), x, (rq, rs, _) in zip(nkeep, xs, ref):
            assert qq.guards_intact() and ss.guards_intact()
            assert_bytes_equal(qq.host(), rq.reshape(-1), "NVFP4 payload")
            assert_bytes_equal(ss.host(), rs, "NVFP4 scales")

    with torch.cuda.stream(s):
        burst()
    torch.cuda.synchronize()
    verify()
    for qq, ss, _ in mkeep + nkeep:
        qq.view.fill_(0xA5)
        ss.view.fill_(0xA5)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            burst()
    g.replay()
    torch.cuda.synchronize()
    verify()
