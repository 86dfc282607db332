"""GPU parity of the AllReduce epilogue (qz_allreduce_rmsnorm_quantize).

Every GPU call here has one GPU, so the ranks are emulated the way a single
kernel over all ranks' data allows: the n rank inputs (and, for the
reduce-scatter + all-gather form, the n ranks' destination buffers) are
separate buffers on the one device, read and written through the same plain
pointers a peer mapping would give.  Nothing waits on another kernel.

* the rank sum: bit-exact with the oracle (a zero residual makes
  residual_out equal to the reduced x), on inputs whose binary32 accumulation
  is inexact, so the rank order decides;
* residual_out bit-exact, norm_out within 1 bf16 ulp of the oracle, quantized
  bytes exact wherever norm_out agrees with the oracle's;
* everything bit-exact with the single-input fused kernel run on the oracle's
  rank sum: the AllReduce prologue changes nothing after x;
* slices: every rank's slice written to every rank's destinations gives, in
  each destination, the one-shot result byte for byte (swizzled padding
  included), inside canary guards;
* the bench's launch shape (8 ranks, T = 4096, H = 7168) on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import Guarded, assert_bytes_equal, bf16_ulp_diff, host_bits

pytestmark = pytest.mark.gpu

qz = pytest.importorskip("nvfp4_quantization_moe_b200")

H = synth.FUSED_NORM["hidden"]
EPS = synth.FUSED_NORM["eps"]


class Dest:
    """One destination's buffers, payload and scales canary-guarded."""

    def __init__(self, T, H, fmt, layout, with_residual=True):
        self.T, self.fmt = T, fmt
        self.qcols = H if fmt == qz.FMT_MXFP8 else H // 2
        self.y = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
        self.h = torch.empty(T, H, dtype=torch.bfloat16, device="cuda") if with_residual else None
        self.q = Guarded(T * self.qcols)
        self.sf = Guarded(qz.sf_bytes(T, H, fmt, layout))

    def entry(self):
        return (self.y, self.h, self.q.view, self.sf.view)

    def result(self):
        torch.cuda.synchronize()
        assert self.q.guards_intact() and self.sf.guards_intact()
        return (host_bits(self.y), None if self.h is None else host_bits(self.h),
                self.q.host().reshape(self.T, self.qcols), self.sf.host())


def amax_tensor(A):
    return None if A is None else torch.tensor([A], dtype=torch.float32, device="cuda")


def run(xs, r, g, fmt, layout, A=None, rows=None, dests=None, with_residual=True):
    T = r.shape[0]
    if dests is None:
        dests = [Dest(T, H, fmt, layout, with_residual)]
    qz.allreduce_rmsnorm_quantize(xs, r, g, EPS, [d.entry() for d in dests], fmt, layout, T, H, rows=rows,
                                  global_amax=amax_tensor(A))
    return dests


def nvfp4_amax(xs_bits, rb, gb, fmt):
    if fmt != qz.FMT_NVFP4:
        return None
    y, _ = oracle.residual_rmsnorm(oracle.rank_sum(xs_bits), rb, gb, EPS)
    return float(np.abs((y.astype(np.uint32) << 16).view(np.float32)).max())


def spread_partials(n, T, seed):
    """Rank inputs with exponents spread over 2^-40 .. 2^40 per element, a few
    negative zeros and subnormals: binary32 accumulation is inexact here."""
    g = torch.Generator().manual_seed(seed)
    xs = []
    for _ in range(n):
        v = torch.randn(T, H, generator=g) * torch.exp2(torch.randint(-40, 41, (T, H), generator=g).float())
        v = v.to(torch.bfloat16)
        v[0, :16] = -0.0
        v[1 % T, 16:32] = 2.0 ** -133 * torch.randint(1, 100, (16,), generator=g).float()
        xs.append(v)
    return xs


@pytest.mark.parametrize("n", [2, 3, 8])
def test_rank_sum_bit_exact(n):
    T = 37
    xs = spread_partials(n, T, seed=40 + n)
    r = torch.zeros(T, H, dtype=torch.bfloat16)
    g = torch.ones(H, dtype=torch.bfloat16)
    want = oracle.rank_sum([host_bits(x) for x in xs])
    want = np.where(want == 0x8000, 0, want).astype(np.uint16)     # x + (+0): -0 becomes +0
    d = run([x.cuda() for x in xs], r.cuda(), g.cuda(), qz.FMT_MXFP8, qz.SF_LINEAR)[0]
    _, h, _, _ = d.result()
    assert_bytes_equal(h, want, f"rank sum of {n} ranks")
    if n >= 3:   # the rank order decides on these inputs: the reversed order differs somewhere
        rev = oracle.rank_sum([host_bits(x) for x in xs[::-1]])
        assert not np.array_equal(rev, oracle.rank_sum([host_bits(x) for x in xs]))


CASES = [(2, 1, qz.FMT_MXFP8, qz.SF_SWIZZLED), (3, 77, qz.FMT_NVFP4, qz.SF_LINEAR),
         (8, 130, qz.FMT_MXFP8, qz.SF_SWIZZLED), (4, 300, qz.FMT_NVFP4, qz.SF_SWIZZLED),
         (5, 64, qz.FMT_MXFP8, qz.SF_LINEAR), (1, 3, qz.FMT_NVFP4, qz.SF_LINEAR)]


@pytest.mark.parametrize("n,T,fmt,layout", CASES)
def test_parity(n, T, fmt, layout):
    xs, r, g = synth.rank_partials(n, T, seed=50 + T)
    xb, rb, gb = [host_bits(x) for x in xs], host_bits(r), host_bits(g)
    A = nvfp4_amax(xb, rb, gb, fmt)
    y_ref, h_ref, q_ref, sf_ref = oracle.allreduce_rmsnorm_quantize(xb, rb, gb, EPS, fmt, layout, A)
    xd, rd, gd = [x.cuda() for x in xs], r.cuda(), g.cuda()
    y, h, q, sf = run(xd, rd, gd, fmt, layout, A)[0].result()
    assert_bytes_equal(h, h_ref, "residual_out")
    d = bf16_ulp_diff(y, y_ref)
    assert d.max() <= 1, f"norm_out off by {d.max()} ulp"
    assert (d > 0).mean() < 1e-3, f"{(d > 0).sum()} elements off by one ulp"
    blk = 32 if fmt == qz.FMT_MXFP8 else 16
    same = (d.reshape(T, H // blk, blk) == 0).all(axis=2)
    qg, qr = q.reshape(T, H // blk, -1), q_ref.reshape(T, H // blk, -1)
    assert np.array_equal(qg[same], qr[same])
    lin_g = sf if layout == qz.SF_LINEAR else oracle.unswizzle(sf, T, H // blk)
    lin_r = sf_ref if layout == qz.SF_LINEAR else oracle.unswizzle(sf_ref, T, H // blk)
    assert np.array_equal(lin_g.reshape(T, -1)[same], lin_r.reshape(T, -1)[same])
    if layout == qz.SF_SWIZZLED:
        lib = oracle.load()
        live = np.zeros(sf.size, dtype=bool)
        for rr in range(T):
            for k in range(0, H // blk, 4):
                live[lib.qzo_sf_offset_swizzled(rr, k, H // blk):][:4] = True
        assert not np.any(sf[~live]), "padded rows of the swizzled layout must be zero"
    # the single-input fused kernel on the oracle's rank sum: identical bytes
    x_sum = torch.from_numpy(oracle.rank_sum(xb).view(np.int16)).view(torch.bfloat16).cuda()
    yf = torch.empty_like(rd)
    hf = torch.empty_like(rd)
    qf = Guarded(q.size)
    sff = Guarded(sf.size)
    qz.rmsnorm_quantize(x_sum, rd, gd, EPS, yf, hf, fmt, qf.view, sff.view, layout, amax_tensor(A))
    torch.cuda.synchronize()
    assert_bytes_equal(y, host_bits(yf), "norm_out vs the fused kernel on the rank sum")
    assert_bytes_equal(h, host_bits(hf), "residual_out vs the fused kernel")
    assert_bytes_equal(q.reshape(-1), qf.host(), "payload vs the fused kernel")
    assert_bytes_equal(sf, sff.host(), "scales vs the fused kernel")


@pytest.mark.parametrize("n,T,fmt,layout", [(4, 300, qz.FMT_MXFP8, qz.SF_SWIZZLED),
                                            (3, 200, qz.FMT_NVFP4, qz.SF_LINEAR),
                                            (2, 128, qz.FMT_NVFP4, qz.SF_SWIZZLED)])
def test_slices_to_every_destination(n, T, fmt, layout):
    """The reduce-scatter + all-gather form: rank k computes rows
    [k T / n, (k+1) T / n) and writes them to all n ranks' destinations."""
    xs, r, g = synth.rank_partials(n, T, seed=60 + n)
    xd, rd, gd = [x.cuda() for x in xs], r.cuda(), g.cuda()
    A = nvfp4_amax([host_bits(x) for x in xs], host_bits(r), host_bits(g), fmt)
    one = run(xd, rd, gd, fmt, layout, A)[0].result()
    dests = [Dest(T, H, fmt, layout) for _ in range(n)]
    bounds = [k * T // n for k in range(n + 1)]
    for k in range(n):
        run(xd, rd, gd, fmt, layout, A, rows=(bounds[k], bounds[k + 1]), dests=dests)
    for k, d in enumerate(dests):
        for a, b, what in zip(d.result(), one, ("norm_out", "residual_out", "payload", "scales")):
            assert_bytes_equal(a, b, f"destination {k} {what}")


def test_empty_slice_at_the_end_writes_only_the_padding():
    T, fmt, layout = 100, qz.FMT_MXFP8, qz.SF_SWIZZLED
    xs, r, g = synth.rank_partials(2, T, seed=70)
    d = Dest(T, H, fmt, layout)
    run([x.cuda() for x in xs], r.cuda(), g.cuda(), fmt, layout, rows=(T, T), dests=[d])
    _, _, q, sf = d.result()
    assert np.all(q == 0xA5), "no payload row is written"
    kv = H // 32
    lib = oracle.load()
    live = np.zeros(sf.size, dtype=bool)
    for rr in range(T):
        for k in range(0, kv, 4):
            live[lib.qzo_sf_offset_swizzled(rr, k, kv):][:4] = True
    assert np.all(sf[live] == 0xA5), "live scale bytes are left alone"
    assert not np.any(sf[~live]), "the invented rows are zeroed"


def test_bench_shape_sampled_rows():
    """8 ranks, T = 4096, H = 7168 (the bench's launch), MXFP8 swizzled: 48
    sampled rows against the oracle; the payload and scales of all rows equal
    the grouped kernel's quantization of the epilogue's own norm_out."""
    n, T = 8, 4096
    xs, r, g = synth.rank_partials(n, T, device="cuda")
    d = run(xs, r, g, qz.FMT_MXFP8, qz.SF_SWIZZLED)[0]
    y, h, q, sf = d.result()
    rows = np.random.default_rng(8).choice(T, 48, replace=False)
    xb = [host_bits(x[rows]) for x in xs]
    y_ref, h_ref = oracle.residual_rmsnorm(oracle.rank_sum(xb), host_bits(r[rows]), host_bits(g), EPS)
    assert_bytes_equal(h[rows], h_ref, "residual_out")
    assert bf16_ulp_diff(y[rows], y_ref).max() <= 1
    e = qz.quantize_experts([d.y], qz.FMT_MXFP8, qz.SF_SWIZZLED, qz.NVFP4_PER_TENSOR_GIVEN, None)[0]
    torch.cuda.synchronize()
    assert_bytes_equal(q.reshape(-1), e.q.cpu().numpy().reshape(-1), "payload vs the grouped kernel on norm_out")
    assert_bytes_equal(sf, e.sf.cpu().numpy(), "scales vs the grouped kernel on norm_out")
