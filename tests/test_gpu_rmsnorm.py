"""GPU parity of the fused residual-add + RMSNorm + quantize kernel.

* residual_out: bit-exact with the oracle's bf16(x + r);
* norm_out: within 1 bf16 ulp of the oracle (binary64 reference) everywhere,
  and the count of elements off by one ulp is reported and bounded;
* quantized output: bit-exact with the oracle in every scale block whose y
  equals the oracle's y; in the other blocks, the payload and scale bytes are
  those the grouped GPU kernel (itself bit-exact against the oracle) produces
  from the fused kernel's own norm_out -- the fold is bitwise the same as
  quantizing norm_out afterwards;
* the swizzled layout's padded rows are zero.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import Guarded, assert_bytes_equal, bf16_ulp_diff, host_bits

pytestmark = pytest.mark.gpu

qz = pytest.importorskip("nvfp4_quantization_moe_b200")


def run_fused(x, r, g, eps, fmt, layout, amax=None, with_residual=True):
    T, H = x.shape
    y = torch.empty_like(x)
    h = torch.empty_like(x) if with_residual else None
    qcols = H if fmt == qz.FMT_MXFP8 else H // 2
    q = Guarded(T * qcols)
    sf = Guarded(qz.sf_bytes(T, H, fmt, layout))
    a = None
    if fmt == qz.FMT_NVFP4:
        a = torch.tensor([amax], dtype=torch.float32, device=x.device)
    qz.rmsnorm_quantize(x, r, g, eps, y, h, fmt, q.view, sf.view, layout, a)
    torch.cuda.synchronize()
    assert q.guards_intact() and sf.guards_intact()
    return y, h, q.host().reshape(T, qcols), sf.host()


def standalone(y, fmt, layout, amax=None):
    """The grouped kernel on the fused kernel's own norm_out."""
    mode = qz.NVFP4_PER_TENSOR_GIVEN
    e = qz.quantize_experts([y], fmt, layout, mode, [amax] if amax is not None else None)[0]
    torch.cuda.synchronize()
    return e.q.cpu().numpy(), e.sf.cpu().numpy()


CASES = [(1, qz.FMT_MXFP8, qz.SF_SWIZZLED), (3, qz.FMT_MXFP8, qz.SF_SWIZZLED), (129, qz.FMT_MXFP8, qz.SF_SWIZZLED),
         (64, qz.FMT_MXFP8, qz.SF_LINEAR), (1, qz.FMT_NVFP4, qz.SF_LINEAR), (77, qz.FMT_NVFP4, qz.SF_LINEAR),
         (130, qz.FMT_NVFP4, qz.SF_SWIZZLED), (256, qz.FMT_NVFP4, qz.SF_LINEAR)]


@pytest.mark.parametrize("T,fmt,layout", CASES)
def test_fused_parity(T, fmt, layout):
    H = synth.FUSED_NORM["hidden"]
    eps = synth.FUSED_NORM["eps"]
    xc, rc, gc = synth.fused_norm_inputs(T, seed=synth.FUSED_NORM["seed"] + T)
    xb, rb, gb = host_bits(xc), host_bits(rc), host_bits(gc)
    y_ref, h_ref = oracle.residual_rmsnorm(xb, rb, gb, eps)
    A = float(np.abs((y_ref.astype(np.uint32) << 16).view(np.float32)).max()) if fmt == qz.FMT_NVFP4 else None
    y_ref, h_ref, q_ref, sf_ref = oracle.rmsnorm_quantize(xb, rb, gb, eps, fmt, layout, A)
    x, r, g = xc.cuda(), rc.cuda(), gc.cuda()
    y, h, q, sf = run_fused(x, r, g, eps, fmt, layout, A)
    yh, hh = host_bits(y), host_bits(h)
    assert_bytes_equal(hh, h_ref, "residual_out")
    d = bf16_ulp_diff(yh, y_ref)
    assert d.max() <= 1, f"norm_out off by {d.max()} ulp"
    assert (d > 0).mean() < 1e-3, f"{(d > 0).sum()} elements off by one ulp"
    # quantized output: exact where y agrees blockwise with the oracle
    blk = 32 if fmt == qz.FMT_MXFP8 else 16
    same = (d.reshape(T, H // blk, blk) == 0).all(axis=2)
    if fmt == qz.FMT_MXFP8:
        qg, qr = q.reshape(T, H // blk, blk), q_ref.reshape(T, H // blk, blk)
    else:
        qg, qr = q.reshape(T, H // blk, blk // 2), q_ref.reshape(T, H // blk, blk // 2)
    assert np.array_equal(qg[same], qr[same])
    lin_g = sf if layout == qz.SF_LINEAR else oracle.unswizzle(sf, T, H // blk)
    lin_r = sf_ref if layout == qz.SF_LINEAR else oracle.unswizzle(sf_ref, T, H // blk)
    assert np.array_equal(lin_g.reshape(T, -1)[same], lin_r.reshape(T, -1)[same])
    # and everywhere equal to the grouped kernel applied to the fused norm_out
    qs, sfs = standalone(y, fmt, layout, A)
    assert_bytes_equal(q, qs.reshape(q.shape), "fused vs standalone payload")
    assert_bytes_equal(sf, sfs, "fused vs standalone scales (padding included)")
    if layout == qz.SF_SWIZZLED:
        lib = oracle.load()
        live = np.zeros(sf.size, dtype=bool)
        for rr in range(T):
            for k in range(H // blk):
                live[lib.qzo_sf_offset_swizzled(rr, k, H // blk)] = True
        assert not np.any(sf[~live]), "padded rows of the swizzled layout must be zero"


def test_fused_without_residual_out_and_sweep_bits():
    """T over the powers of two up to 4096 (the fused workload's sweep):
    residual_out omitted, norm_out within 1 ulp, quantized bytes equal to the
    grouped kernel on norm_out."""
    H = synth.FUSED_NORM["hidden"]
    for T in synth.FUSED_NORM["tokens"]:
        xc, rc, gc = synth.fused_norm_inputs(T, device="cuda")
        y, h, q, sf = run_fused(xc, rc, gc, 1e-6, qz.FMT_MXFP8, qz.SF_SWIZZLED, with_residual=False)
        qs, sfs = standalone(y, qz.FMT_MXFP8, qz.SF_SWIZZLED)
        assert_bytes_equal(q, qs.reshape(q.shape), f"T={T} payload")
        assert_bytes_equal(sf, sfs, f"T={T} scales")
        if T <= 256:
            y_ref, _ = oracle.residual_rmsnorm(host_bits(xc), host_bits(rc), host_bits(gc), 1e-6)
            assert bf16_ulp_diff(host_bits(y), y_ref).max() <= 1


def test_fused_full_size_sampled_rows():
    """T = 4096 rows at H = 7168 in the bench's launch shape; 64 sampled rows
    compared with the oracle row by row."""
    T, H = 4096, synth.FUSED_NORM["hidden"]
    xc, rc, gc = synth.fused_norm_inputs(T, device="cuda")
    y, h, q, sf = run_fused(xc, rc, gc, 1e-6, qz.FMT_MXFP8, qz.SF_SWIZZLED)
    rows = np.random.default_rng(4).choice(T, 64, replace=False)
    xb, rb, gb = host_bits(xc[rows]), host_bits(rc[rows]), host_bits(gc)
    y_ref, h_ref = oracle.residual_rmsnorm(xb, rb, gb, 1e-6)
    assert_bytes_equal(host_bits(h)[rows], h_ref, "residual_out")
    assert bf16_ulp_diff(host_bits(y)[rows], y_ref).max() <= 1
    qs, sfs = standalone(y, qz.FMT_MXFP8, qz.SF_SWIZZLED)
    assert_bytes_equal(q, qs.reshape(q.shape), "payload")
    assert_bytes_equal(sf, sfs, "scales")
