"""GPU parity of the fused residual-add + RMSNorm + quantize kernel.

* residual_out: bit-exact with the oracle's bf16(x + r);
* norm_out: within 1 bf16 ulp of the oracle (binary64 reference) everywhere,
  and the count of elements off by one ulp is reported and bounded;
* quantized output: bit-exact with the oracle in every scale block whose y
  equals the oracle's y, and everywhere bit-exact with the oracle quantizer
  applied to the fused kernel's own norm_out (the fold must equal quantizing
  norm_out afterwards; TensorRT-LLM "NVFP4 linear-SF AllReduce epilogue",
  commit 3: atol = rtol = 0 against quantizing the norm output), padding
  included;
* the swizzled layout's padded rows are zero;
* both launch shapes of the kernel: the latency shape (T <= 2 x SMs, one
  896-thread CTA per row) and the throughput shape (T above that, 224-thread
  CTAs, four 16-byte chunks per thread), in both formats and layouts.
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


def oracle_on_y(y, fmt, layout, amax=None):
    """The oracle quantizer applied to the fused kernel's own norm_out."""
    yb = host_bits(y)
    if fmt == qz.FMT_MXFP8:
        return oracle.quantize_mxfp8(yb, layout)
    q, sf, _ = oracle.quantize_nvfp4(yb, layout, oracle.NVFP4_PER_TENSOR_GIVEN, amax)
    return q, sf


def check_fold(y, q, sf, fmt, layout, amax, what):
    qo, sfo = oracle_on_y(y, fmt, layout, amax)
    assert_bytes_equal(q, qo.reshape(q.shape), f"{what}: payload vs the oracle on norm_out")
    assert_bytes_equal(sf, sfo, f"{what}: scales vs the oracle on norm_out (padding included)")


def oracle_amax(xc, rc, gc, eps):
    """The NVFP4 global amax of the fused workload: the amax of the oracle's y."""
    y_ref, _ = oracle.residual_rmsnorm(host_bits(xc), host_bits(rc), host_bits(gc), eps)
    return float(np.abs((y_ref.astype(np.uint32) << 16).view(np.float32)).max())


CASES = [(1, qz.FMT_MXFP8, qz.SF_SWIZZLED), (3, qz.FMT_MXFP8, qz.SF_SWIZZLED), (129, qz.FMT_MXFP8, qz.SF_SWIZZLED),
         (64, qz.FMT_MXFP8, qz.SF_LINEAR), (1, qz.FMT_NVFP4, qz.SF_LINEAR), (77, qz.FMT_NVFP4, qz.SF_LINEAR),
         (130, qz.FMT_NVFP4, qz.SF_SWIZZLED), (256, qz.FMT_NVFP4, qz.SF_LINEAR),
         # throughput shape (T > 2 x 148 SMs)
         (297, qz.FMT_NVFP4, qz.SF_SWIZZLED), (297, qz.FMT_MXFP8, qz.SF_LINEAR),
         (512, qz.FMT_NVFP4, qz.SF_LINEAR), (512, qz.FMT_NVFP4, qz.SF_SWIZZLED),
         (512, qz.FMT_MXFP8, qz.SF_SWIZZLED), (1000, qz.FMT_MXFP8, qz.SF_LINEAR),
         (4096, qz.FMT_NVFP4, qz.SF_LINEAR), (4096, qz.FMT_NVFP4, qz.SF_SWIZZLED),
         (4096, qz.FMT_MXFP8, qz.SF_SWIZZLED)]


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
    # and everywhere equal to the oracle quantizer applied to the fused norm_out
    check_fold(y, q, sf, fmt, layout, A, f"T={T}")
    if layout == qz.SF_SWIZZLED and T <= 512:   # (larger T: covered by the padding-inclusive check above)
        lib = oracle.load()
        live = np.zeros(sf.size, dtype=bool)
        for rr in range(T):
            for k in range(H // blk):
                live[lib.qzo_sf_offset_swizzled(rr, k, H // blk)] = True
        assert not np.any(sf[~live]), "padded rows of the swizzled layout must be zero"


@pytest.mark.parametrize("fmt,layout", [(qz.FMT_MXFP8, qz.SF_SWIZZLED), (qz.FMT_NVFP4, qz.SF_LINEAR)])
def test_fused_sweep_without_residual_out(fmt, layout):
    """T over the powers of two up to 4096 (the fused workload's sweep, in
    its two prescribed forms: MXFP8 swizzled, NVFP4 linear with the global
    amax taken from the oracle's y): residual_out omitted, norm_out within 1
    ulp of the oracle, quantized bytes equal to the oracle quantizer on the
    kernel's own norm_out."""
    eps = synth.FUSED_NORM["eps"]
    for T in synth.FUSED_NORM["tokens"]:
        xc, rc, gc = synth.fused_norm_inputs(T, device="cuda")
        A = oracle_amax(xc, rc, gc, eps) if fmt == qz.FMT_NVFP4 else None
        y, h, q, sf = run_fused(xc, rc, gc, eps, fmt, layout, A, with_residual=False)
        check_fold(y, q, sf, fmt, layout, A, f"T={T}")
        y_ref, _ = oracle.residual_rmsnorm(host_bits(xc), host_bits(rc), host_bits(gc), eps)
        assert bf16_ulp_diff(host_bits(y), y_ref).max() <= 1, f"T={T}"


@pytest.mark.parametrize("fmt,layout", [(qz.FMT_MXFP8, qz.SF_SWIZZLED), (qz.FMT_NVFP4, qz.SF_LINEAR),
                                        (qz.FMT_NVFP4, qz.SF_SWIZZLED)])
def test_fused_full_size_sampled_rows(fmt, layout):
    """T = 4096 rows at H = 7168 in the bench's launch shape: 64 sampled rows
    of norm_out and residual_out compared with the oracle row by row, every
    quantized byte with the oracle quantizer on the kernel's norm_out."""
    T, H = 4096, synth.FUSED_NORM["hidden"]
    eps = synth.FUSED_NORM["eps"]
    xc, rc, gc = synth.fused_norm_inputs(T, device="cuda")
    A = oracle_amax(xc, rc, gc, eps) if fmt == qz.FMT_NVFP4 else None
    y, h, q, sf = run_fused(xc, rc, gc, eps, fmt, layout, A)
    rows = np.random.default_rng(4).choice(T, 64, replace=False)
    xb, rb, gb = host_bits(xc[rows]), host_bits(rc[rows]), host_bits(gc)
    y_ref, h_ref = oracle.residual_rmsnorm(xb, rb, gb, eps)
    assert_bytes_equal(host_bits(h)[rows], h_ref, "residual_out")
    assert bf16_ulp_diff(host_bits(y)[rows], y_ref).max() <= 1
    check_fold(y, q, sf, fmt, layout, A, "T=4096")
