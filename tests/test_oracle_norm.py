"""Pins of the oracle's residual-add + RMSNorm: hand-worked closed forms,
power-of-two scale invariance, constant rows, the bf16 residual against torch."""
import numpy as np
import pytest
import torch

import oracle
import synth
from golden_io import rows


def bf(vals):
    t = torch.tensor([float(v) for v in vals], dtype=torch.float32).to(torch.bfloat16)
    return synth.bf16_bits(t).reshape(1, -1)


def test_closed_forms_golden():
    for case, H, xs, rs, gs, eps, yh, hh in rows("rmsnorm_closed_form.txt"):
        x = bf(xs.split(","))
        r = bf(rs.split(","))
        g = bf(gs.split(",")).reshape(-1)
        y, h = oracle.residual_rmsnorm(x, r, g, float(eps))
        assert [f"{v:04X}" for v in y[0]] == yh.split(","), case
        assert [f"{v:04X}" for v in h[0]] == hh.split(","), case


def test_scale_invariance_power_of_two():
    x, r, g = synth.fused_norm_inputs(4, hidden=512, seed=3)
    y0, _ = oracle.residual_rmsnorm(synth.bf16_bits(x), synth.bf16_bits(r), synth.bf16_bits(g), 0.0)
    for k in (-6, 3, 17):
        y1, _ = oracle.residual_rmsnorm(synth.bf16_bits(x * 2.0 ** k), synth.bf16_bits(r * 2.0 ** k),
                                        synth.bf16_bits(g), 0.0)
        assert np.array_equal(y0, y1)


def test_constant_row_gives_gamma():
    H = 384
    g = synth.bf16_bits((torch.rand(H, generator=torch.Generator().manual_seed(2)) + 0.5).to(torch.bfloat16))
    for c in (1.0, -3.0, 0.3, 1.0 + 2.0 ** -8):
        x = bf([c] * H)
        r = bf([2.0 ** -9] * H)          # x + r is inexact in bf16 for c = 1 + 2^-8
        y, h = oracle.residual_rmsnorm(x, r, g, 0.0)
        gt = torch.from_numpy(g.view(np.int16)).view(torch.bfloat16)
        hv = torch.from_numpy(h[0].view(np.int16)).view(torch.bfloat16).float()
        expect = synth.bf16_bits(gt * torch.sign(hv).to(torch.bfloat16))
        assert np.array_equal(y[0], expect), c


def test_residual_matches_torch():
    x, r, g = synth.fused_norm_inputs(8, hidden=1024, seed=9)
    _, h = oracle.residual_rmsnorm(synth.bf16_bits(x), synth.bf16_bits(r), synth.bf16_bits(g), 1e-6)
    ref = synth.bf16_bits((x.float() + r.float()).to(torch.bfloat16))
    assert np.array_equal(h, ref)


def test_unit_rms_when_eps_zero():
    x, r, _ = synth.fused_norm_inputs(6, hidden=2048, seed=10)
    g = synth.bf16_bits(torch.ones(2048, dtype=torch.bfloat16))
    y, _ = oracle.residual_rmsnorm(synth.bf16_bits(x), synth.bf16_bits(r), g, 0.0)
    yv = (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ms = (yv ** 2).mean(axis=1)
    assert np.all(np.abs(ms - 1.0) < 2 ** -7)


@pytest.mark.parametrize("fmt,layout", [(oracle.MXFP8, oracle.SWIZZLED), (oracle.NVFP4, oracle.LINEAR)])
def test_fused_equals_norm_then_quantize(fmt, layout):
    x, r, g = synth.fused_norm_inputs(5, hidden=7168, seed=4)
    xb, rb, gb = synth.bf16_bits(x), synth.bf16_bits(r), synth.bf16_bits(g)
    y, h = oracle.residual_rmsnorm(xb, rb, gb, 1e-6)
    A = float(np.abs((y.astype(np.uint32) << 16).view(np.float32)).max())
    y2, h2, q, sf = oracle.rmsnorm_quantize(xb, rb, gb, 1e-6, fmt, layout, A)
    assert np.array_equal(y, y2) and np.array_equal(h, h2)
    if fmt == oracle.MXFP8:
        q3, sf3 = oracle.quantize_mxfp8(y, layout)
    else:
        q3, sf3, _ = oracle.quantize_nvfp4(y, layout, oracle.NVFP4_PER_TENSOR_GIVEN, A)
    assert np.array_equal(q, q3) and np.array_equal(sf, sf3)
