"""Pins of the oracle's AllReduce ahead of the fused epilogue (reading R15: the
bf16 rounding of a binary32 sum taken in rank order): hand-worked elements
where the order and the binary32 accumulation decide, exact integer sums at
every rank count, the identities of one rank and of zero ranks, and the
epilogue fed with a sum known without the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from golden_io import rows


def bf(vals):
    t = torch.tensor([float(v) for v in vals], dtype=torch.float32).to(torch.bfloat16)
    return synth.bf16_bits(t).reshape(1, -1)


def test_worked_examples_golden():
    for case, expect, *values in rows("rank_sum.txt"):
        out = oracle.rank_sum([bf([v]) for v in values])
        assert f"{int(out[0, 0]):04X}" == expect, case


def integer_ranks(n, shape, seed):
    g = torch.Generator().manual_seed(seed)
    return [torch.randint(-16, 17, shape, generator=g).to(torch.float32) for _ in range(n)]


@pytest.mark.parametrize("n", range(1, 9))
def test_integer_sums_are_exact_in_any_rank_order(n):
    # |sum| <= 128: every partial sum and the result are exact in binary32 and bf16
    xs = integer_ranks(n, (3, 64), seed=n)
    expect = synth.bf16_bits(sum(xs).to(torch.bfloat16))
    bits = [synth.bf16_bits(x.to(torch.bfloat16)) for x in xs]
    assert np.array_equal(oracle.rank_sum(bits), expect)
    assert np.array_equal(oracle.rank_sum(bits[::-1]), expect)


def test_one_rank_is_the_identity():
    x = synth.bf16_bits(synth.random_finite_bf16((16, 256), seed=21))
    assert np.array_equal(oracle.rank_sum([x]), x)


def test_zero_ranks_add_nothing_but_the_sign_of_zero():
    x = synth.bf16_bits(synth.random_finite_bf16((16, 256), seed=22))
    z = np.zeros_like(x)
    expect = np.where(x == 0x8000, 0, x).astype(np.uint16)   # -0 + +0 = +0
    assert np.array_equal(oracle.rank_sum([x, z, z]), expect)
    assert np.array_equal(oracle.rank_sum([z, x]), expect)


def test_two_exact_halves_give_the_whole():
    x, _, _ = synth.fused_norm_inputs(4, hidden=512, seed=23)
    half = synth.bf16_bits((x.float() * 0.5).to(torch.bfloat16))   # exact: normal values halved
    assert np.array_equal(oracle.rank_sum([half, half]), synth.bf16_bits(x))


@pytest.mark.parametrize("fmt,layout", [(oracle.MXFP8, oracle.SWIZZLED), (oracle.NVFP4, oracle.LINEAR),
                                        (oracle.NVFP4, oracle.SWIZZLED)])
def test_epilogue_runs_on_the_sum(fmt, layout):
    n, T, H = 4, 5, 256
    xs = integer_ranks(n, (T, H), seed=30 + fmt)
    x_sum = synth.bf16_bits(sum(xs).to(torch.bfloat16))
    _, r, g = synth.fused_norm_inputs(T, hidden=H, seed=31)
    r, g = synth.bf16_bits(r), synth.bf16_bits(g)
    amax = 80.0 if fmt == oracle.NVFP4 else None
    got = oracle.allreduce_rmsnorm_quantize([synth.bf16_bits(x.to(torch.bfloat16)) for x in xs], r, g, 1e-6,
                                            fmt, layout, amax)
    want = oracle.rmsnorm_quantize(x_sum, r, g, 1e-6, fmt, layout, amax)
    for a, b in zip(got, want):
        assert np.array_equal(a, b)
