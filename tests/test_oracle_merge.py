"""Pins of the oracle's attention decode merge (R12) by the cases whose
result is exact: one split (each element rounded to bf16), splits with equal
log-sum-exps (the plain mean, rounded once), one split dominating by e^200,
log-sum-exps near 1000 (the maximum must be subtracted before exp), and
shift invariance on exactly representable shifts."""
from fractions import Fraction

import numpy as np

import oracle
from test_oracle_dequant import bf16_rne


def rne_f32_to_bf16(a: np.ndarray) -> np.ndarray:
    """bf16 bits of float32 values, round half to even, on the integer bits."""
    u = a.astype(np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def parts(S, T, H, seed):
    rng = np.random.default_rng(seed)
    O = (rng.standard_normal((S, T, H)) * np.exp2(rng.uniform(-8, 8, (S, T, 1)))).astype(np.float32)
    lse = np.round(rng.uniform(-4, 4, (S, T)) * 1024) / 1024
    return O, lse.astype(np.float32)


def test_single_split_is_the_rounded_input():
    O, lse = parts(1, 5, 96, 1)
    assert np.array_equal(oracle.attention_merge(O, lse), rne_f32_to_bf16(O[0]))


def test_equal_weights_give_the_mean():
    S, T, H = 3, 4, 64
    O, _ = parts(S, T, H, 2)
    lse = np.full((S, T), 1.25, dtype=np.float32)
    y = oracle.attention_merge(O, lse)
    for t in range(T):
        for i in range(H):
            mean = sum(Fraction(float(O[s, t, i])) for s in range(S)) / S
            assert y[t, i] == bf16_rne(mean, mean < 0), (t, i)


def test_dominant_split_and_large_lse():
    S, T, H = 4, 3, 32
    O, lse = parts(S, T, H, 3)
    lse = lse + np.float32(1000.0)        # exp would overflow without subtracting the maximum
    lse[2] += np.float32(200.0)           # split 2 outweighs the others by e^200
    assert np.array_equal(oracle.attention_merge(O, lse), rne_f32_to_bf16(O[2]))


def test_shift_invariance():
    O, lse = parts(5, 6, 48, 4)
    a = oracle.attention_merge(O, lse)
    b = oracle.attention_merge(O, (lse + np.float32(16.0)).astype(np.float32))   # exact shift (lse on 2^-10)
    assert np.array_equal(a, b)


def test_quantized_form_is_the_quantizer_on_the_merge():
    """The merged tensor's MXFP8 form is the plain quantizer applied to it
    (nothing else is defined for it)."""
    O, lse = parts(8, 3, 256, 5)
    y = oracle.attention_merge(O, lse)
    q, sf = oracle.quantize_mxfp8(y, oracle.SWIZZLED)
    assert q.shape == (3, 256) and sf.size == oracle.sf_region_bytes(3, 8, oracle.SWIZZLED)
