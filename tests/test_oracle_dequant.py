"""Pins of the oracle's dequantization (R11): decoded values against an
independent decoder -- torch's float8_e4m3fn conversion and the e2m1 code
table of tests/golden for the element values, exact rational products, and a
bf16 rounding written here on exact rationals -- plus the MXFP8 round trip
quantize(dequantize(q)) == q and the agreement of the two SF layouts."""
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth
from golden_io import rows

E2M1 = {int(c): Fraction(v) for c, v in rows("e2m1_values.txt")}


def e4m3_values():
    """float64 values of all 256 e4m3 codes (torch's float8_e4m3fn decoder)."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def bf16_rne(v: Fraction, negative: bool) -> int:
    """bf16 bits of the exact rational |v| with the given sign, round half to even
    (8 significant bits; subnormal step 2^-133)."""
    sign = 0x8000 if negative else 0
    a = abs(v)
    if a == 0:
        return sign
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)
    step = Fraction(2) ** (e - 7)
    n = a / step
    f = n.numerator // n.denominator
    rem = n - f
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and f % 2 == 1):
        f += 1
    r = f * step
    bits = struct.unpack("<I", struct.pack("<f", float(r)))[0]   # r has <= 9 significant bits
    assert bits & 0xFFFF == 0
    return sign | (bits >> 16)


def sf_linear(sf, rows_, kv, layout):
    return sf.reshape(rows_, kv) if layout == oracle.LINEAR else oracle.unswizzle(sf, rows_, kv).reshape(rows_, kv)


@pytest.mark.parametrize("layout", [oracle.LINEAR, oracle.SWIZZLED])
def test_mxfp8_dequant_matches_independent_decode(layout):
    vals = e4m3_values()
    for x in (synth.tiny_group()[1], synth.blockwise_scaled((96, 320), 32, seed=11)):
        xb = synth.bf16_bits(x)
        q, sf = oracle.quantize_mxfp8(xb, layout)
        y = oracle.dequantize_mxfp8(q, sf, layout)
        R, C = xb.shape
        s = sf_linear(sf, R, C // 32, layout).astype(np.int64)
        ref = vals[q] * np.exp2(np.repeat(s, 32, axis=1) - 127.0)   # exact in binary64
        f32 = ref.astype(np.float32)
        assert np.array_equal(f32.astype(np.float64), ref)          # representable: no rounding
        bits = f32.view(np.uint32)
        assert not np.any(bits & 0xFFFF)
        assert np.array_equal(y, (bits >> 16).astype(np.uint16))


@pytest.mark.parametrize("layout", [oracle.LINEAR, oracle.SWIZZLED])
def test_mxfp8_requantize_round_trip(layout):
    """Decoded MXFP8 values are exact bf16 numbers of at most 4 significant
    bits, so quantizing them again loses nothing: the decode of the second
    quantization equals the first decode.  (The bytes themselves can differ: a
    block whose largest element rounds to exactly 224 * 2^e gets the scale
    2^(e-1) the second time, and every code doubles.)"""
    x = synth.blockwise_scaled((128, 256), 32, seed=12)
    xb = synth.bf16_bits(x)
    q, sf = oracle.quantize_mxfp8(xb, layout)
    y = oracle.dequantize_mxfp8(q, sf, layout)
    q2, sf2 = oracle.quantize_mxfp8(y, layout)
    assert np.array_equal(oracle.dequantize_mxfp8(q2, sf2, layout), y)
    vals = e4m3_values()
    s = sf_linear(sf, 128, 8, layout).astype(np.int64)
    s2 = sf_linear(sf2, 128, 8, layout).astype(np.int64)
    top = np.abs(vals[q]).reshape(128, 8, 32).max(axis=2)
    assert np.array_equal(s2, np.where(top == 224.0, s - 1, s))   # the only change of scale


@pytest.mark.parametrize("per_row", [False, True])
def test_nvfp4_dequant_every_code_and_scale(per_row):
    """Every e2m1 code under every finite block-scale code, exact products
    rounded once to bf16."""
    vals = e4m3_values()
    scales = np.arange(127, dtype=np.uint8)             # 0x00 .. 0x7E
    R = len(scales)
    codes = np.arange(16, dtype=np.uint8)
    q = np.tile((codes[0::2] | (codes[1::2] << 4)).astype(np.uint8), (R, 1))   # one 16-element block per row
    # the last three make some product round differently if it were first
    # rounded to binary32 (found by a search over amax values)
    amaxes = [3.0, 1.0 / 3.0, 448.0 * 6.0, 0.0171, 2.0 ** -90, 5.0e4, 27.50284194946289, 36.21154022216797, 76.34375]
    for A in amaxes:
        amax = np.full(R if per_row else 1, A, dtype=np.float32)
        if per_row:
            amax = (amax * np.linspace(0.5, 2.0, R)).astype(np.float32)
        y = oracle.dequantize_nvfp4(q, scales.copy(), amax, per_row, oracle.LINEAR)
        for r in range(R):
            g = np.float32(amax[r] if per_row else amax[0]) / np.float32(2688.0)   # binary32 quotient
            s_val = Fraction(float(vals[scales[r]]))
            for c in range(16):
                v = E2M1[c & 7] * s_val * Fraction(float(g))
                assert y[r, c] == bf16_rne(v, negative=bool(c & 8)), (A, r, c)


def test_nvfp4_dequant_swizzled_equals_linear():
    x = synth.bf16_bits(synth.blockwise_scaled((200, 96), 16, seed=13))
    out = []
    for layout in (oracle.LINEAR, oracle.SWIZZLED):
        q, sf, amax = oracle.quantize_nvfp4(x, layout, oracle.NVFP4_PER_ROW)
        out.append(oracle.dequantize_nvfp4(q, sf, amax, True, layout))
    assert np.array_equal(out[0], out[1])


def test_nvfp4_dequant_close_to_input():
    """The decoded tensor approximates the input: every element within a
    quarter of its block's amax (the coarsest e2m1 step is 2 of 6)."""
    xb = synth.bf16_bits(synth.normal_bf16((64, 128), 1.0, seed=14))
    q, sf, amax = oracle.quantize_nvfp4(xb, oracle.LINEAR, oracle.NVFP4_PER_TENSOR_COMPUTE)
    y = oracle.dequantize_nvfp4(q, sf, amax, False, oracle.LINEAR)
    xf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    yf = (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    bmax = np.abs(xf).reshape(64, 8, 16).max(axis=2, keepdims=True)
    err = np.abs(xf - yf).reshape(64, 8, 16)
    assert np.all(err <= bmax / 4 + 1e-30)
