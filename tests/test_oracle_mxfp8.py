"""Pins of the oracle's MXFP8 path: the E8M0 exponent rule against a closed
form on every bf16 amax, the block invariants and dequantization bound, brute
force on tiny blocks, zero blocks and signed zeros, strided input."""
import math

import numpy as np
import torch

import oracle
import synth


def all_positive_finite_bf16():
    bits = np.arange(1, 0x7F80, dtype=np.uint32)          # +subnormals .. largest finite
    vals = (bits << 16).view(np.float32).astype(np.float64)
    return bits, vals


def closed_form_exponent(bits):
    """Smallest e with amax <= 448 * 2^e, from the bf16 fields alone:
    amax = (1 + m/128) * 2^E; 448 = 1.75 * 2^8, so e = E - 8 when the
    significand is at most 1.75 (m <= 96) and E - 7 otherwise; subnormal
    amax (< 2^-126) lies below 448 * 2^-128 and clamps to -127."""
    E = ((bits >> 7) & 0xFF).astype(np.int64) - 127
    m = (bits & 0x7F).astype(np.int64)
    e = np.where(m <= 96, E - 8, E - 7)
    e = np.where(((bits >> 7) & 0xFF) == 0, -127, e)
    return np.maximum(e, -127)


def test_e8m0_exhaustive_closed_form(olib):
    bits, vals = all_positive_finite_bf16()
    got = np.array([olib.qzo_mx_scale_exponent(float(v)) for v in vals])
    assert np.array_equal(got, closed_form_exponent(bits))


def test_e8m0_invariants(olib):
    _, vals = all_positive_finite_bf16()
    for v in vals[::37]:
        e = olib.qzo_mx_scale_exponent(float(v))
        assert -127 <= e <= 120
        assert v <= 448.0 * 2.0 ** e
        if e > -127:
            assert v > 224.0 * 2.0 ** e         # not representable with e - 1


def test_e8m0_exact_at_powers(olib):
    for j in range(-126, 121):
        assert olib.qzo_mx_scale_exponent(448.0 * 2.0 ** j) == max(j, -127)
    assert olib.qzo_mx_scale_exponent(0.0) == -127


def test_mx_reciprocal_ftz(olib):
    assert olib.qzo_mx_reciprocal(127) == 0.0          # 2^-127 is subnormal -> 0
    assert olib.qzo_mx_reciprocal(126) == 2.0 ** -126
    assert olib.qzo_mx_reciprocal(-127) == 2.0 ** 127
    assert olib.qzo_mx_reciprocal(0) == 1.0


def _fp32(a):
    return np.asarray(a, dtype=np.float32)


def _decode_e4m3(codes):
    return torch.from_numpy(codes.astype(np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def check_block_bounds(xb, q, sf_lin):
    """Dequantization bound and scale invariants for MXFP8 rows."""
    xf = xb.astype(np.uint32) << 16
    x = xf.view(np.float32).astype(np.float64)
    rows, cols = x.shape
    kv = cols // 32
    e = sf_lin.reshape(rows, kv).astype(np.int64) - 127
    deq = _decode_e4m3(q) * np.exp2(np.repeat(e, 32, axis=1).astype(np.float64))
    amax = np.abs(x).reshape(rows, kv, 32).max(axis=2)
    live = (amax > 0) & (e > -127)
    sc = amax[live] * np.exp2(-e[live].astype(np.float64))
    assert np.all(sc <= 448.0) and np.all(sc > 224.0)
    ee = np.repeat(e, 32, axis=1).astype(np.float64)
    tol = np.maximum(np.abs(x) * 2.0 ** -4, np.exp2(ee - 10))
    assert np.all(np.abs(x - deq) <= tol)
    # sign carried, zeros included
    neg = np.signbit(x)
    assert np.array_equal((q & 0x80) != 0, neg)


def test_mxfp8_bounds_blockwise_scaled():
    x = synth.bf16_bits(synth.blockwise_scaled((96, 320), 32, seed=5))
    for layout in (oracle.LINEAR, oracle.SWIZZLED):
        q, sf = oracle.quantize_mxfp8(x, layout)
        lin = sf if layout == oracle.LINEAR else oracle.unswizzle(sf, 96, 10)
        check_block_bounds(x, q, lin)


def test_mxfp8_bounds_random_bits():
    x = synth.bf16_bits(synth.random_finite_bf16((64, 256), seed=9))
    q, sf = oracle.quantize_mxfp8(x, oracle.LINEAR)
    check_block_bounds(x, q, sf)


def test_mxfp8_bruteforce_tiny_blocks(olib):
    """Every e in [-127, 127]: the chosen one is the least for which no scaled
    element exceeds 448; each code is the nearest (ties even) e4m3 value of
    the binary32 product x * 2^-e."""
    t = _decode_e4m3(np.arange(128))
    cand = [c for c in range(127)]
    cv = t[cand]
    x = synth.bf16_bits(synth.blockwise_scaled((6, 64), 32, seed=21, lo=-20, hi=20))
    q, sf = oracle.quantize_mxfp8(x, oracle.LINEAR)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    for r in range(6):
        for k in range(2):
            blk = xf[r, k * 32:(k + 1) * 32].astype(np.float64)
            ok = [e for e in range(-127, 128) if np.all(np.abs(blk) <= 448.0 * 2.0 ** e)]
            e = min(ok)
            assert sf[r * 2 + k] == e + 127
            for i in range(32):
                y = np.float32(xf[r, k * 32 + i]) * np.float32(2.0 ** -e)
                d = np.abs(cv - min(abs(float(y)), 448.0))
                best = [cand[b] for b in np.nonzero(d == d.min())[0]]
                if len(best) > 1:
                    best = [b for b in best if b % 2 == 0]
                code = best[0] | (0x80 if np.signbit(y) else 0)
                assert q[r, k * 32 + i] == code


def test_mxfp8_zero_and_negative_zero_blocks():
    x = np.zeros((2, 64), dtype=np.uint16)
    x[1, 32:] = 0x8000                                    # -0.0
    q, sf = oracle.quantize_mxfp8(x, oracle.LINEAR)
    assert np.all(sf == 0)
    assert np.all(q[0] == 0) and np.all(q[1, :32] == 0) and np.all(q[1, 32:] == 0x80)


def test_mxfp8_strided_rows_equal_contiguous():
    full = synth.bf16_bits(synth.normal_bf16((40, 384), seed=4))
    view = full[:, :256]
    q1, s1 = oracle.quantize_mxfp8(view, oracle.SWIZZLED)
    q2, s2 = oracle.quantize_mxfp8(np.ascontiguousarray(view), oracle.SWIZZLED)
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


def test_mxfp8_swizzled_equals_linear_after_unswizzle():
    x = synth.bf16_bits(synth.tiny_group()[0])
    q1, lin = oracle.quantize_mxfp8(x, oracle.LINEAR)
    q2, swz = oracle.quantize_mxfp8(x, oracle.SWIZZLED)
    assert np.array_equal(q1, q2)
    assert np.array_equal(oracle.unswizzle(swz, 64, 8), lin)
    assert np.array_equal(oracle.swizzle(lin, 64, 8), swz)
    lib = oracle.load()
    live = np.zeros(swz.size, dtype=bool)
    for r in range(64):
        for k in range(8):
            live[lib.qzo_sf_offset_swizzled(r, k, 8)] = True
    assert swz.size == 128 * 8 and live.sum() == 64 * 8
    assert np.all(swz[~live] == 0)
