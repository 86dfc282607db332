"""Pins of the oracle's NVFP4 path: dequantization bound of every element,
scale-range invariants, the all-zero and zero-block special cases, the
per-tensor amax against numpy's max, split == per-expert for row scaling."""
import numpy as np
import pytest
import torch

import oracle
import synth
from golden_io import rows

E2M1 = {int(c): float(v) for c, v in rows("e2m1_values.txt")}


def e4m3_vals(codes):
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def unpack(q):
    lo = q & 0xF
    hi = q >> 4
    out = np.empty((q.shape[0], q.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def fvals(xb):
    return (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check_nvfp4(xb, q, sf_lin, A_rows):
    """A_rows: the second-level amax that applies to each row."""
    x = fvals(xb)
    R, K = x.shape
    kv = K // 16
    s = e4m3_vals(sf_lin.reshape(R, kv))
    assert np.all(s >= 0) and np.all(s <= 448)
    g = (np.asarray(A_rows, dtype=np.float32) / np.float32(2688.0)).astype(np.float64)
    codes = unpack(q)
    qv = np.vectorize(E2M1.get)(codes).astype(np.float64)
    sc = np.repeat(s, 16, axis=1) * g[:, None]              # decode scale per element
    b = np.abs(x).reshape(R, kv, 16).max(axis=2)
    # zero-amax blocks: scale byte 0 and every code a (signed) zero
    zb = np.repeat(b == 0, 16, axis=1)
    assert np.all(sf_lin.reshape(R, kv)[b == 0] == 0)
    assert np.all(qv[zb] == 0)
    # dequantization bound: |x/sc - q| <= half the e2m1 step at |x/sc|, plus
    # whatever lies beyond the saturation point 6
    live = sc > 0
    y = np.zeros_like(x)
    y[live] = x[live] / sc[live]
    ay = np.abs(y)
    half = np.where(ay < 2, 0.25, np.where(ay < 4, 0.5, 1.0))
    excess = np.maximum(ay - 6.0, 0)
    err = np.abs(y - qv)
    assert np.all(err[live] <= (half + excess)[live] * (1 + 2.0 ** -18) + 1e-30)
    # a normal e4m3 block scale rounds b / (6 g) to within 2^-4 relative, so
    # nothing in such a block saturates by more than that (subnormal scales
    # are coarser and may clip more)
    normal = live & (np.repeat(s, 16, axis=1) >= 2.0 ** -6)
    assert np.all(ay[normal] <= 6.0 * (1 + 2.0 ** -3))
    # blocks with a zero scale but non-zero amax are tiny relative to A
    tiny = (sf_lin.reshape(R, kv) == 0) & (b > 0)
    if tiny.any():
        rr = np.nonzero(tiny)[0]
        assert np.all(b[tiny] * 448.0 / np.asarray(A_rows, dtype=np.float64)[rr] < 2.0 ** -9)
    # sign carried
    assert np.array_equal(codes >= 8, np.signbit(x))
    return s, b


@pytest.mark.parametrize("layout", [oracle.LINEAR, oracle.SWIZZLED])
def test_nvfp4_per_tensor_compute_bounds(layout):
    xb = synth.bf16_bits(synth.blockwise_scaled((80, 192), 16, seed=2, lo=-12, hi=4))
    q, sf, amax = oracle.quantize_nvfp4(xb, layout, oracle.NVFP4_PER_TENSOR_COMPUTE)
    A = np.abs(fvals(xb)).max()
    assert amax[0] == np.float32(A)
    lin = sf if layout == oracle.LINEAR else oracle.unswizzle(sf, 80, 12)
    s, b = check_nvfp4(xb, q, lin, np.full(80, A))
    # the block holding the tensor amax gets the largest scale, 448
    assert np.all(s[b == A] == 448.0)


def test_nvfp4_given_equals_compute():
    xb = synth.bf16_bits(synth.normal_bf16((32, 128), seed=8))
    q1, s1, a1 = oracle.quantize_nvfp4(xb, oracle.SWIZZLED, oracle.NVFP4_PER_TENSOR_COMPUTE)
    q2, s2, a2 = oracle.quantize_nvfp4(xb, oracle.SWIZZLED, oracle.NVFP4_PER_TENSOR_GIVEN, float(a1[0]))
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


def test_nvfp4_per_row_bounds_and_amax():
    xb = synth.bf16_bits(synth.split_activation(tokens=96, hidden=256, seed=5))
    q, sf, amax = oracle.quantize_nvfp4(xb, oracle.LINEAR, oracle.NVFP4_PER_ROW)
    A = np.abs(fvals(xb)).max(axis=1).astype(np.float32)
    assert np.array_equal(amax, A)
    s, b = check_nvfp4(xb, q, sf, A)
    assert np.all(s[b == A[:, None]] == 448.0)


def test_nvfp4_random_bits_bounds():
    xb = synth.bf16_bits(synth.random_finite_bf16((48, 64), seed=12))
    # keep amax where the encode scale is finite (A >= 2^-100)
    x = fvals(xb)
    keep = np.abs(x).max(axis=1) >= 2.0 ** -100
    xb = np.ascontiguousarray(xb[keep])
    q, sf, amax = oracle.quantize_nvfp4(xb, oracle.LINEAR, oracle.NVFP4_PER_ROW)
    check_nvfp4(xb, q, sf, amax)


def test_nvfp4_all_zero_tensor():
    xb = np.zeros((4, 32), dtype=np.uint16)
    xb[2, 5] = 0x8000
    q, sf, amax = oracle.quantize_nvfp4(xb, oracle.LINEAR, oracle.NVFP4_PER_TENSOR_COMPUTE)
    assert amax[0] == 0 and np.all(sf == 0)
    codes = unpack(q)
    assert codes[2, 5] == 8 and np.count_nonzero(codes) == 1


def test_nvfp4_zero_block_in_live_tensor():
    xb = synth.bf16_bits(synth.normal_bf16((2, 64), seed=1)).copy()
    xb[0, 16:32] = 0
    q, sf, amax = oracle.quantize_nvfp4(xb, oracle.LINEAR, oracle.NVFP4_PER_ROW)
    assert sf[1] == 0 and np.all(q[0, 8:16] == 0)


def test_nvfp4_split_equals_per_expert():
    """Row scaling: quantizing the concatenated activation and cutting it by
    expert equals quantizing each expert's rows (linear layout)."""
    xb = synth.bf16_bits(synth.split_activation(tokens=200, hidden=128, seed=6))
    counts = synth.dirichlet_splits(tokens=200, experts=8, alpha=0.3, seed=6, force_empty=(3,))
    qa, sfa, aa = oracle.quantize_nvfp4(xb, oracle.LINEAR, oracle.NVFP4_PER_ROW)
    off = 0
    for c in counts:
        q, sf, a = oracle.quantize_nvfp4(xb[off:off + c], oracle.LINEAR, oracle.NVFP4_PER_ROW)
        assert np.array_equal(q, qa[off:off + c])
        assert np.array_equal(sf, sfa[off * 8:(off + c) * 8])
        assert np.array_equal(a, aa[off:off + c])
        off += c


def test_nvfp4_packing_low_nibble_first(olib):
    xb = np.zeros((1, 16), dtype=np.uint16)
    vals = np.array([6, 1, -2, 0.5] + [0] * 12, dtype=np.float32)
    xb[0] = (vals.view(np.uint32) >> 16).astype(np.uint16)
    q, sf, amax = oracle.quantize_nvfp4(xb, oracle.LINEAR, oracle.NVFP4_PER_TENSOR_GIVEN, 6.0 * 448)
    # A = 2688 -> g = 1, S = 1; block amax 6 -> v = 1 -> scale 1.0 (0x38)
    assert sf[0] == 0x38
    assert q[0, 0] == (0x7 | (0x2 << 4)) and q[0, 1] == (0xC | (0x1 << 4))


# ---------------------------------------------------------------------------
# rounding order of the two-level scale (readings R2, R3, R4), hand-worked
# cases in tests/golden/nvfp4_rounding_order.txt
# ---------------------------------------------------------------------------

from fractions import Fraction  # noqa: E402
import struct  # noqa: E402


def _bf16(bits):
    return Fraction(struct.unpack("<f", struct.pack("<I", int(bits) << 16))[0])


def _rn32(q):
    """Exact rational -> nearest binary32 (ties to even), as a rational."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (max(e, -126) - 23)
    n = a / ulp
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * ulp


def _nearest(table, v):
    """Index of the nearest table value to v >= 0, ties to the even index
    (the even code; values beyond the last entry saturate to it)."""
    v = min(v, table[-1])
    best = None
    for i, t in enumerate(table):
        d = abs(t - v)
        if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
            best = (d, i)
    return best[1]


_E4M3 = [Fraction(c & 7, 8) * Fraction(2) ** -6 if c >> 3 == 0 else (1 + Fraction(c & 7, 8)) * Fraction(2) ** ((c >> 3) - 7)
         for c in range(0x7F)]
_E2M1 = [Fraction(v) for v in ("0", "1/2", "1", "3/2", "2", "3", "4", "6")]


def _e2m1(v):
    return (8 if v < 0 else 0) | _nearest(_E2M1, abs(v))


def _worked_row(elems, encode, block, rcp):
    """The row's scale bytes and payload by the given orders of rounding."""
    xs = [_bf16(b) for b in elems]
    A = max(abs(v) for v in xs)
    S = encode(A)
    sf, codes = [], []
    for k in range(len(xs) // 16):
        blk = xs[16 * k:16 * k + 16]
        b = max(abs(v) for v in blk)
        s = _nearest(_E4M3, block(b, S)) if b else 0
        r = rcp(S, _E4M3[s]) if s else Fraction(0)
        sf.append(s)
        codes += [_e2m1(_rn32(v * r)) for v in blk]
    return A, sf, bytes(codes[2 * j] | (codes[2 * j + 1] << 4) for j in range(len(codes) // 2))


_READING = dict(encode=lambda A: _rn32(1 / _rn32(A / 2688)),                 # R2
                block=lambda b, S: _rn32(_rn32(b / 6) * S),                   # R3
                rcp=lambda S, m: _rn32(S / m))                                # R4
_OTHER = {"encode_order": dict(_READING, encode=lambda A: _rn32(Fraction(2688) / A)),
          "block_order": dict(_READING, block=lambda b, S: _rn32(_rn32(b * S) / 6)),
          "rcp_order": dict(_READING, rcp=lambda S, m: _rn32(S * _rn32(1 / m)))}
_ORDER_CASES = rows("nvfp4_rounding_order.txt")


def _order_row(case):
    name, e0, e16, e17 = case[:4]
    elems = [0] * 32
    elems[0], elems[16], elems[17] = int(e0, 16), int(e16, 16), int(e17, 16)
    return name, elems


@pytest.mark.parametrize("case", _ORDER_CASES, ids=[c[0] for c in _ORDER_CASES])
def test_rounding_order_golden_is_worked_right(case):
    """The golden's bytes follow from readings R2-R4 in exact arithmetic, and
    the alternative order the case was built for gives other bytes."""
    name, elems = _order_row(case)
    A, sf, q = _worked_row(elems, **_READING)
    assert float(A).hex() == case[4]
    assert sf == [int(case[5], 16), int(case[6], 16)]
    assert q.hex().upper() == case[7]
    _, sf_alt, q_alt = _worked_row(elems, **_OTHER[name])
    assert (sf_alt, q_alt) != (sf, q)


@pytest.mark.parametrize("mode", [oracle.NVFP4_PER_TENSOR_COMPUTE, oracle.NVFP4_PER_ROW])
@pytest.mark.parametrize("case", _ORDER_CASES, ids=[c[0] for c in _ORDER_CASES])
def test_rounding_order_golden(case, mode):
    """The oracle takes its binary32 roundings in the order of R2-R4."""
    _, elems = _order_row(case)
    xb = np.array([elems], dtype=np.uint16)
    q, sf, amax = oracle.quantize_nvfp4(xb, oracle.LINEAR, mode)
    assert float(amax[0]).hex() == case[4]
    assert list(sf) == [int(case[5], 16), int(case[6], 16)]
    assert q[0].tobytes().hex().upper() == case[7]
