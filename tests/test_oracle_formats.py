"""Pins of the oracle's number formats (e4m3, e2m1, bf16) against things other
than the oracle: torch's float8 / bfloat16 conversions, brute-force nearest
search over the code tables, and hand-worked fixtures from the OCP MX spec."""
import math
import struct

import numpy as np
import pytest
import torch

from golden_io import rows


def f32(v):
    return struct.unpack("<f", struct.pack("<f", v))[0]


def e4m3_table_from_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_matches_torch(olib):
    t = e4m3_table_from_torch()
    for c in range(256):
        v = olib.qzo_e4m3_value(c)
        if c in (0x7F, 0xFF):
            assert math.isnan(v) and math.isnan(t[c])
        else:
            assert v == t[c] and math.copysign(1, v) == math.copysign(1, t[c]), c


def test_e4m3_golden_values(olib):
    for code, val in rows("e4m3_values.txt"):
        c = int(code, 16)
        v = float(val)
        assert olib.qzo_e4m3_value(c) == v
        assert math.copysign(1, olib.qzo_e4m3_value(c)) == math.copysign(1, v)
        assert olib.qzo_e4m3_encode(v) == c


def _probe_values_e4m3():
    t = e4m3_table_from_torch()
    pos = np.sort(np.unique(t[np.isfinite(t) & (t >= 0)]))
    mids = (pos[1:] + pos[:-1]) / 2
    vals = [pos, mids]
    for m in mids:
        a = np.float32(m)
        vals.append(np.array([np.nextafter(a, np.float32(0)), np.nextafter(a, np.float32(1e9))], dtype=np.float64))
    rng = np.random.default_rng(7)
    vals.append(np.exp2(rng.uniform(-13, 9, 20000)).astype(np.float32).astype(np.float64))
    v = np.concatenate(vals).astype(np.float32)
    return np.concatenate([v, -v])


def test_e4m3_encode_matches_torch_in_range(olib):
    v = _probe_values_e4m3()
    v = v[np.abs(v) <= 464.0]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([olib.qzo_e4m3_encode(float(a)) for a in v], dtype=np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(v[i]), int(got[i]), int(ref[i])) for i in bad[:10]]


def test_e4m3_encode_bruteforce_nearest_even(olib):
    """Nearest code by exhaustive search, ties to the code with mantissa LSB 0,
    magnitudes above 448 saturate to 448."""
    t = e4m3_table_from_torch()
    cand = [c for c in range(128) if np.isfinite(t[c])]
    cv = np.array([t[c] for c in cand])
    v = _probe_values_e4m3()
    v = np.concatenate([v, np.array([449, 463.9, 464, 470, 1e6, 3e38, -500], dtype=np.float32)])
    for a in v:
        mag = min(abs(float(a)), 448.0)
        d = np.abs(cv - mag)
        best = np.nonzero(d == d.min())[0]
        if len(best) > 1:
            best = [b for b in best if cand[b] % 2 == 0]
        code = cand[best[0]] | (0x80 if math.copysign(1, float(a)) < 0 else 0)
        assert olib.qzo_e4m3_encode(float(a)) == code, (float(a), code)


def test_e4m3_saturation_and_signed_zero(olib):
    assert olib.qzo_e4m3_encode(1e30) == 0x7E
    assert olib.qzo_e4m3_encode(-1e30) == 0xFE
    assert olib.qzo_e4m3_encode(470.0) == 0x7E
    assert olib.qzo_e4m3_encode(-0.0) == 0x80
    assert olib.qzo_e4m3_encode(0.0) == 0x00
    assert olib.qzo_e4m3_encode(-(2.0 ** -11)) == 0x80
    assert olib.qzo_e4m3_encode(2.0 ** -10) == 0x00          # tie -> even (0)
    assert olib.qzo_e4m3_encode(3 * 2.0 ** -10) == 0x02      # tie 1.5 ulp -> even (2)


def test_e2m1_values_golden(olib):
    for code, val in rows("e2m1_values.txt"):
        v = float(val)
        got = olib.qzo_e2m1_value(int(code))
        assert got == v and math.copysign(1, got) == math.copysign(1, v)


def test_e2m1_rounding_golden(olib):
    for val, code in rows("e2m1_rounding.txt"):
        assert olib.qzo_e2m1_encode(float(val)) == int(code), val


def test_e2m1_encode_bruteforce(olib):
    table = {int(c): float(v) for c, v in rows("e2m1_values.txt")}
    mags = [table[c] for c in range(8)]
    rng = np.random.default_rng(11)
    probe = list(rng.uniform(-8, 8, 20000).astype(np.float32))
    for a, b in zip(mags[:-1], mags[1:]):
        m = np.float32((a + b) / 2)
        probe += [m, np.nextafter(m, np.float32(-1)), np.nextafter(m, np.float32(9))]
    for x in probe:
        mag = min(abs(float(x)), 6.0)
        d = np.abs(np.array(mags) - mag)
        best = np.nonzero(d == d.min())[0]
        if len(best) > 1:
            best = [b for b in best if b % 2 == 0]
        code = int(best[0]) | (8 if math.copysign(1, float(x)) < 0 else 0)
        assert olib.qzo_e2m1_encode(float(x)) == code, float(x)


def test_bf16_value_matches_torch(olib):
    bits = np.arange(0, 1 << 16, 97, dtype=np.int64).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    for b, r in zip(bits, ref):
        v = olib.qzo_bf16_value(int(b))
        assert (v == r) or (math.isnan(v) and math.isnan(r))


def test_bf16_rounding_matches_torch_on_float_inputs(olib):
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(20000) * np.exp2(rng.uniform(-130, 120, 20000)),
                        rng.standard_normal(2000)]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([olib.qzo_bf16_from_double(float(a)) for a in v], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_rounding_single_rounding_from_double(olib):
    # 1 + 2^-8 + 2^-40 lies above the tie 1 + 2^-8, so it rounds up to 1 + 2^-7
    # (a detour through binary32 would drop 2^-40 and round to even, 1.0).
    assert olib.qzo_bf16_from_double(1 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    assert olib.qzo_bf16_from_double(1 + 2.0 ** -8) == 0x3F80
    assert olib.qzo_bf16_from_double(-(1 + 3 * 2.0 ** -8)) == 0xBF82
