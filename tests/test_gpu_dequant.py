"""GPU parity of the grouped dequantization (qz_dequantize_grouped) against
the oracle's decoder: random payloads, scales and amax values from the seeded
generators (both formats, both layouts, per tensor and per row, ragged and
empty experts, strided outputs with canaries), the round trip through the
GPU quantizer, invalid entries, grid invariance and a Qwen3-30B-A3B gate_up
layer at full size."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import assert_bytes_equal, host_bits

pytestmark = pytest.mark.gpu

qz = pytest.importorskip("nvfp4_quantization_moe_b200")
LAYOUTS = [qz.SF_LINEAR, qz.SF_SWIZZLED]


def _dev_bytes(a: np.ndarray, extra: int = 0) -> torch.Tensor:
    """A 16-byte aligned device copy of a uint8 array (with `extra` spare bytes)."""
    flat = np.ascontiguousarray(a).reshape(-1)
    t = torch.zeros(max(flat.size + extra, 16), dtype=torch.uint8, device="cuda")
    if flat.size:
        t[:flat.size] = torch.from_numpy(flat).cuda()
    return t


def random_expert(rows, cols, fmt, layout, per_row, seed):
    block = 32 if fmt == qz.FMT_MXFP8 else 16
    q = synth.random_payload(rows, cols, fmt, seed)
    nsf = qz.sf_bytes(rows, cols, fmt, layout) if rows else 0
    sf = synth.random_scale_bytes(nsf, fmt, seed + 1)
    amax = synth.random_amax(rows if per_row else 1, seed + 2) if fmt == qz.FMT_NVFP4 else None
    return q, sf, amax, block


def run_dequant(experts, fmt, layout, per_row, ld_pad=0, err=None, max_ctas=0):
    entries, outs = [], []
    for q, sf, amax, rows, cols in experts:
        ys = torch.full((rows, cols + ld_pad + 16), -7.0, dtype=torch.bfloat16, device="cuda")  # canary columns
        y = ys[:, :cols]
        a = torch.from_numpy(amax).cuda() if amax is not None else None
        entries.append(qz.DqEntry(_dev_bytes(q), _dev_bytes(sf), y, a))
        outs.append(ys)
    qz.dequantize_grouped(qz.DqTable(entries, device=torch.device("cuda")), fmt, per_row, layout, err=err,
                          max_ctas=max_ctas)
    torch.cuda.synchronize()
    return outs


SHAPES = [(0, 64), (1, 64), (5, 96), (127, 160), (129, 128), (200, 416), (300, 2048)]


@pytest.mark.parametrize("per_row", [False, True])
@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("fmt", [qz.FMT_MXFP8, qz.FMT_NVFP4])
def test_random_codes(fmt, layout, per_row):
    if fmt == qz.FMT_MXFP8 and per_row:
        pytest.skip("per_row applies to NVFP4 only")
    experts = []
    for i, (rows, cols) in enumerate(SHAPES):
        q, sf, amax, _ = random_expert(rows, cols, fmt, layout, per_row, 300 + 7 * i)
        experts.append((q, sf, amax, rows, cols))
    outs = run_dequant(experts, fmt, layout, per_row, ld_pad=8)
    for i, ((q, sf, amax, rows, cols), ys) in enumerate(zip(experts, outs)):
        got = host_bits(ys)
        if fmt == qz.FMT_MXFP8:
            ref = oracle.dequantize_mxfp8(q, sf, layout)
        else:
            ref = oracle.dequantize_nvfp4(q, sf, amax, per_row, layout)
        assert_bytes_equal(got[:, :cols], ref, f"expert {i} ({rows}x{cols})")
        canary = host_bits(torch.full((1,), -7.0, dtype=torch.bfloat16))[0]
        assert np.all(got[:, cols:] == canary), f"expert {i}: write past the row"


@pytest.mark.parametrize("layout", LAYOUTS)
def test_round_trip_through_the_quantizer(layout):
    """GPU quantize then GPU dequantize equals the oracle's dequantization of
    the oracle's quantization of the same input."""
    xs = [synth.blockwise_scaled((130, 256), 32, seed=321, lo=-10, hi=10).cuda(),
          synth.normal_bf16((64, 512), 1.0, seed=322).cuda()]
    for fmt, mode in ((qz.FMT_MXFP8, None), (qz.FMT_NVFP4, qz.NVFP4_PER_ROW), (qz.FMT_NVFP4, qz.NVFP4_PER_TENSOR_COMPUTE)):
        ents = qz.alloc_outputs(xs, fmt, layout, mode if mode is not None else qz.NVFP4_PER_ROW)
        tab = qz.ExpertTable(ents)
        if fmt == qz.FMT_MXFP8:
            qz.quantize_grouped_mxfp8(tab, layout)
        else:
            qz.quantize_grouped_nvfp4(tab, mode, layout)
        ys = [torch.empty_like(x) for x in xs]
        per_row = mode == qz.NVFP4_PER_ROW
        qz.dequantize_grouped(qz.DqTable([qz.DqEntry(e.q, e.sf, y, e.amax) for e, y in zip(ents, ys)]), fmt,
                              per_row, layout)
        torch.cuda.synchronize()
        for i, (x, y) in enumerate(zip(xs, ys)):
            xb = host_bits(x)
            if fmt == qz.FMT_MXFP8:
                q, sf = oracle.quantize_mxfp8(xb, layout)
                ref = oracle.dequantize_mxfp8(q, sf, layout)
            else:
                q, sf, amax = oracle.quantize_nvfp4(xb, layout, mode)
                ref = oracle.dequantize_nvfp4(q, sf, amax, per_row, layout)
            assert_bytes_equal(host_bits(y), ref, f"fmt {fmt} mode {mode} expert {i}")


def test_invalid_entries_are_skipped_and_reported():
    q, sf, amax, _ = random_expert(64, 64, qz.FMT_NVFP4, qz.SF_LINEAR, False, 5)
    qd, sfd, ad = _dev_bytes(q), _dev_bytes(sf), torch.from_numpy(amax).cuda()
    y = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    bad_y = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    raw = [(qd.data_ptr(), sfd.data_ptr(), ad.data_ptr(), 64, 64, y.data_ptr(), 64),
           (qd.data_ptr(), sfd.data_ptr(), ad.data_ptr(), 64, 40, bad_y.data_ptr(), 64),      # cols % 16
           (qd.data_ptr(), sfd.data_ptr(), 0, 64, 64, bad_y.data_ptr(), 64),                  # amax NULL
           (qd.data_ptr(), sfd.data_ptr(), ad.data_ptr(), 64, 64, bad_y.data_ptr() + 2, 64)]  # y misaligned
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    qz.dequantize_grouped(qz.DqTable.from_raw(raw, "cuda"), qz.FMT_NVFP4, False, qz.SF_LINEAR, err=err)
    torch.cuda.synchronize()
    bits = int(err.item())
    assert bits & qz.DERR_SHAPE and bits & qz.DERR_NULL and bits & qz.DERR_ALIGN
    assert torch.count_nonzero(bad_y).item() == 0
    assert_bytes_equal(host_bits(y), oracle.dequantize_nvfp4(q, sf, amax, False, qz.SF_LINEAR), "valid entry")


@pytest.mark.parametrize("max_ctas", [1, 7, 148])
def test_grid_invariance(max_ctas):
    experts = []
    for i, (rows, cols) in enumerate([(257, 384), (3, 64), (128, 1024)]):
        q, sf, amax, _ = random_expert(rows, cols, qz.FMT_NVFP4, qz.SF_SWIZZLED, True, 900 + i)
        experts.append((q, sf, amax, rows, cols))
    outs = run_dequant(experts, qz.FMT_NVFP4, qz.SF_SWIZZLED, True, max_ctas=max_ctas)
    for i, ((q, sf, amax, rows, cols), ys) in enumerate(zip(experts, outs)):
        ref = oracle.dequantize_nvfp4(q, sf, amax, True, qz.SF_SWIZZLED)
        assert_bytes_equal(host_bits(ys)[:, :cols], ref, f"expert {i}")


@pytest.mark.parametrize("fmt", [qz.FMT_MXFP8, qz.FMT_NVFP4])
def test_qwen3_30b_gate_up_layer_sampled(fmt):
    """128 experts of [1536, 2048] in one call; every expert's rows 0, 777 and
    1535 against the oracle."""
    cfg = synth.QWEN3_30B
    rows, cols = cfg["gate_up"]
    n = cfg["experts"]
    experts = []
    for i in range(n):
        q, sf, amax, _ = random_expert(rows, cols, fmt, qz.SF_LINEAR, False, 5000 + 3 * i)
        experts.append((q, sf, amax, rows, cols))
    outs = run_dequant(experts, fmt, qz.SF_LINEAR, False)
    kv = cols // (32 if fmt == qz.FMT_MXFP8 else 16)
    for i, ((q, sf, amax, _, _), ys) in enumerate(zip(experts, outs)):
        got = host_bits(ys)
        for r in (0, 777, rows - 1):
            sfr = sf.reshape(rows, kv)[r:r + 1].reshape(-1)
            if fmt == qz.FMT_MXFP8:
                ref = oracle.dequantize_mxfp8(q[r:r + 1], sfr, qz.SF_LINEAR)
            else:
                ref = oracle.dequantize_nvfp4(q[r:r + 1], sfr, amax, False, qz.SF_LINEAR)
            assert_bytes_equal(got[r:r + 1, :cols], ref, f"expert {i} row {r}")


def _every_code_and_scale(amaxes, per_row):
    """Decode every e2m1 code under every finite E4M3 scale code for each amax
    A in `amaxes` (per row: A spread over [A/2, 2A] down the rows) and compare
    with the oracle's decoder; returns how many binary32 products landed on a
    bf16 midpoint."""
    scales = np.arange(127, dtype=np.uint8)
    R = len(scales)
    codes = np.arange(16, dtype=np.uint8)
    q = np.tile((codes[0::2] | (codes[1::2] << 4)).astype(np.uint8), (R, 1))
    e2m1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6], dtype=np.float32)
    e4m3 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    midpoints = 0
    for A in amaxes:
        amax = np.full(R if per_row else 1, A, dtype=np.float32)
        if per_row:
            amax = (amax * np.linspace(0.5, 2.0, R)).astype(np.float32)
        with np.errstate(over="ignore", under="ignore"):
            g = (amax / np.float32(2688.0)).astype(np.float32).reshape(-1, 1)
            prod = ((e2m1[None, :] * e4m3[scales][:, None]).astype(np.float32) * g).astype(np.float32)
        midpoints += int(np.count_nonzero((prod.view(np.uint32) & 0xFFFF) == 0x8000))
        out = run_dequant([(q, scales.copy(), amax, R, 16)], qz.FMT_NVFP4, qz.SF_LINEAR, per_row)[0]
        ref = oracle.dequantize_nvfp4(q, scales.copy(), amax, per_row, oracle.LINEAR)
        assert_bytes_equal(host_bits(out)[:, :16], ref, f"amax {A}")
    return midpoints


@pytest.mark.parametrize("per_row", [False, True])
def test_every_code_and_scale_at_extreme_amax(per_row):
    """Amax values whose decode scale is subnormal or whose products approach
    the binary32 overflow: the decoder builds these tables entry by entry (its
    two-product shortcut needs every entry normal and finite) and must still
    round each exact product once."""
    amaxes = (1e-36, 3e-37, 2e-38, 5e-39, 3e-40, 1e37, 8e37, 1.5e38)
    _every_code_and_scale(amaxes if per_row else amaxes + (3.3e38,), per_row)  # per row: up to 2A, finite


@pytest.mark.parametrize("per_row", [False, True])
def test_every_code_and_scale_including_midpoint_products(per_row):
    """Every e2m1 code under every finite E4M3 scale code, for amax values
    among which some binary32 products RN(value(q) * value(s) * g) land exactly
    on a bf16 midpoint (those elements need the exact product to round): the
    decoder must match the oracle there too."""
    midpoints = _every_code_and_scale((3.0, 1.0 / 3.0, 5.0e4, 27.50284194946289, 36.21154022216797, 76.34375),
                                      per_row)
    assert midpoints > 0, "no product fell on a bf16 midpoint: the exact-rounding path went untested"

