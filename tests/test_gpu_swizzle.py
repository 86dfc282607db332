"""GPU parity of the standalone linear -> swizzled 128x4 conversion, and the
external pin of the oracle's layouts and encodings: cuBLAS's block-scaled
GEMM (through torch._scaled_mm) fed with ORACLE-produced MXFP8 / NVFP4
operands must equal the binary64 product of the oracle-dequantized operands."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import Guarded, assert_bytes_equal, host_bits

pytestmark = pytest.mark.gpu

qz = pytest.importorskip("nvfp4_quantization_moe_b200")


def test_swizzle_kernel_matches_oracle():
    rng = np.random.default_rng(0)
    shapes = [(1, 1), (5, 3), (127, 8), (128, 4), (129, 6), (300, 64), (1536, 64), (0, 8), (2048, 24)]
    pairs, keep, lin_host = [], [], []
    for rows, kv in shapes:
        lin = rng.integers(0, 256, rows * kv, dtype=np.uint8)
        src = torch.from_numpy(lin).cuda() if lin.size else torch.empty(0, dtype=torch.uint8, device="cuda")
        dst = Guarded(oracle.sf_region_bytes(rows, kv, oracle.SWIZZLED))
        pairs.append((src if rows else None, dst.view if rows else None, rows, kv))
        keep.append((src, dst))
        lin_host.append(lin)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    qz.swizzle_scales(qz.SfPairTable(pairs, "cuda"), err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for (rows, kv), lin, (_, dst) in zip(shapes, lin_host, keep):
        assert dst.guards_intact()
        assert_bytes_equal(dst.host(), oracle.swizzle(lin, rows, kv), f"swizzle {rows}x{kv}")


def test_swizzle_of_grouped_linear_equals_grouped_swizzled():
    xs = [synth.normal_bf16((200, 768), seed=i).cuda() for i in range(3)]
    lin = qz.quantize_experts(xs, qz.FMT_MXFP8, qz.SF_LINEAR)
    swz = qz.quantize_experts(xs, qz.FMT_MXFP8, qz.SF_SWIZZLED)
    dsts = [torch.full((qz.sf_bytes(200, 768, 0, 1),), 0xEE, dtype=torch.uint8, device="cuda") for _ in xs]
    qz.swizzle_scales(qz.SfPairTable([(e.sf, d, 200, 24) for e, d in zip(lin, dsts)], "cuda"))
    torch.cuda.synchronize()
    for d, e in zip(dsts, swz):
        assert torch.equal(d, e.sf)


def _scaled_mm_or_skip(*args, **kw):
    try:
        return torch._scaled_mm(*args, **kw)
    except (RuntimeError, NotImplementedError, TypeError) as exc:  # pragma: no cover
        pytest.skip(f"block-scaled torch._scaled_mm unavailable here: {exc}")


def _e4m3(codes):
    return torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64)


def test_cublas_pins_oracle_mxfp8_layout():
    M, N, K = 256, 192, 512
    a = synth.normal_bf16((M, K), seed=1)
    b = synth.blockwise_scaled((N, K), 32, seed=2, lo=-6, hi=6)
    qa, sfa = oracle.quantize_mxfp8(synth.bf16_bits(a), oracle.SWIZZLED)
    qb, sfb = oracle.quantize_mxfp8(synth.bf16_bits(b), oracle.SWIZZLED)
    _, la = oracle.quantize_mxfp8(synth.bf16_bits(a), oracle.LINEAR)
    _, lb = oracle.quantize_mxfp8(synth.bf16_bits(b), oracle.LINEAR)
    deq_a = _e4m3(qa) * torch.exp2(torch.from_numpy(la.astype(np.float64) - 127).view(M, K // 32)).repeat_interleave(32, 1)
    deq_b = _e4m3(qb) * torch.exp2(torch.from_numpy(lb.astype(np.float64) - 127).view(N, K // 32)).repeat_interleave(32, 1)
    ref = deq_a @ deq_b.T
    A = torch.from_numpy(qa).cuda().view(torch.float8_e4m3fn)
    B = torch.from_numpy(qb).cuda().view(torch.float8_e4m3fn)
    SA = torch.from_numpy(sfa).cuda().view(torch.float8_e8m0fnu)
    SB = torch.from_numpy(sfb).cuda().view(torch.float8_e8m0fnu)
    out = _scaled_mm_or_skip(A, B.t(), SA, SB, out_dtype=torch.float32).double().cpu()
    scale = (deq_a.abs() @ deq_b.abs().T)
    assert torch.all((out - ref).abs() <= 1e-5 * scale + 1e-30), float(((out - ref).abs() / scale).max())


def test_cublas_pins_oracle_nvfp4_layout_and_nibbles():
    M, N, K = 128, 256, 256
    a = synth.normal_bf16((M, K), seed=3)
    b = synth.split_activation(tokens=N, hidden=K, seed=4)
    Aa = float(a.float().abs().max())
    Ab = float(b.float().abs().max())
    qa, sfa, _ = oracle.quantize_nvfp4(synth.bf16_bits(a), oracle.SWIZZLED, oracle.NVFP4_PER_TENSOR_GIVEN, Aa)
    qb, sfb, _ = oracle.quantize_nvfp4(synth.bf16_bits(b), oracle.SWIZZLED, oracle.NVFP4_PER_TENSOR_GIVEN, Ab)
    _, la, _ = oracle.quantize_nvfp4(synth.bf16_bits(a), oracle.LINEAR, oracle.NVFP4_PER_TENSOR_GIVEN, Aa)
    _, lb, _ = oracle.quantize_nvfp4(synth.bf16_bits(b), oracle.LINEAR, oracle.NVFP4_PER_TENSOR_GIVEN, Ab)
    e2m1 = torch.tensor([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6], dtype=torch.float64)

    def deq(q, lin, rows):
        codes = torch.from_numpy(np.stack([q & 0xF, q >> 4], axis=-1).reshape(rows, K).astype(np.int64))
        s = _e4m3(lin).view(rows, K // 16).repeat_interleave(16, 1)
        return e2m1[codes] * s

    ref = deq(qa, la, M) @ deq(qb, lb, N).T
    ga = float(np.float32(Aa) / np.float32(2688.0))
    gb = float(np.float32(Ab) / np.float32(2688.0))
    A = torch.from_numpy(qa).cuda().view(torch.float4_e2m1fn_x2)
    B = torch.from_numpy(qb).cuda().view(torch.float4_e2m1fn_x2)
    SA = torch.from_numpy(sfa).cuda().view(torch.float8_e4m3fn)
    SB = torch.from_numpy(sfb).cuda().view(torch.float8_e4m3fn)
    out = _scaled_mm_or_skip(A, B.t(), SA, SB, out_dtype=torch.float32).double().cpu()
    scale = deq(qa, la, M).abs() @ deq(qb, lb, N).abs().T
    assert torch.all((out - ref).abs() <= 1e-5 * scale + 1e-30), float(((out - ref).abs() / scale).max())
    # the decode scales complete the dequantization: out * ga * gb approximates a @ b.T
    approx = out * ga * gb
    exact = a.double() @ b.double().T
    rel = ((approx - exact).abs().sum() / exact.abs().sum()).item()
    assert rel < 0.2
