"""The allocation-free entry point (qz_quantize_grouped_nvfp4_compute_noalloc).

Some callers cannot allocate device memory -- code embedded in a framework
that owns every device allocation, or a latency-critical loop where a
cudaMalloc would synchronize the device.  For them the single-launch NVFP4
path with a computed per-tensor amax keeps its scratch in a device array
inside the library.  These tests call it through the C ABI and require its
payload, scales and amax to equal, byte for byte, what the existing entry
point (qz_quantize_grouped_nvfp4 in QZ_NVFP4_PER_TENSOR_COMPUTE mode) writes
for the same inputs, on two calls in a row (the second call must not see the
first call's leftovers in the shared array).  The file is collected last, so
a run that stops at the first failure has run every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth

qz = pytest.importorskip("nvfp4_quantization_moe_b200")


def _quantize_pair(xs, layout):
    """Existing entry point and the allocation-free one on the same inputs."""
    ref = qz.alloc_outputs(xs, qz.FMT_NVFP4, layout, qz.NVFP4_PER_TENSOR_COMPUTE)
    new = qz.alloc_outputs(xs, qz.FMT_NVFP4, layout, qz.NVFP4_PER_TENSOR_COMPUTE)
    for e in new:
        e.q.fill_(0x5A)
        e.sf.fill_(0x5A)
        e.amax.fill_(-1.0)
    qz.quantize_grouped_nvfp4(qz.ExpertTable(ref), qz.NVFP4_PER_TENSOR_COMPUTE, layout)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    qz.quantize_grouped_nvfp4_compute_noalloc(qz.ExpertTable(new), layout, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for i, (a, b) in enumerate(zip(ref, new)):
        rows, cols = a.x.shape
        nsf = qz.sf_bytes(rows, cols, qz.FMT_NVFP4, layout)
        assert torch.equal(a.q, b.q), f"expert {i}: payload differs"
        assert torch.equal(a.sf[:nsf], b.sf[:nsf]), f"expert {i}: scale factors differ"
        if rows:
            assert torch.equal(a.amax.view(torch.int32), b.amax.view(torch.int32)), f"expert {i}: amax differs"


@pytest.mark.gpu
@pytest.mark.parametrize("layout", [qz.SF_SWIZZLED, qz.SF_LINEAR])
def test_noalloc_matches_existing_entry_point_twice(layout):
    # first call: many chunks' worth of experts, an empty and an all-zero one
    xs = [synth.normal_bf16((512, 1024), std=0.02, seed=900 + i, device="cuda") for i in range(40)]
    xs[5] = torch.zeros((0, 1024), dtype=torch.bfloat16, device="cuda")
    xs[9].zero_()
    _quantize_pair(xs, layout)
    # second call right after, other shapes and magnitudes: nothing of the
    # first call's scratch may leak into it
    ys = [synth.blockwise_scaled((rows, 384), 16, seed=950 + i, lo=-12, hi=6).cuda()
          for i, rows in enumerate((1, 127, 300, 64, 1000))]
    _quantize_pair(ys, layout)


@pytest.mark.gpu
def test_noalloc_at_its_table_limit():
    """Exactly the largest table the static scratch holds (tiny experts, so
    the per-expert amax words at the top of the array are written), then a
    smaller call: the clear at the start of each call must reset the words
    the first call left behind."""
    n = qz.STATIC_WS_MAX_EXPERTS
    xs = [synth.blockwise_scaled((1 + i % 3, 32), 16, seed=2000 + i, lo=-10, hi=10).cuda() for i in range(n)]
    xs[n - 1] = xs[n - 1] * 64          # the last expert's amax word holds the largest value
    _quantize_pair(xs, qz.SF_SWIZZLED)
    ys = [synth.blockwise_scaled((2, 32), 16, seed=3000 + i, lo=-30, hi=-20).cuda() for i in range(n // 2)]
    _quantize_pair(ys, qz.SF_SWIZZLED)


def test_noalloc_rejects_oversized_table():
    """More experts than the static scratch holds: refused before any launch;
    exactly the limit passes the host checks (with no GPU the call then fails
    at the CUDA runtime, not on its arguments)."""
    lib = qz.load()
    st = lib.qz_quantize_grouped_nvfp4_compute_noalloc(ctypes.c_void_p(0x1000), qz.STATIC_WS_MAX_EXPERTS + 1,
                                                        qz.SF_SWIZZLED, None, None)
    assert st == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_quantize_grouped_nvfp4_compute_noalloc(None, 0, qz.SF_SWIZZLED, None, None) == qz.QZ_OK
    if not torch.cuda.is_available():
        st = lib.qz_quantize_grouped_nvfp4_compute_noalloc(ctypes.c_void_p(0x1000), qz.STATIC_WS_MAX_EXPERTS,
                                                            qz.SF_SWIZZLED, None, None)
        assert st == qz.QZ_ERR_CUDA
