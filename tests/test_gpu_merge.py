"""GPU checks of the attention decode merge with its MXFP8 form
(qz_attention_merge_quantize) and of the public device functions of
include/qz_quant.cuh.  The merged bf16 output is within one bf16 ulp of the
oracle's binary64 merge (both accumulate in binary64, but the device exp and
the host exp may differ in their last bits, which can move a result that lies
next to a bf16 rounding boundary); its MXFP8
payload and scales equal the oracle quantizer applied to the GPU's own bf16
output, byte for byte, padded scale rows included.  The device functions are
compiled here into a small test kernel and must match the oracle quantizers."""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import assert_bytes_equal, host_bits

pytestmark = pytest.mark.gpu

qz = pytest.importorskip("nvfp4_quantization_moe_b200")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def bf16_ulps(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in bf16 steps between bf16 bit patterns (sign-magnitude order)."""
    def key(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, -(u & 0x7FFF), u)
    return np.abs(key(a) - key(b))


def run_merge(O, lse, layout, quantize=True):
    S, T, H = O.shape
    Od = torch.from_numpy(O).cuda()
    ld = torch.from_numpy(lse).cuda()
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    q = sf = None
    if quantize:
        q = torch.full((T, H), 0xA5, dtype=torch.uint8, device="cuda")
        sf = torch.full((max(qz.sf_bytes(T, H, qz.FMT_MXFP8, layout), 16),), 0xA5, dtype=torch.uint8, device="cuda")
    qz.attention_merge_quantize(Od, ld, y, q, sf, layout)
    torch.cuda.synchronize()
    return y, q, sf


@pytest.mark.parametrize("layout", [qz.SF_LINEAR, qz.SF_SWIZZLED])
@pytest.mark.parametrize("S,T,H", [(1, 1, 128), (4, 3, 7168), (16, 130, 1024), (8, 64, 2048), (3, 257, 512)])
def test_merge_and_mxfp8(S, T, H, layout):
    O, lse = synth.merge_partials(S, T, H, seed=S * 1000 + T)
    y, q, sf = run_merge(O, lse, layout)
    gy = host_bits(y)
    ref = oracle.attention_merge(O, lse)
    d = bf16_ulps(gy, ref)
    assert d.max() <= 1, f"merge off by {d.max()} bf16 ulps"
    assert np.mean(d) < 0.01
    rq, rsf = oracle.quantize_mxfp8(gy, layout)          # the oracle quantizer on the GPU's own output
    assert_bytes_equal(q.cpu().numpy(), rq, "payload")
    n = qz.sf_bytes(T, H, qz.FMT_MXFP8, layout)
    assert_bytes_equal(sf.cpu().numpy()[:n], rsf, "scale factors (padded rows included)")


def test_merge_without_quantized_form():
    O, lse = synth.merge_partials(5, 7, 1024, seed=77)
    y, _, _ = run_merge(O, lse, qz.SF_SWIZZLED, quantize=False)
    assert bf16_ulps(host_bits(y), oracle.attention_merge(O, lse)).max() <= 1


DEMO = r"""
#include "qz_quant.cuh"
__global__ void k_mx(const uint32_t* x, int64_t n_blocks, uint32_t* q, uint8_t* sf) {
    const int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= n_blocks) return;
    uint32_t w[16], c[8];
    for (int i = 0; i < 16; ++i) w[i] = x[b * 16 + i];
    sf[b] = (uint8_t)qzq::mxfp8_block(w, c);
    for (int i = 0; i < 8; ++i) q[b * 8 + i] = c[i];
}
__global__ void k_nv(const uint32_t* x, int64_t n_blocks, float amax, uint32_t* q, uint8_t* sf) {
    const int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= n_blocks) return;
    uint32_t w[8], c[2];
    for (int i = 0; i < 8; ++i) w[i] = x[b * 8 + i];
    sf[b] = (uint8_t)qzq::nvfp4_block(w, qzq::nvfp4_encode_scale(amax), c);
    q[b * 2] = c[0];
    q[b * 2 + 1] = c[1];
}
extern "C" int run_mx(const void* x, long long n, void* q, void* sf) {
    k_mx<<<(unsigned)((n + 127) / 128), 128>>>((const uint32_t*)x, n, (uint32_t*)q, (uint8_t*)sf);
    return (int)cudaDeviceSynchronize();
}
extern "C" int run_nv(const void* x, long long n, float amax, void* q, void* sf) {
    k_nv<<<(unsigned)((n + 127) / 128), 128>>>((const uint32_t*)x, n, amax, (uint32_t*)q, (uint8_t*)sf);
    return (int)cudaDeviceSynchronize();
}
"""


@pytest.fixture(scope="module")
def demo_lib():
    d = tempfile.mkdtemp(prefix="qz_demo_")
    src = os.path.join(d, "demo.cu")
    with open(src, "w") as f:
        f.write(DEMO)
    so = os.path.join(d, "demo.so")
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-fmad=false",
                    "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"), "-o", so, src], check=True)
    lib = ctypes.CDLL(so)
    lib.run_mx.argtypes = [ctypes.c_void_p, ctypes.c_longlong, ctypes.c_void_p, ctypes.c_void_p]
    lib.run_nv.argtypes = [ctypes.c_void_p, ctypes.c_longlong, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]
    return lib


def test_device_functions_match_the_quantizers(demo_lib):
    x = synth.blockwise_scaled((96, 512), 16, seed=31, lo=-30, hi=10)
    xb = host_bits(x)
    xd = x.cuda().contiguous()
    R, C = xb.shape
    q = torch.zeros((R, C), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((R * C // 32,), dtype=torch.uint8, device="cuda")
    assert demo_lib.run_mx(xd.data_ptr(), R * C // 32, q.data_ptr(), sf.data_ptr()) == 0
    rq, rsf = oracle.quantize_mxfp8(xb, oracle.LINEAR)
    assert_bytes_equal(q.cpu().numpy(), rq, "mxfp8_block payload")
    assert_bytes_equal(sf.cpu().numpy(), rsf, "mxfp8_block scales")
    amax = float(np.abs((xb.astype(np.uint32) << 16).view(np.float32)).max())
    q4 = torch.zeros((R, C // 2), dtype=torch.uint8, device="cuda")
    sf4 = torch.zeros((R * C // 16,), dtype=torch.uint8, device="cuda")
    assert demo_lib.run_nv(xd.data_ptr(), R * C // 16, amax, q4.data_ptr(), sf4.data_ptr()) == 0
    rq4, rsf4, _ = oracle.quantize_nvfp4(xb, oracle.LINEAR, oracle.NVFP4_PER_TENSOR_GIVEN, amax)
    assert_bytes_equal(q4.cpu().numpy(), rq4, "nvfp4_block payload")
    assert_bytes_equal(sf4.cpu().numpy(), rsf4, "nvfp4_block scales")
