/*
 * qz_quant.cuh -- device functions for producer kernels that emit MXFP8 /
 * NVFP4 directly from registers (sm_100a, CUDA C++).
 *
 * TensorRT-LLM "MXFP8 carrier and quantize folds": a standalone quantize
 * kernel re-reads from HBM what the producing kernel held in registers
 * (commit 1); a function the producer calls on the tile it holds writes the
 * quantized form alongside its normal output, bit for bit what the
 * standalone quantizer writes, flush-to-zero of the block scale's reciprocal
 * included (commit 2); and the producer can also write the scale-factor rows
 * that the swizzled layout invents past the last live row (commit 3).
 *
 * These are the library's own block quantizers (the grouped kernels in
 * libqz.so use the same code), so a producer calling them matches
 * qz_quantize_grouped_mxfp8 / qz_quantize_grouped_nvfp4 byte for byte.
 * Element order: element 0 of a block is the low half of the first bf16x2
 * word; codes are returned element 0 first (low byte for e4m3, low nibble
 * for e2m1).  Scale bytes go where sf_offset says, in the layout of
 * include/qz.h (QZ_SF_LINEAR or QZ_SF_SWIZZLED_128x4).
 */
#pragma once

#include "qz.h"
#include "../nvfp4_quantization_moe_b200/csrc/qz_device.cuh"

namespace qzq {

/* MXFP8: one 32-element block held by one thread (x: 16 bf16x2 words).
 * Returns the E8M0 byte; q receives the 32 e4m3 codes (8 words). */
__device__ __forceinline__ uint32_t mxfp8_block(const uint32_t (&x)[16], uint32_t (&q)[8]) {
    const uint32_t scale = qz::e8m0_byte(qz::absmax_words<16>(x));
    const float r = qz::e8m0_reciprocal(scale);
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = qz::e4m3x4_words(x[2 * i], x[2 * i + 1], r);
    return scale;
}

/* MXFP8: one 32-element block spread over four consecutive lanes 4j..4j+3,
 * each holding 8 consecutive elements (x: 4 bf16x2 words; lane 4j has
 * elements 0-7).  Every lane of the warp must call it (full-warp shuffles).
 * Returns the block's E8M0 byte in all four lanes; q receives the lane's 8
 * e4m3 codes (2 words). */
__device__ __forceinline__ uint32_t mxfp8_block_x4(const uint32_t (&x)[4], uint32_t (&q)[2]) {
    uint32_t m = qz::absmax_words<4>(x);
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    const uint32_t scale = qz::e8m0_byte(m);
    const float r = qz::e8m0_reciprocal(scale);
    q[0] = qz::e4m3x4_words(x[0], x[1], r);
    q[1] = qz::e4m3x4_words(x[2], x[3], r);
    return scale;
}

/* NVFP4: the encode scale S = RN(1 / RN(amax / 2688)) of a tensor (or row)
 * amax, 0 when the decode scale is 0. */
__device__ __forceinline__ float nvfp4_encode_scale(float amax) { return qz::nvfp4_encode_scale(amax); }

/* NVFP4: one 16-element block held by one thread (x: 8 bf16x2 words) with
 * encode scale S.  Returns the E4M3 scale code; q receives the 16 packed e2m1
 * codes (2 words). */
__device__ __forceinline__ uint32_t nvfp4_block(const uint32_t (&x)[8], float S, uint32_t (&q)[2]) {
    const float b = qz::bits_to_float_bf16(qz::absmax_words<8>(x));
    const uint32_t s = (b == 0.0f) ? 0u : qz::e4m3_of(__fmul_rn(qz::div6_rn(b), S));
    float rcp = 0.0f;
    if (s != 0u) {
        // RN(S / value(s)) as the library computes it: value(s) = m * 2^k,
        // RN(S / m) by the quotient correction with c = RN(1 / m), then 2^-k
        const uint32_t ef = s >> 3;
        const uint32_t m = ef ? ((s & 7u) | 8u) : s;
        const float c = __frcp_rn((float)m);
        const float q0 = __fmul_rn(S, c);
        const float r = __fmaf_rn(-q0, (float)m, S);
        const float qm = __fmaf_rn(r, c, q0);
        rcp = __fmul_rn(qm, __uint_as_float((137u - max(ef, 1u)) << 23));
        if (rcp < 0x1p-126f) rcp = 0.0f;  // flush a subnormal multiplier to zero
    }
    q[0] = qz::e2m1x8_words(x[0], x[1], x[2], x[3], rcp);
    q[1] = qz::e2m1x8_words(x[4], x[5], x[6], x[7], rcp);
    return s;
}

/* Byte offset of scale (row, k) in an expert's SF region with kv scale
 * columns (layout QZ_SF_LINEAR or QZ_SF_SWIZZLED_128x4). */
__device__ __forceinline__ int64_t sf_offset(int64_t row, int64_t k, int64_t kv, int layout) {
    return layout == QZ_SF_SWIZZLED_128x4 ? qz::swz_offset(row, k, kv) : row * kv + k;
}

/* Rows of the swizzled region past the last live row (they must read as
 * 0x00): pad(rows, 128) - rows. */
__device__ __forceinline__ int64_t sf_padded_rows(int64_t rows) { return ((rows + 127) & ~(int64_t)127) - rows; }

}  // namespace qzq
