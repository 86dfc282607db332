// qz_rmsnorm.cu -- fused residual add + RMSNorm + MXFP8/NVFP4 quantize (sm_100a).
//
// TensorRT-LLM "NVFP4 linear-SF AllReduce epilogue" (commits 2 and 3) and
// "MXFP8 carrier and quantize folds" (commit 6): the epilogue that already
// holds the bf16 norm in registers emits its quantized form too, from the very
// bf16 values it stores to norm_out, so the result equals quantizing norm_out
// afterwards; the swizzled layout's invented rows are zeroed by the kernel.
//
// One 128-thread CTA per row.  Thread t holds chunks t + 128 i (8 bf16 each)
// of h = bf16(x + r) in registers between the two phases:
//   phase 1: load x, r; h; sum of h^2 (h^2 is exact in binary32; the sum is
//            compensated per thread and reduced across the CTA in binary64);
//   phase 2: rstd = 1 / sqrt(mean + eps) in binary64, split into two binary32
//            words; y = h * gamma * rstd rounded once to bf16 (the product
//            h * gamma is exact, the error of the final product is carried in
//            an FMA so the bf16 rounding sees the binary64-accurate value);
//            store y, then quantize y exactly like the grouped kernels.
// A block of 32 (MXFP8) or 16 (NVFP4) elements is 4 or 2 consecutive chunks,
// which sit in consecutive threads, so block amax is a butterfly shuffle.
#include "qz_device.cuh"

namespace qz {

constexpr int kNormThreads = 128;

// bf16 (nearest-even) of hi + e, where |e| <= half an ulp of hi: the rounding
// of hi decides unless hi sits exactly on a bf16 midpoint, where e breaks the tie.
__device__ __forceinline__ uint32_t bf16_rne_with_residue(float hi, float e) {
    const uint32_t b = __float_as_uint(hi);
    const uint32_t low = b & 0xFFFFu;
    uint32_t up;
    if (low == 0x8000u) {
        if (e == 0.0f) up = (b >> 16) & 1u;
        else up = ((e > 0.0f) == (hi > 0.0f)) ? 1u : 0u;
    } else {
        up = low > 0x8000u ? 1u : 0u;
    }
    return ((b >> 16) + up) & 0xFFFFu;
}

// bf16 of p * (rh + rl): p * rh exactly as hi + lo (FMA), plus p * rl.
__device__ __forceinline__ uint32_t bf16_scaled(float p, float rh, float rl) {
    const float hi = __fmul_rn(p, rh);
    float lo = __fmaf_rn(p, rh, -hi);
    lo = __fmaf_rn(p, rl, lo);
    const float s = __fadd_rn(hi, lo);
    const float e = __fsub_rn(lo, __fsub_rn(s, hi));
    return bf16_rne_with_residue(s, e);
}

// bf16 nearest-even of the exact sum a + b (TwoSum gives its binary32
// rounding and the error).
__device__ __forceinline__ uint32_t bf16_of_sum(float a, float b) {
    const float s = __fadd_rn(a, b);
    const float bp = __fsub_rn(s, a);
    const float e = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bp)), __fsub_rn(b, bp));
    return bf16_rne_with_residue(s, e);
}

__device__ __forceinline__ void two_sum_add(float& sh, float& sl, float t) {
    const float s = __fadd_rn(sh, t);
    const float bp = __fsub_rn(s, sh);
    const float err = __fadd_rn(__fsub_rn(sh, __fsub_rn(s, bp)), __fsub_rn(t, bp));
    sh = s;
    sl = __fadd_rn(sl, err);
}

template <int FMT, int LAYOUT, int CPT>
__global__ void __launch_bounds__(kNormThreads) rmsnorm_quant_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ res, const uint16_t* __restrict__ gamma, float eps,
    int64_t T, int64_t H, uint16_t* __restrict__ norm_out, uint16_t* __restrict__ res_out, uint8_t* __restrict__ q,
    uint8_t* __restrict__ sf, const float* __restrict__ global_amax) {
    constexpr int BLOCK = (FMT == QZ_FMT_MXFP8) ? 32 : 16;
    constexpr int CPB = BLOCK / 8;  // chunks per scale block
    const int t = threadIdx.x, lane = t & 31;
    const int64_t row = blockIdx.x;
    const int64_t nch = H >> 3;
    const int64_t kv = H / BLOCK;

    if (row >= T) {
        // an invented row of the swizzled layout: zero scale bytes (kv % 4 == 0)
        for (int64_t k0 = 4 * t; k0 < kv; k0 += 4 * kNormThreads) st_u32(sf + swz_offset(row, k0, kv), 0u);
        return;
    }

    const uint16_t* xr = x + row * H;
    const uint16_t* rr = res + row * H;
    uint4 h[CPT];
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int64_t c = (int64_t)i * kNormThreads + t;
        h[i] = (c < nch) ? ld_stream(xr + c * 8) : make_uint4(0, 0, 0, 0);
    }
    float sh = 0.0f, sl = 0.0f;
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int64_t c = (int64_t)i * kNormThreads + t;
        const uint4 rv = (c < nch) ? ld_stream(rr + c * 8) : make_uint4(0, 0, 0, 0);
        uint32_t* hw = reinterpret_cast<uint32_t*>(&h[i]);
        const uint32_t* rw = reinterpret_cast<const uint32_t*>(&rv);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t lo = bf16_of_sum(bf16_lo(hw[j]), bf16_lo(rw[j]));
            const uint32_t hi = bf16_of_sum(bf16_hi(hw[j]), bf16_hi(rw[j]));
            hw[j] = lo | (hi << 16);
            const float a = bf16_lo(hw[j]), b = bf16_hi(hw[j]);
            two_sum_add(sh, sl, __fmul_rn(a, a));
            two_sum_add(sh, sl, __fmul_rn(b, b));
        }
        if (res_out && c < nch) st_v4(res_out + row * H + c * 8, h[i]);
    }

    // CTA reduction of the sum of squares in binary64
    __shared__ double s_red[kNormThreads / 32];
    double ss = (double)sh + (double)sl;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    if (lane == 0) s_red[t >> 5] = ss;
    __syncthreads();
    double tot = 0.0;
#pragma unroll
    for (int w = 0; w < kNormThreads / 32; ++w) tot += s_red[w];
    const double rstd = 1.0 / sqrt(tot / (double)H + (double)eps);
    const float rh = (float)rstd;
    const float rl = (float)(rstd - (double)rh);

    float S = 0.0f;
    if (FMT == QZ_FMT_NVFP4) S = nvfp4_encode_scale(__ldg(global_amax));

#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int64_t c = (int64_t)i * kNormThreads + t;
        if ((int64_t)i * kNormThreads >= nch) break;  // uniform across the CTA
        const uint4 gv = (c < nch) ? __ldg(reinterpret_cast<const uint4*>(gamma + c * 8)) : make_uint4(0, 0, 0, 0);
        const uint32_t* hw = reinterpret_cast<const uint32_t*>(&h[i]);
        const uint32_t* gw = reinterpret_cast<const uint32_t*>(&gv);
        uint4 y;
        uint32_t* yw = reinterpret_cast<uint32_t*>(&y);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t lo = bf16_scaled(__fmul_rn(bf16_lo(hw[j]), bf16_lo(gw[j])), rh, rl);
            const uint32_t hi = bf16_scaled(__fmul_rn(bf16_hi(hw[j]), bf16_hi(gw[j])), rh, rl);
            yw[j] = lo | (hi << 16);
        }
        if (c < nch) st_v4(norm_out + row * H + c * 8, y);

        // quantize y
        uint32_t m = absmax_bits(y);
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        uint32_t scale;
        if (FMT == QZ_FMT_MXFP8) {
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
            scale = e8m0_byte(m);
            const uint2 codes = e4m3x8_scaled(y, e8m0_reciprocal(scale));
            if (c < nch) st_v2(q + row * H + c * 8, codes.x, codes.y);
        } else {
            const Nvfp4Block blk = nvfp4_block(bits_to_float_bf16(m), S);
            scale = blk.scale;
            const uint32_t codes = e2m1x8_scaled(y, blk.rcp);
            if (c < nch) st_u32(q + row * (H >> 1) + c * 4, codes);
        }
        // scale bytes of 4 consecutive blocks: threads base, base+CPB, base+2CPB, base+3CPB
        const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, scale, CPB);
        const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, scale, 2 * CPB);
        const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, scale, 3 * CPB);
        if ((lane & (4 * CPB - 1)) == 0 && c < nch) {
            const int64_t k0 = c / CPB;
            const uint32_t word = scale | (s1 << 8) | (s2 << 16) | (s3 << 24);
            if (LAYOUT == QZ_SF_SWIZZLED_128x4) {
                st_u32(sf + swz_offset(row, k0, kv), word);
            } else {
                const int64_t base = row * kv + k0;
                if (k0 + 4 <= kv && (base & 3) == 0) st_u32(sf + base, word);
                else for (int j = 0; j < 4 && k0 + j < kv; ++j) sf[base + j] = (uint8_t)(word >> (8 * j));
            }
        }
    }
}

template <int FMT, int LAYOUT>
static cudaError_t launch_norm_fmt(const uint16_t* x, const uint16_t* r, const uint16_t* g, float eps, int64_t T,
                                   int64_t H, uint16_t* y, uint16_t* h, uint8_t* q, uint8_t* sf, const float* amax,
                                   cudaStream_t s) {
    const int64_t grid = (LAYOUT == QZ_SF_SWIZZLED_128x4) ? pad_to(T, 128) : T;
    const int64_t per_thread = (H / 8 + kNormThreads - 1) / kNormThreads;
    if (per_thread <= 2)
        rmsnorm_quant_kernel<FMT, LAYOUT, 2><<<(unsigned)grid, kNormThreads, 0, s>>>(x, r, g, eps, T, H, y, h, q, sf, amax);
    else if (per_thread <= 4)
        rmsnorm_quant_kernel<FMT, LAYOUT, 4><<<(unsigned)grid, kNormThreads, 0, s>>>(x, r, g, eps, T, H, y, h, q, sf, amax);
    else if (per_thread <= 8)
        rmsnorm_quant_kernel<FMT, LAYOUT, 8><<<(unsigned)grid, kNormThreads, 0, s>>>(x, r, g, eps, T, H, y, h, q, sf, amax);
    else
        rmsnorm_quant_kernel<FMT, LAYOUT, 16><<<(unsigned)grid, kNormThreads, 0, s>>>(x, r, g, eps, T, H, y, h, q, sf, amax);
    return cudaGetLastError();
}

cudaError_t launch_rmsnorm_quant(const uint16_t* x, const uint16_t* r, const uint16_t* g, float eps, int64_t T,
                                 int64_t H, uint16_t* y, uint16_t* h, int fmt, uint8_t* q, uint8_t* sf, int layout,
                                 const float* amax, cudaStream_t s) {
    if (fmt == QZ_FMT_MXFP8) {
        return layout == QZ_SF_SWIZZLED_128x4
                   ? launch_norm_fmt<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4>(x, r, g, eps, T, H, y, h, q, sf, amax, s)
                   : launch_norm_fmt<QZ_FMT_MXFP8, QZ_SF_LINEAR>(x, r, g, eps, T, H, y, h, q, sf, amax, s);
    }
    return layout == QZ_SF_SWIZZLED_128x4
               ? launch_norm_fmt<QZ_FMT_NVFP4, QZ_SF_SWIZZLED_128x4>(x, r, g, eps, T, H, y, h, q, sf, amax, s)
               : launch_norm_fmt<QZ_FMT_NVFP4, QZ_SF_LINEAR>(x, r, g, eps, T, H, y, h, q, sf, amax, s);
}

}  // namespace qz
