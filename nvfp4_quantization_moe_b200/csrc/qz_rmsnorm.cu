// qz_rmsnorm.cu -- fused residual add + RMSNorm + MXFP8/NVFP4 quantize (sm_100a).
//
// TensorRT-LLM "NVFP4 linear-SF AllReduce epilogue" (commits 2 and 3) and
// "MXFP8 carrier and quantize folds" (commit 6): the epilogue that already
// holds the bf16 norm in registers emits its quantized form too, from the very
// bf16 values it stores to norm_out, so the result equals quantizing norm_out
// afterwards; the swizzled layout's invented rows are zeroed by the kernel.
//
// One CTA per row; its threads hold chunks t + nt*i (8 bf16 each, nt =
// blockDim.x) of x, residual and gamma in registers.  Small T runs wide CTAs
// (one chunk per thread, latency mode), large T narrow ones (four chunks per
// thread, throughput mode).
//   phase 1: h = bf16(x + r) with one packed bf16 add (the correctly rounded
//            sum, as the oracle's single rounding); sum of h^2: each chunk's
//            eight exact squares are added in binary32 and the chunk sums are
//            merged with TwoSum, then reduced across the CTA in binary64;
//   phase 2: rstd = 1 / sqrt(mean + eps) in binary64 = rh + rl (two binary32
//            words); y = bf16(h * gamma * rstd): h * gamma is exact, y32 =
//            RN(h * gamma * rh) is within two binary32 ulps of the binary64
//            value, so its bf16 rounding is final unless y32 lies within two
//            ulps of a bf16 midpoint, where the exact residue decides;
//            store y, then quantize y exactly like the grouped kernels.
// A block of 32 (MXFP8) or 16 (NVFP4) elements is 4 or 2 consecutive chunks,
// which sit in consecutive threads, so block amax is a butterfly shuffle.
#include "qz_device.cuh"

namespace qz {

constexpr int kNormMaxThreads = 1024;

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

// bf16 of p * (rh + rl), decided on the exact residue: p * rh = hi + lo
// exactly (FMA), plus p * rl; FastTwoSum gives RN32 of the sum and its error.
__device__ __forceinline__ uint32_t bf16_scaled_exact(float p, float rh, float rl) {
    const float hi = __fmul_rn(p, rh);
    float lo = __fmaf_rn(p, rh, -hi);
    lo = __fmaf_rn(p, rl, lo);
    const float s = __fadd_rn(hi, lo);
    const float e = __fsub_rn(lo, __fsub_rn(s, hi));
    return bf16_rne_with_residue(s, e);
}

// Whether binary32 y lies within two ulps of a bf16 rounding midpoint.
__device__ __forceinline__ bool near_bf16_midpoint(float y) {
    return ((__float_as_uint(y) - 0x7FFEu) & 0xFFFFu) <= 4u;
}

__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t add_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Two y values (packed bf16x2) from two exact products p = h * gamma.
__device__ __forceinline__ uint32_t y_pair(float p0, float p1, float rh, float rl) {
    const float y0 = __fmul_rn(p0, rh), y1 = __fmul_rn(p1, rh);
    if (near_bf16_midpoint(y0) || near_bf16_midpoint(y1))
        return bf16_scaled_exact(p0, rh, rl) | (bf16_scaled_exact(p1, rh, rl) << 16);
    return cvt_bf16x2(y0, y1);
}

__device__ __forceinline__ void two_sum_add(float& sh, float& sl, float t) {
    const float s = __fadd_rn(sh, t);
    const float bp = __fsub_rn(s, sh);
    const float err = __fadd_rn(__fsub_rn(sh, __fsub_rn(s, bp)), __fsub_rn(t, bp));
    sh = s;
    sl = __fadd_rn(sl, err);
}

// Thread limit of an instance with CPT chunks per thread (register budget).
__host__ __device__ constexpr int norm_max_threads(int cpt) { return cpt <= 2 ? 1024 : (cpt == 4 ? 512 : 256); }

template <int FMT, int LAYOUT, int CPT>
__global__ void __launch_bounds__(norm_max_threads(CPT)) rmsnorm_quant_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ res, const uint16_t* __restrict__ gamma, float eps,
    int64_t T, int64_t H, uint16_t* __restrict__ norm_out, uint16_t* __restrict__ res_out, uint8_t* __restrict__ q,
    uint8_t* __restrict__ sf, const float* __restrict__ global_amax) {
    constexpr int BLOCK = (FMT == QZ_FMT_MXFP8) ? 32 : 16;
    constexpr int CPB = BLOCK / 8;  // chunks per scale block
    const int t = threadIdx.x, lane = t & 31, nt = blockDim.x;
    const int64_t row = blockIdx.x;
    const int nch = (int)(H >> 3);
    const int kv = (int)(H / BLOCK);

    if (row >= T) {
        // an invented row of the swizzled layout: zero scale bytes (kv % 4 == 0)
        for (int k0 = 4 * t; k0 < kv; k0 += 4 * nt) st_u32(sf + swz_offset(row, k0, kv), 0u);
        return;
    }

    const uint16_t* xr = x + row * H;
    const uint16_t* rr = res + row * H;
    uint4 h[CPT], rv[CPT], gv[CPT];
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = i * nt + t;
        const bool ok = c < nch;
        h[i] = ok ? ld_stream(xr + c * 8) : make_uint4(0, 0, 0, 0);
        rv[i] = ok ? ld_stream(rr + c * 8) : make_uint4(0, 0, 0, 0);
        gv[i] = ok ? __ldg(reinterpret_cast<const uint4*>(gamma + c * 8)) : make_uint4(0, 0, 0, 0);
    }
    float sh = 0.0f, sl = 0.0f;
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = i * nt + t;
        uint32_t* hw = reinterpret_cast<uint32_t*>(&h[i]);
        const uint32_t* rw = reinterpret_cast<const uint32_t*>(&rv[i]);
        float cs = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            hw[j] = add_bf16x2(hw[j], rw[j]);
            const float a = bf16_lo(hw[j]), b = bf16_hi(hw[j]);
            cs = __fmaf_rn(a, a, cs);  // a * a is exact; one rounding per add
            cs = __fmaf_rn(b, b, cs);
        }
        two_sum_add(sh, sl, cs);
        if (res_out && c < nch) st_v4(res_out + row * H + c * 8, h[i]);
    }

    // CTA reduction of the sum of squares in binary64
    __shared__ double s_red[kNormMaxThreads / 32];
    __shared__ float s_inv[16];
    if (FMT == QZ_FMT_NVFP4) fill_inv_table(s_inv);  // published by the barrier below
    double ss = (double)sh + (double)sl;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    if (lane == 0) s_red[t >> 5] = ss;
    __syncthreads();
    double tot = 0.0;
    for (int w = 0; w < (nt >> 5); ++w) tot += s_red[w];
    const double rstd = 1.0 / sqrt(tot / (double)H + (double)eps);
    const float rh = (float)rstd;
    const float rl = (float)(rstd - (double)rh);

    float S = 0.0f;
    if (FMT == QZ_FMT_NVFP4) S = nvfp4_encode_scale(__ldg(global_amax));

#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = i * nt + t;
        if (i * nt >= nch) break;  // uniform across the CTA
        const uint32_t* hw = reinterpret_cast<const uint32_t*>(&h[i]);
        const uint32_t* gw = reinterpret_cast<const uint32_t*>(&gv[i]);
        uint4 y;
        uint32_t* yw = reinterpret_cast<uint32_t*>(&y);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            yw[j] = y_pair(__fmul_rn(bf16_lo(hw[j]), bf16_lo(gw[j])), __fmul_rn(bf16_hi(hw[j]), bf16_hi(gw[j])), rh, rl);
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
            const Nvfp4Block blk = nvfp4_block(bits_to_float_bf16(m), S, s_inv);
            scale = blk.scale;
            const uint32_t codes = e2m1x8_scaled(y, blk.rcp);
            if (c < nch) st_u32(q + row * (H >> 1) + c * 4, codes);
        }
        // scale bytes of 4 consecutive blocks: threads base, base+CPB, base+2CPB, base+3CPB
        const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, scale, CPB);
        const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, scale, 2 * CPB);
        const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, scale, 3 * CPB);
        if ((lane & (4 * CPB - 1)) == 0 && c < nch) {
            const int k0 = c / CPB;
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
                                   cudaStream_t s, bool latency_mode) {
    const int64_t grid = (LAYOUT == QZ_SF_SWIZZLED_128x4) ? pad_to(T, 128) : T;
    const int nch = (int)(H / 8);
    // latency mode: as few chunks per thread as 1024 threads allow;
    // throughput mode: four chunks per thread (fewer, narrower CTAs per row)
    int cpt = latency_mode ? 1 : 4;
    while ((nch + cpt - 1) / cpt > norm_max_threads(cpt)) cpt *= 2;
    const int threads = (int)pad_to((nch + cpt - 1) / cpt, 32);
    switch (cpt) {
        case 1: rmsnorm_quant_kernel<FMT, LAYOUT, 1><<<(unsigned)grid, threads, 0, s>>>(x, r, g, eps, T, H, y, h, q, sf, amax); break;
        case 2: rmsnorm_quant_kernel<FMT, LAYOUT, 2><<<(unsigned)grid, threads, 0, s>>>(x, r, g, eps, T, H, y, h, q, sf, amax); break;
        case 4: rmsnorm_quant_kernel<FMT, LAYOUT, 4><<<(unsigned)grid, threads, 0, s>>>(x, r, g, eps, T, H, y, h, q, sf, amax); break;
        default: rmsnorm_quant_kernel<FMT, LAYOUT, 8><<<(unsigned)grid, threads, 0, s>>>(x, r, g, eps, T, H, y, h, q, sf, amax); break;
    }
    return cudaGetLastError();
}

// latency_mode: few rows (at most about two per SM), so each row gets a wide CTA.
cudaError_t launch_rmsnorm_quant(const uint16_t* x, const uint16_t* r, const uint16_t* g, float eps, int64_t T,
                                 int64_t H, uint16_t* y, uint16_t* h, int fmt, uint8_t* q, uint8_t* sf, int layout,
                                 const float* amax, cudaStream_t s, bool latency_mode) {
    if (fmt == QZ_FMT_MXFP8) {
        return layout == QZ_SF_SWIZZLED_128x4
                   ? launch_norm_fmt<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4>(x, r, g, eps, T, H, y, h, q, sf, amax, s, latency_mode)
                   : launch_norm_fmt<QZ_FMT_MXFP8, QZ_SF_LINEAR>(x, r, g, eps, T, H, y, h, q, sf, amax, s, latency_mode);
    }
    return layout == QZ_SF_SWIZZLED_128x4
               ? launch_norm_fmt<QZ_FMT_NVFP4, QZ_SF_SWIZZLED_128x4>(x, r, g, eps, T, H, y, h, q, sf, amax, s, latency_mode)
               : launch_norm_fmt<QZ_FMT_NVFP4, QZ_SF_LINEAR>(x, r, g, eps, T, H, y, h, q, sf, amax, s, latency_mode);
}

}  // namespace qz
