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
//
// The same kernel, instantiated with MULTI, opens with the tensor-parallel
// AllReduce that feeds the epilogue (the "AllReduce epilogue" of both pages):
// x is the sum of up to eight rank inputs, read through plain pointers that
// may be peer mappings of other GPUs' buffers, accumulated in binary32 in rank
// order and rounded once to bf16, so every rank reduces to the same bits.  It
// takes a row range (one rank's slice, or all rows) and writes every output to
// up to eight destinations (the ranks' own buffers, for the all-gather half).
// A row's rank inputs are read one after another, so each CTA first asks L2
// for the whole row of every rank after the first (one bulk prefetch per
// rank), and throughput mode runs two chunks per thread (two CTAs of 448
// threads per SM at H = 7168) to keep more of those reads in flight.
#include "qz_device.cuh"

namespace qz {

constexpr int kNormMaxThreads = 1024;
constexpr int kMaxRanks = QZ_MAX_RANKS;

struct NormDst {
    uint16_t* y;   // norm_out, bf16 [T, H]
    uint16_t* h;   // residual_out, bf16 [T, H], nullable
    uint8_t* q;    // payload of T rows
    uint8_t* sf;   // SF region of T rows
};

struct NormArgs {
    const uint16_t* x[kMaxRanks];  // rank inputs, bf16 [T, H] each
    NormDst dst[kMaxRanks];
    const uint16_t* res;           // residual bf16 [T, H]
    const uint16_t* gamma;         // bf16 [H]
    const float* global_amax;      // NVFP4 per-tensor amax
    int64_t T, H;
    int64_t row0;                  // first row of this launch (CTA b runs row row0 + b)
    float eps;
    int n_x, n_dst;
};

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

// bf16x2 words of the rank sum of chunks t + nt*i of one row: binary32
// accumulation in rank order (rank 0 exactly, then one rounding per rank), one
// bf16 rounding at the end.  Ranks after the first are loaded G at a time (all
// of them with one chunk per thread, two at a time otherwise), so that G
// chunks' loads per thread are in flight before the first of them is added.
template <int CPT>
__device__ __forceinline__ void rank_sum_row(const NormArgs& a, int64_t row, int nch, int t, int nt,
                                             uint4 (&h)[CPT]) {
    constexpr int G = CPT == 1 ? kMaxRanks - 1 : 2;
    float acc[CPT][8];
    uint4 v[G][CPT];
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = i * nt + t;
        v[0][i] = c < nch ? ld_stream(a.x[0] + row * a.H + c * 8) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const uint32_t* vw = reinterpret_cast<const uint32_t*>(&v[0][i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            acc[i][2 * j] = bf16_lo(vw[j]);
            acc[i][2 * j + 1] = bf16_hi(vw[j]);
        }
    }
    for (int r = 1; r < a.n_x; r += G) {
#pragma unroll
        for (int k = 0; k < G; ++k) {
            const bool live = r + k < a.n_x;
            const uint16_t* xk = a.x[live ? r + k : 0] + row * a.H;
#pragma unroll
            for (int i = 0; i < CPT; ++i) {
                const int c = i * nt + t;
                v[k][i] = (live && c < nch) ? ld_stream(xk + c * 8) : make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int k = 0; k < G; ++k) {
            if (r + k >= a.n_x) break;
#pragma unroll
            for (int i = 0; i < CPT; ++i) {
                const uint32_t* vw = reinterpret_cast<const uint32_t*>(&v[k][i]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[i][2 * j] = __fadd_rn(acc[i][2 * j], bf16_lo(vw[j]));
                    acc[i][2 * j + 1] = __fadd_rn(acc[i][2 * j + 1], bf16_hi(vw[j]));
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        uint32_t* hw = reinterpret_cast<uint32_t*>(&h[i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) hw[j] = cvt_bf16x2(acc[i][2 * j], acc[i][2 * j + 1]);
    }
}

// Bring `bytes` (a multiple of 16, 16-byte aligned) at p into L2; no registers
// wait on it.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// MULTI == false: one input, one destination, row0 == 0 (qz_rmsnorm_quantize).
template <int FMT, int LAYOUT, int CPT, bool MULTI>
__global__ void __launch_bounds__(norm_max_threads(CPT)) rmsnorm_quant_kernel(const __grid_constant__ NormArgs a) {
    constexpr int BLOCK = (FMT == QZ_FMT_MXFP8) ? 32 : 16;
    constexpr int CPB = BLOCK / 8;  // chunks per scale block
    const int t = threadIdx.x, lane = t & 31, nt = blockDim.x;
    const int64_t T = a.T, H = a.H;
    const int64_t row = (MULTI ? a.row0 : 0) + blockIdx.x;
    const int nch = (int)(H >> 3);
    const int kv = (int)(H / BLOCK);
    const int n_dst = MULTI ? a.n_dst : 1;

    if (row >= T) {
        // an invented row of the swizzled layout: zero scale bytes (kv % 4 == 0)
        for (int d = 0; d < n_dst; ++d)
            for (int k0 = 4 * t; k0 < kv; k0 += 4 * nt) st_u32(a.dst[d].sf + swz_offset(row, k0, kv), 0u);
        return;
    }

    // thread k < n_x - 1 prefetches this row of rank k + 1 (H * 2 bytes, 16-byte aligned)
    if (MULTI && t + 1 < a.n_x) prefetch_l2_bulk(a.x[t + 1] + row * H, (uint32_t)(H * 2));
    const uint16_t* rr = a.res + row * H;
    uint4 h[CPT], rv[CPT], gv[CPT];
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = i * nt + t;
        const bool ok = c < nch;
        if (!MULTI) h[i] = ok ? ld_stream(a.x[0] + row * H + c * 8) : make_uint4(0, 0, 0, 0);
        rv[i] = ok ? ld_stream(rr + c * 8) : make_uint4(0, 0, 0, 0);
        gv[i] = ok ? __ldg(reinterpret_cast<const uint4*>(a.gamma + c * 8)) : make_uint4(0, 0, 0, 0);
    }
    if (MULTI) rank_sum_row<CPT>(a, row, nch, t, nt, h);
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
            const float a0 = bf16_lo(hw[j]), b0 = bf16_hi(hw[j]);
            cs = __fmaf_rn(a0, a0, cs);  // a0 * a0 is exact; one rounding per add
            cs = __fmaf_rn(b0, b0, cs);
        }
        two_sum_add(sh, sl, cs);
        if (c < nch)
            for (int d = 0; d < n_dst; ++d)
                if (a.dst[d].h) st_v4(a.dst[d].h + row * H + c * 8, h[i]);
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
    const double rstd = 1.0 / sqrt(tot / (double)H + (double)a.eps);
    const float rh = (float)rstd;
    const float rl = (float)(rstd - (double)rh);

    float S = 0.0f;
    if (FMT == QZ_FMT_NVFP4) S = nvfp4_encode_scale(__ldg(a.global_amax));

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
        if (c < nch)
            for (int d = 0; d < n_dst; ++d) st_v4(a.dst[d].y + row * H + c * 8, y);

        // quantize y
        uint32_t m = absmax_bits(y);
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        uint32_t scale;
        if (FMT == QZ_FMT_MXFP8) {
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
            scale = e8m0_byte(m);
            const uint2 codes = e4m3x8_scaled(y, e8m0_reciprocal(scale));
            if (c < nch)
                for (int d = 0; d < n_dst; ++d) st_v2(a.dst[d].q + row * H + c * 8, codes.x, codes.y);
        } else {
            const Nvfp4Block blk = nvfp4_block(bits_to_float_bf16(m), S, s_inv);
            scale = blk.scale;
            const uint32_t codes = e2m1x8_scaled(y, blk.rcp);
            if (c < nch)
                for (int d = 0; d < n_dst; ++d) st_u32(a.dst[d].q + row * (H >> 1) + c * 4, codes);
        }
        // scale bytes of 4 consecutive blocks: threads base, base+CPB, base+2CPB, base+3CPB
        const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, scale, CPB);
        const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, scale, 2 * CPB);
        const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, scale, 3 * CPB);
        if ((lane & (4 * CPB - 1)) == 0 && c < nch) {
            const int k0 = c / CPB;
            const uint32_t word = scale | (s1 << 8) | (s2 << 16) | (s3 << 24);
            for (int d = 0; d < n_dst; ++d) {
                uint8_t* sf = a.dst[d].sf;
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
}

template <int FMT, int LAYOUT, bool MULTI>
static cudaError_t launch_norm_fmt(const NormArgs& a, int64_t ctas, cudaStream_t s, bool latency_mode) {
    const int nch = (int)(a.H / 8);
    // latency mode: as few chunks per thread as 1024 threads allow;
    // throughput mode: four chunks per thread (fewer, narrower CTAs per row),
    // two with the rank sum (its accumulators cost registers, and more
    // resident threads keep more rank reads in flight)
    int cpt = latency_mode ? 1 : (MULTI ? 2 : 4);
    while ((nch + cpt - 1) / cpt > norm_max_threads(cpt)) cpt *= 2;
    const int threads = (int)pad_to((nch + cpt - 1) / cpt, 32);
    switch (cpt) {
        case 1: rmsnorm_quant_kernel<FMT, LAYOUT, 1, MULTI><<<(unsigned)ctas, threads, 0, s>>>(a); break;
        case 2: rmsnorm_quant_kernel<FMT, LAYOUT, 2, MULTI><<<(unsigned)ctas, threads, 0, s>>>(a); break;
        case 4: rmsnorm_quant_kernel<FMT, LAYOUT, 4, MULTI><<<(unsigned)ctas, threads, 0, s>>>(a); break;
        default: rmsnorm_quant_kernel<FMT, LAYOUT, 8, MULTI><<<(unsigned)ctas, threads, 0, s>>>(a); break;
    }
    return cudaGetLastError();
}

template <bool MULTI>
static cudaError_t launch_norm(const NormArgs& a, int fmt, int layout, int64_t ctas, cudaStream_t s,
                               bool latency_mode) {
    if (fmt == QZ_FMT_MXFP8) {
        return layout == QZ_SF_SWIZZLED_128x4
                   ? launch_norm_fmt<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4, MULTI>(a, ctas, s, latency_mode)
                   : launch_norm_fmt<QZ_FMT_MXFP8, QZ_SF_LINEAR, MULTI>(a, ctas, s, latency_mode);
    }
    return layout == QZ_SF_SWIZZLED_128x4
               ? launch_norm_fmt<QZ_FMT_NVFP4, QZ_SF_SWIZZLED_128x4, MULTI>(a, ctas, s, latency_mode)
               : launch_norm_fmt<QZ_FMT_NVFP4, QZ_SF_LINEAR, MULTI>(a, ctas, s, latency_mode);
}

// latency_mode: few rows (at most about two per SM), so each row gets a wide CTA.
cudaError_t launch_rmsnorm_quant(const uint16_t* x, const uint16_t* r, const uint16_t* g, float eps, int64_t T,
                                 int64_t H, uint16_t* y, uint16_t* h, int fmt, uint8_t* q, uint8_t* sf, int layout,
                                 const float* amax, cudaStream_t s, bool latency_mode) {
    NormArgs a = {};
    a.x[0] = x;
    a.dst[0] = NormDst{y, h, q, sf};
    a.res = r;
    a.gamma = g;
    a.global_amax = amax;
    a.T = T;
    a.H = H;
    a.row0 = 0;
    a.eps = eps;
    a.n_x = 1;
    a.n_dst = 1;
    const int64_t ctas = (layout == QZ_SF_SWIZZLED_128x4) ? pad_to(T, 128) : T;
    return launch_norm<false>(a, fmt, layout, ctas, s, latency_mode);
}

// Rows [row_begin, row_end) of the AllReduce epilogue; the slice that ends at
// T also zeroes the swizzled layout's invented rows of every destination.
cudaError_t launch_allreduce_norm_quant(const uint16_t* const* xs, int n_x, const uint16_t* r, const uint16_t* g,
                                        float eps, int64_t T, int64_t H, int64_t row_begin, int64_t row_end,
                                        const qz_norm_dest* dsts, int n_dst, int fmt, int layout, const float* amax,
                                        cudaStream_t s, bool latency_mode) {
    if (n_x < 1 || n_x > kMaxRanks || n_dst < 1 || n_dst > kMaxRanks) return cudaErrorInvalidValue;
    NormArgs a = {};
    for (int i = 0; i < n_x; ++i) a.x[i] = xs[i];
    for (int d = 0; d < n_dst; ++d)
        a.dst[d] = NormDst{static_cast<uint16_t*>(dsts[d].norm_out), static_cast<uint16_t*>(dsts[d].residual_out),
                           static_cast<uint8_t*>(dsts[d].q), dsts[d].sf};
    a.res = r;
    a.gamma = g;
    a.global_amax = amax;
    a.T = T;
    a.H = H;
    a.row0 = row_begin;
    a.eps = eps;
    a.n_x = n_x;
    a.n_dst = n_dst;
    const int64_t last = (row_end == T && layout == QZ_SF_SWIZZLED_128x4) ? pad_to(T, 128) : row_end;
    const int64_t ctas = last - row_begin;
    if (ctas <= 0) return cudaSuccess;
    return launch_norm<true>(a, fmt, layout, ctas, s, latency_mode);
}

}  // namespace qz
