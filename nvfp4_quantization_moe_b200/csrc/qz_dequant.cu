// qz_dequant.cu -- grouped dequantization of MXFP8 / NVFP4 tensors to bf16 (sm_100a).
//
// The inverse map of the grouped quantizers, for reference paths and error
// checks (TransformerEngine PR #3800, Changes: the regression tests compare
// dequantized values; TensorRT-LLM "MXFP8 carrier and quantize folds",
// commit 1: the dequant reference path needs the high-precision tensor).
// An element decodes to the exact product of its code's value and its block
// scale's value (and, for NVFP4, the FP32 decode scale g = RN(A / 2688) of the
// tensor or row), rounded once to bf16 (round to nearest, ties to even).
//
// One persistent launch walks all experts' 128 x 128 tiles like the quantize
// kernels: lane l of warp w owns one scale block per pass (MXFP8: 32
// elements, NVFP4: 16) of rows w + 8 * (lane / LPR) + 32 p of the tile.  All
// of a tile's payload loads are issued before any decoding; the bf16 output
// leaves as 16-byte stores.
#include <cuda_fp16.h>

#include "qz_device.cuh"

namespace qz {

constexpr int kDqThreads = 256;

template <int FMT>
struct DqGeo {
    static constexpr int kBlock = FMT == QZ_FMT_MXFP8 ? 32 : 16;  // elements per scale block
    static constexpr int kLpr = kTileCols / kBlock;                // lanes per tile row: 4 / 8
    static constexpr int kRpp = 8 * (32 / kLpr);                   // tile rows per pass (8 warps): 64 / 32
    static constexpr int kPasses = kTileRows / kRpp;               // passes per tile: 2 / 4
    static constexpr int kQBytes = FMT == QZ_FMT_MXFP8 ? 32 : 8;           // payload bytes per block
    static constexpr int kQWords = kQBytes / 4;
};

__device__ __forceinline__ unsigned dq_entry_errors(const qz_dq_expert& e, int fmt, int layout, bool per_row) {
    const int64_t block = (fmt == QZ_FMT_MXFP8) ? 32 : 16;
    unsigned bad = 0;
    if (e.rows < 0 || e.cols <= 0 || (e.cols % block) != 0 || e.ldy < e.cols || e.ldy > QZ_MAX_LD) bad |= QZ_DERR_SHAPE;
    if (e.rows > 0) {
        if (!e.q || !e.sf || !e.y || (fmt == QZ_FMT_NVFP4 && !e.amax)) bad |= QZ_DERR_NULL;
        if (!aligned(e.y, 16) || (e.ldy & 7) != 0) bad |= QZ_DERR_ALIGN;
        if (!aligned(e.q, fmt == QZ_FMT_MXFP8 ? 16 : 8)) bad |= QZ_DERR_ALIGN;
        if (fmt == QZ_FMT_NVFP4 && !aligned(e.amax, 4)) bad |= QZ_DERR_ALIGN;
    }
    (void)layout;
    (void)per_row;
    return bad;
}

__device__ __forceinline__ qz_dq_expert load_dq_entry(const qz_dq_expert* t, int i) {
    qz_dq_expert e;
    const int64_t* p = reinterpret_cast<const int64_t*>(t + i);
    e.q = reinterpret_cast<const void*>(__ldg(p + 0));
    e.sf = reinterpret_cast<const uint8_t*>(__ldg(p + 1));
    e.amax = reinterpret_cast<const float*>(__ldg(p + 2));
    e.rows = __ldg(p + 3);
    e.cols = __ldg(p + 4);
    e.y = reinterpret_cast<void*>(__ldg(p + 5));
    e.ldy = __ldg(p + 6);
    return e;
}

template <int FMT, int LAYOUT>
struct DqTiles {
    const qz_dq_expert* table;
    bool per_row;
    unsigned* d_err;
    __device__ long long operator()(int i) const {
        const qz_dq_expert e = load_dq_entry(table, i);
        const unsigned bad = dq_entry_errors(e, FMT, LAYOUT, per_row);
        if (bad && d_err && blockIdx.x == 0) atomicOr(d_err, bad);
        if (bad || e.rows == 0) return 0;
        return ((e.rows + kTileRows - 1) / kTileRows) * ((e.cols + kTileCols - 1) / kTileCols);
    }
};

// bf16 bits of the exact value hi + lo (hi = RN32 of it, lo the exact
// remainder), rounded to nearest even: rounding hi again is right unless hi
// lies exactly halfway between two bf16 numbers, where lo decides.
__device__ __forceinline__ uint32_t bf16_of_exact(float hi, float lo) {
    const uint32_t u = __float_as_uint(hi);
    if ((u & 0xFFFFu) == 0x8000u && lo != 0.0f) {
        const bool larger = (lo > 0.0f) == (hi > 0.0f);  // the exact magnitude exceeds |hi|
        return (u >> 16) + (larger ? 1u : 0u);
    }
    return (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
}

// Two e4m3 codes (low byte first) as two binary32 values, exactly.
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t pair) {
    uint32_t h;
    asm("{\n\t.reg .b16 c;\n\tcvt.u16.u32 c, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}" : "=r"(h) : "r"(pair));
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// Two e2m1 codes (low nibble first) as two binary32 values, exactly.
__device__ __forceinline__ float2 e2m1x2_to_f32x2(uint32_t pair) {
    uint32_t h;
    asm("{\n\t.reg .b8 c;\n\tcvt.u8.u32 c, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, c;\n\t}" : "=r"(h) : "r"(pair));
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

__device__ __forceinline__ int64_t dq_sf_index(int layout, int64_t row, int64_t k, int64_t kv) {
    return layout == QZ_SF_SWIZZLED_128x4 ? swz_offset(row, k, kv) : row * kv + k;
}

template <int FMT, int LAYOUT>
__global__ void __launch_bounds__(kDqThreads, 3) dequant_kernel(const qz_dq_expert* __restrict__ table, int n,
                                                                bool per_row, unsigned* d_err) {
    using G = DqGeo<FMT>;
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    const int total = block_prefix(n, s_prefix, s_scan, DqTiles<FMT, LAYOUT>{table, per_row, d_err}, d_err);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kb = lane % G::kLpr;
    int e = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        while (tile >= s_prefix[e + 1]) ++e;  // tiles increase; s_prefix[n] == total > tile
        const qz_dq_expert E = load_dq_entry(table, e);
        const int local = tile - s_prefix[e];
        const int nct = (int)((E.cols + kTileCols - 1) / kTileCols);
        const int rt = local / nct, ct = local - rt * nct;
        const int64_t kv = E.cols / G::kBlock;
        const int64_t k = (int64_t)ct * (kTileCols / G::kBlock) + kb;  // the lane's scale column
        const bool col_ok = k < kv;
        const int64_t qld = FMT == QZ_FMT_MXFP8 ? E.cols : E.cols >> 1;
        // every pass's payload words and scale byte first
        uint32_t qw[G::kPasses][G::kQWords];
        uint32_t sc[G::kPasses];
        int64_t rowp[G::kPasses];
        bool live[G::kPasses];
#pragma unroll
        for (int p = 0; p < G::kPasses; ++p) {
            const int64_t row = (int64_t)rt * kTileRows + p * G::kRpp + w + 8 * (lane / G::kLpr);
            rowp[p] = row;
            live[p] = col_ok && row < E.rows;
            if (live[p]) {
                const uint8_t* src = static_cast<const uint8_t*>(E.q) + row * qld + k * G::kQBytes;
                if (FMT == QZ_FMT_MXFP8) {
                    const uint4 a = ld_stream(src), b = ld_stream(src + 16);
                    qw[p][0] = a.x; qw[p][1] = a.y; qw[p][2] = a.z; qw[p][3] = a.w;
                    qw[p][4] = b.x; qw[p][5] = b.y; qw[p][6] = b.z; qw[p][7] = b.w;
                } else {
                    const uint2 a = __ldg(reinterpret_cast<const uint2*>(src));
                    qw[p][0] = a.x;
                    qw[p][1] = a.y;
                }
                sc[p] = __ldg(E.sf + dq_sf_index(LAYOUT, row, k, kv));
            }
        }
#pragma unroll
        for (int p = 0; p < G::kPasses; ++p) {
            if (!live[p]) continue;
            uint16_t* dst = static_cast<uint16_t*>(E.y) + rowp[p] * E.ldy + k * G::kBlock;
            if (FMT == QZ_FMT_MXFP8) {
                // 2^(byte - 127); byte 0 is the subnormal 2^-127
                const float s = sc[p] ? __uint_as_float(sc[p] << 23) : __uint_as_float(0x00400000u);
#pragma unroll
                for (int h = 0; h < 4; ++h) {  // 8 elements per 16-byte store
                    uint4 o;
                    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t word = qw[p][2 * h + (j >> 1)];
                        const float2 v = e4m3x2_to_f32x2((j & 1) ? (word >> 16) : (word & 0xFFFFu));
                        // exact products (at least 2^-136, above the binary32 subnormal step)
                        const uint32_t lo = bf16_of_exact(__fmul_rn(v.x, s), 0.0f);
                        const uint32_t hi = bf16_of_exact(__fmul_rn(v.y, s), 0.0f);
                        ow[j] = lo | (hi << 16);
                    }
                    st_v4(dst + 8 * h, o);
                }
            } else {
                const float A = __ldg(per_row ? E.amax + rowp[p] : E.amax);
                const float g = __fdiv_rn(A, 2688.0f);  // the FP32 decode scale
                const float sv = e4m3_value(sc[p]);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint4 o;
                    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 c = e2m1x2_to_f32x2((qw[p][h] >> (8 * j)) & 0xFFu);
                        const float p0 = __fmul_rn(c.x, sv), p1 = __fmul_rn(c.y, sv);  // exact: <= 6 bits
                        const float h0 = __fmul_rn(p0, g), h1 = __fmul_rn(p1, g);
                        const float l0 = __fmaf_rn(p0, g, -h0), l1 = __fmaf_rn(p1, g, -h1);
                        ow[j] = bf16_of_exact(h0, l0) | (bf16_of_exact(h1, l1) << 16);
                    }
                    st_v4(dst + 8 * h, o);
                }
            }
        }
    }
}

cudaError_t launch_dequant(const qz_dq_expert* table, int n, int fmt, bool per_row, int layout, int grid,
                           cudaStream_t s, unsigned* d_err) {
    const size_t smem = (size_t)(n + 1) * sizeof(int);
    if (fmt == QZ_FMT_MXFP8) {
        if (layout == QZ_SF_SWIZZLED_128x4)
            dequant_kernel<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4><<<grid, kDqThreads, smem, s>>>(table, n, per_row, d_err);
        else
            dequant_kernel<QZ_FMT_MXFP8, QZ_SF_LINEAR><<<grid, kDqThreads, smem, s>>>(table, n, per_row, d_err);
    } else {
        if (layout == QZ_SF_SWIZZLED_128x4)
            dequant_kernel<QZ_FMT_NVFP4, QZ_SF_SWIZZLED_128x4><<<grid, kDqThreads, smem, s>>>(table, n, per_row, d_err);
        else
            dequant_kernel<QZ_FMT_NVFP4, QZ_SF_LINEAR><<<grid, kDqThreads, smem, s>>>(table, n, per_row, d_err);
    }
    return cudaGetLastError();
}

int dequant_blocks_per_sm(int n) {
    int b = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, dequant_kernel<QZ_FMT_NVFP4, QZ_SF_SWIZZLED_128x4>, kDqThreads,
                                                  (size_t)(n + 1) * sizeof(int));
    return b > 0 ? b : 1;
}

}  // namespace qz
