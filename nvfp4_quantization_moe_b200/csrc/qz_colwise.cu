// qz_colwise.cu -- grouped column-wise (transposed) MXFP8 / NVFP4 quantization (sm_100a).
//
// TransformerEngine PR #3800 names its fast path "rowwise-only": the backward
// pass also wants each tensor quantized with the blocks running down the
// columns (the operand of the weight-gradient GEMM).  Column-wise
// quantization of x [rows, cols] is the row-wise quantization of x^T: the
// payload is [cols, rows] (MXFP8) or [cols, rows / 2] (NVFP4), the scale
// factors those of a [cols, rows] matrix in the linear or swizzled 128x4
// layout, padding written as 0x00 by the kernel.
//
// One persistent launch walks all experts' 128 x 128 tiles, each CTA a
// contiguous run of them (so its expert -- the entry and the NVFP4 scale --
// changes rarely).  Each CTA keeps three tiles in flight: asynchronous
// 16-byte copies (cp.async, zero-filled past the matrix) bring a tile
// row-major into one of three shared-memory stages while the tile before it
// is quantized, so the loads never wait on the arithmetic and one CTA
// barrier per tile suffices.  A thread reads one
// 32-bit word per row -- two neighbouring columns -- for 32 rows, pairs
// consecutive rows of each column into bf16x2 words, quantizes the two
// 32-element column segments with the library's block quantizers
// (include/qz_quant.cuh) and writes them to the transposed payload.  NVFP4
// takes the tensor amax as given (the row-wise computed-amax call of the
// same tensor produces it).
#include "../../include/qz_quant.cuh"
#include "qz_async.cuh"

namespace qz {

constexpr int kColThreads = 256;

// NVFP4 block scale codes of two 16-element blocks (8 bf16x2 words each).
__device__ __forceinline__ uint32_t tile_scales_nv_words(const uint32_t* w0, const uint32_t* w1, float S) {
    return nvfp4_scale_pair(bits_to_float_bf16(absmax_words<8>(w0)), bits_to_float_bf16(absmax_words<8>(w1)), S);
}

// Column-wise entries: the block runs down the columns, so rows (not cols)
// must be a multiple of the block; the payload rows are `rows` elements long.
__device__ __forceinline__ unsigned colwise_entry_errors(const qz_expert& e, int fmt, int layout) {
    const int64_t block = (fmt == QZ_FMT_MXFP8) ? 32 : 16;
    unsigned bad = 0;
    if (e.rows < 0 || e.cols <= 0 || (e.rows % block) != 0 || e.ld < e.cols || e.ld > QZ_MAX_LD) bad |= QZ_DERR_SHAPE;
    if (e.rows > 0) {
        if (!e.x || !e.q || !e.sf || (fmt == QZ_FMT_NVFP4 && !e.amax)) bad |= QZ_DERR_NULL;
        if (!aligned(e.x, 16) || (e.ld & 7) != 0) bad |= QZ_DERR_ALIGN;
        if (!aligned(e.q, fmt == QZ_FMT_MXFP8 ? 16 : 8)) bad |= QZ_DERR_ALIGN;
        if (layout == QZ_SF_SWIZZLED_128x4 && !aligned(e.sf, 16)) bad |= QZ_DERR_ALIGN;
        if (fmt == QZ_FMT_NVFP4 && !aligned(e.amax, 4)) bad |= QZ_DERR_ALIGN;
    }
    return bad;
}

template <int FMT, int LAYOUT>
struct ColTiles {
    const qz_expert* table;
    unsigned* d_err;
    __device__ long long operator()(int i) const {
        const qz_expert e = load_entry(table, i);
        const unsigned bad = colwise_entry_errors(e, FMT, LAYOUT);
        if (bad && d_err && blockIdx.x == 0) atomicOr(d_err, bad);
        if (bad || e.rows == 0) return 0;
        return ((e.rows + kTileRows - 1) / kTileRows) * ((e.cols + kTileCols - 1) / kTileCols);
    }
};

// A walk over consecutive tiles of the call: the tile's expert (its entry)
// and its row / column tile.  Moving to the next tile reloads the entry only
// when the expert changes.
struct ColRef {
    const uint16_t* x;
    int64_t R, C, ld;
    uint8_t* q;
    uint8_t* sf;
    const float* amax;
    int rt, ct, nct;
    int expert;
};

__device__ __forceinline__ ColRef col_ref(const qz_expert* table, const int* s_prefix, int tile, int e) {
    while (tile >= s_prefix[e + 1]) ++e;  // tiles increase; s_prefix[n] == total > tile
    const qz_expert E = load_entry(table, e);
    const int local = tile - s_prefix[e];
    ColRef r;
    r.nct = (int)((E.cols + kTileCols - 1) / kTileCols);
    r.rt = local / r.nct;
    r.ct = local - r.rt * r.nct;
    r.x = static_cast<const uint16_t*>(E.x);
    r.R = E.rows;
    r.C = E.cols;
    r.ld = E.ld;
    r.q = static_cast<uint8_t*>(E.q);
    r.sf = E.sf;
    r.amax = E.amax;
    r.expert = e;
    return r;
}

// r describes tile - 1; make it describe tile.
__device__ __forceinline__ void col_next(ColRef& r, const qz_expert* table, const int* s_prefix, int tile) {
    if (tile < s_prefix[r.expert + 1]) {
        if (++r.ct == r.nct) {
            r.ct = 0;
            ++r.rt;
        }
    } else {
        r = col_ref(table, s_prefix, tile, r.expert + 1);
    }
}

constexpr int kColStages = 3;                                     // tiles in flight per CTA
constexpr int kColStageBytes = kTileRows * kTileCols * 2;         // one bf16 tile, row-major (32 KB)

// Issue thread t's copies of a tile into a stage: chunk t % 16 (8 columns)
// of rows t / 16 + 16 k.  Rows past the matrix and columns past its last one
// are zero-filled without reading.
__device__ __forceinline__ void col_issue(const ColRef& r, uint32_t stage, int t) {
    const int cc = t & 15;
    const int64_t c = (int64_t)r.ct * kTileCols + 8 * cc;
    const int64_t cols_left = r.C - c;
    const int cbytes = cols_left >= 8 ? 16 : (cols_left > 0 ? (int)cols_left * 2 : 0);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int row = (t >> 4) + 16 * k;
        const int64_t rg = (int64_t)r.rt * kTileRows + row;
        const bool in = rg < r.R && cbytes > 0;
        const void* src = in ? static_cast<const void*>(r.x + rg * r.ld + c) : static_cast<const void*>(r.x);
        cp_async_16(stage + (uint32_t)(row * (kTileCols * 2) + 16 * cc), src, in ? cbytes : 0);
    }
}

template <int FMT, int LAYOUT>
__global__ void __launch_bounds__(kColThreads, 2) colwise_kernel(const qz_expert* __restrict__ table, int n,
                                                                 unsigned* d_err) {
    constexpr int kBlock = FMT == QZ_FMT_MXFP8 ? 32 : 16;
    extern __shared__ __align__(16) int s_prefix[];  // [n + 1] prefix, then the stages (16-byte aligned)
    __shared__ long long s_scan[33];
    __shared__ float s_inv[16];
    if (FMT == QZ_FMT_NVFP4) fill_inv_table(s_inv);  // published by the barriers in block_prefix
    const int total = block_prefix(n, s_prefix, s_scan, ColTiles<FMT, LAYOUT>{table, d_err}, d_err);
    const int t = threadIdx.x;
    const uint32_t stages = (uint32_t)__cvta_generic_to_shared(s_prefix + ((n + 4) & ~3));
    const uint32_t* s_words = reinterpret_cast<const uint32_t*>(s_prefix + ((n + 4) & ~3));

    // this CTA's tiles: a contiguous run [beg, end) of the call's tiles, so the
    // expert (entry, NVFP4 scale) changes at most a few times per CTA
    const int beg = (int)((int64_t)total * blockIdx.x / gridDim.x);
    const int end = (int)((int64_t)total * (blockIdx.x + 1) / gridDim.x);
    if (beg >= end) return;
    ColRef iss = col_ref(table, s_prefix, beg, find_owner(s_prefix, n, beg));  // the walk issuing copies
    ColRef cur = iss;                                                         // the walk quantizing
    // prologue: the first kColStages - 1 tiles in flight
#pragma unroll
    for (int s = 0; s < kColStages - 1; ++s) {
        if (beg + s < end) {
            if (s > 0) col_next(iss, table, s_prefix, beg + s);
            col_issue(iss, stages + s * kColStageBytes, t);
        }
        cp_async_commit();
    }
    const int w = t >> 5, lane = t & 31;
    const int ch = w & 1, rs = w >> 1;  // this warp's column half and 32-row segment of a tile
    // NVFP4: the expert's encode scale, and lanes 1..15 holding RN(S / m)
    int scale_expert = -1;
    float S = 0.0f, qm = 0.0f;
    for (int k = 0;; ++k) {
        const int tile = beg + k;
        if (tile >= end) break;
        const int cur_s = k % kColStages;
        cp_async_wait<kColStages - 2>();  // this thread's copies of tile k have landed
        __syncthreads();                  // ... and everyone's; tile k - 1's stage is free again
        {
            const int ahead = tile + kColStages - 1;
            if (ahead < end) {
                col_next(iss, table, s_prefix, ahead);
                col_issue(iss, stages + ((k + kColStages - 1) % kColStages) * kColStageBytes, t);
            }
            cp_async_commit();
        }
        if (k > 0) col_next(cur, table, s_prefix, tile);
        if (FMT == QZ_FMT_NVFP4 && cur.expert != scale_expert) {
            scale_expert = cur.expert;
            S = nvfp4_encode_scale(__ldg(cur.amax));
            qm = rcp_lane_quotient(S, s_inv, lane);  // every lane: the shuffles below need all
        }
        const int64_t R = cur.R, C = cur.C;
        // ---- thread (warp w, lane l) quantizes tile columns 64 ch + 2 l and + 1,
        //      rows 32 rs .. 32 rs + 31 of each: one word per row holds both columns
        const uint32_t* tw = s_words + cur_s * (kColStageBytes / 4) + (32 * rs) * (kTileCols / 2) + 32 * ch + lane;
        uint32_t xa[16], xb[16];  // column pairs (row 2i low, row 2i + 1 high) of the two columns
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t r0 = tw[(2 * i) * (kTileCols / 2)], r1 = tw[(2 * i + 1) * (kTileCols / 2)];
            xa[i] = __byte_perm(r0, r1, 0x5410);
            xb[i] = __byte_perm(r0, r1, 0x7632);
        }
        const int64_t cg = (int64_t)cur.ct * kTileCols + 64 * ch + 2 * lane;  // x column = transposed row
        const int64_t e0 = (int64_t)cur.rt * kTileRows + 32 * rs;             // first x row of the segment
        const int64_t cpad = LAYOUT == QZ_SF_SWIZZLED_128x4 ? ((C + 127) & ~(int64_t)127) : C;
        const int64_t kvT = R / kBlock;  // scale columns of the transposed matrix
        const int64_t kvs = LAYOUT == QZ_SF_SWIZZLED_128x4 ? ((kvT + 3) & ~(int64_t)3) : kvT;
        const int64_t k0 = e0 / kBlock;  // the segment's first scale column
        constexpr int kSeg = 32 / kBlock;  // scale blocks per column segment: 1 / 2
        uint32_t sc[2][kSeg];
        if (FMT == QZ_FMT_MXFP8) {
            uint32_t qa[8], qb[8];
            sc[0][0] = qzq::mxfp8_block(xa, qa);
            sc[1][0] = qzq::mxfp8_block(xb, qb);
            if (e0 < R) {
                const bool q32 = ((reinterpret_cast<uintptr_t>(cur.q) & 31) == 0);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    if (cg + j >= C) continue;
                    const uint32_t* qq = j ? qb : qa;
                    uint8_t* dst = cur.q + (cg + j) * R + e0;
                    const uint4 lo = make_uint4(qq[0], qq[1], qq[2], qq[3]), hi = make_uint4(qq[4], qq[5], qq[6], qq[7]);
                    if (q32) {
                        st_v8(dst, lo, hi);
                    } else {
                        st_v4(dst, lo);
                        st_v4(dst + 16, hi);
                    }
                }
            }
        } else {
            // the tile kernels' NVFP4 arithmetic (same bytes as qzq::nvfp4_block): block
            // scales two at a time, element multipliers from 16 per-tile quotients
            uint32_t c[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const uint32_t* xx = j ? xb : xa;
                const uint32_t two = tile_scales_nv_words(xx, xx + 8, S);
                sc[j][0] = two & 0xFFu;
                sc[j][1] = two >> 8;
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    const float rcp = nvfp4_rcp_warp(qm, sc[j][b]);
                    c[j][2 * b] = e2m1x8_words(xx[8 * b], xx[8 * b + 1], xx[8 * b + 2], xx[8 * b + 3], rcp);
                    c[j][2 * b + 1] = e2m1x8_words(xx[8 * b + 4], xx[8 * b + 5], xx[8 * b + 6], xx[8 * b + 7], rcp);
                }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                if (cg + j >= C || e0 >= R) continue;
                uint8_t* dst = cur.q + (cg + j) * (R >> 1) + (e0 >> 1);
                if (e0 + 32 <= R && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
                    st_v4(dst, make_uint4(c[j][0], c[j][1], c[j][2], c[j][3]));
                } else {
                    st_v2(dst, c[j][0], c[j][1]);
                    if (e0 + 32 <= R) st_v2(dst + 8, c[j][2], c[j][3]);
                }
            }
        }
        // scale bytes: kSeg consecutive ones per column (blocks past the last row
        // hold zeros and get scale 0; padded transposed rows C <= cg < cpad get 0x00)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int64_t row = cg + j;
            if (row >= cpad) continue;
            const bool live = row < C;
#pragma unroll
            for (int b = 0; b < kSeg; ++b)
                if (k0 + b < kvs) cur.sf[qzq::sf_offset(row, k0 + b, kvT, LAYOUT)] = live ? (uint8_t)sc[j][b] : (uint8_t)0;
        }
    }
    cp_async_wait<0>();  // nothing is left in flight at exit
}

cudaError_t launch_colwise(const qz_expert* table, int n, int fmt, int layout, int grid, cudaStream_t s,
                           unsigned* d_err) {
    const size_t smem = (size_t)((n + 4) & ~3) * sizeof(int) + (size_t)kColStages * kColStageBytes;
    if (fmt == QZ_FMT_MXFP8) {
        if (layout == QZ_SF_SWIZZLED_128x4)
            colwise_kernel<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4><<<grid, kColThreads, smem, s>>>(table, n, d_err);
        else
            colwise_kernel<QZ_FMT_MXFP8, QZ_SF_LINEAR><<<grid, kColThreads, smem, s>>>(table, n, d_err);
    } else {
        if (layout == QZ_SF_SWIZZLED_128x4)
            colwise_kernel<QZ_FMT_NVFP4, QZ_SF_SWIZZLED_128x4><<<grid, kColThreads, smem, s>>>(table, n, d_err);
        else
            colwise_kernel<QZ_FMT_NVFP4, QZ_SF_LINEAR><<<grid, kColThreads, smem, s>>>(table, n, d_err);
    }
    return cudaGetLastError();
}

// Resident CTAs per SM (for a one-wave persistent grid).  The stages plus the
// largest prefix table exceed 48 KB, so every instantiation is allowed more
// dynamic shared memory on the current device first (this runs once per
// device before its first launch).
int colwise_blocks_per_sm(int n) {
    const int bytes = (int)((size_t)((QZ_MAX_EXPERTS + 4) & ~3) * sizeof(int) + (size_t)kColStages * kColStageBytes);
    cudaFuncSetAttribute(colwise_kernel<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    cudaFuncSetAttribute(colwise_kernel<QZ_FMT_MXFP8, QZ_SF_LINEAR>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    cudaFuncSetAttribute(colwise_kernel<QZ_FMT_NVFP4, QZ_SF_SWIZZLED_128x4>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    cudaFuncSetAttribute(colwise_kernel<QZ_FMT_NVFP4, QZ_SF_LINEAR>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    int b = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, colwise_kernel<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4>, kColThreads,
                                                  (size_t)((n + 4) & ~3) * sizeof(int) + (size_t)kColStages * kColStageBytes);
    return b > 0 ? b : 1;
}

}  // namespace qz
