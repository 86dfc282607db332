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
// One persistent launch walks all experts' 128 x 128 tiles.  A CTA loads a
// tile with coalesced 16-byte loads (the next tile's loads fly while the
// current one is quantized), pairs the elements of two consecutive rows into
// one 32-bit word per column and writes the tile transposed into
// shared memory (XOR-swizzled so that both the scattered writes and the
// 16-byte row reads stay nearly conflict-free); then each thread quantizes
// 64 consecutive elements of one transposed row with the library's block
// quantizers (include/qz_quant.cuh) and writes them to the transposed
// payload.  NVFP4 takes the tensor amax as given (the row-wise computed-amax
// call of the same tensor produces it).
#include "../../include/qz_quant.cuh"

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

// Word index of (tile column cl, row pair rp) in the transposed shared tile:
// 64 words (128 rows) per column, row pairs XOR-swizzled by
// ((cl ^ cl / 8) mod 8) in bits 2-4.  The load phase writes 16 columns
// 8 apart at a time and the quantize phase reads 8 consecutive columns at a
// time; both see 8 different swizzles, so writes are at most 2-way and the
// 16-byte reads conflict-free.  Bits 0-1 are untouched: 4 consecutive row
// pairs from a multiple of 4 stay one aligned 16-byte chunk.
__device__ __forceinline__ int col_word(int cl, int rp) { return cl * 64 + (rp ^ (((cl ^ (cl >> 3)) & 7) << 2)); }

// One thread's share of a tile: 16 bf16 pairs (rows r0, r0 + 1 of 8 columns, 4 row pairs).
struct ColLoad {
    uint4 a[4], b[4];
};

struct ColRef {
    const uint16_t* x;
    int64_t R, C, ld;
    int rt, ct;
    int expert;
};

__device__ __forceinline__ ColRef col_ref(const qz_expert* table, const int* s_prefix, int tile, int e) {
    while (tile >= s_prefix[e + 1]) ++e;  // tiles increase; s_prefix[n] == total > tile
    const qz_expert E = load_entry(table, e);
    const int local = tile - s_prefix[e];
    const int nct = (int)((E.cols + kTileCols - 1) / kTileCols);
    ColRef r;
    r.rt = local / nct;
    r.ct = local - r.rt * nct;
    r.x = static_cast<const uint16_t*>(E.x);
    r.R = E.rows;
    r.C = E.cols;
    r.ld = E.ld;
    r.expert = e;
    return r;
}

// Thread t's loads of a tile: 8 columns (chunk t % 16) of row pairs t / 16 + 16 k.
__device__ __forceinline__ void col_load(const ColRef& r, int t, ColLoad& v) {
    const int cc = t & 15;
    const int64_t c = (int64_t)r.ct * kTileCols + 8 * cc;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int rp = (t >> 4) + 16 * k;
        const int64_t r0 = (int64_t)r.rt * kTileRows + 2 * rp;
        v.a[k] = make_uint4(0, 0, 0, 0);
        v.b[k] = make_uint4(0, 0, 0, 0);
        if (c < r.C) {
            if (c + 8 <= r.C) {
                if (r0 < r.R) v.a[k] = ld_stream(r.x + r0 * r.ld + c);
                if (r0 + 1 < r.R) v.b[k] = ld_stream(r.x + (r0 + 1) * r.ld + c);
            } else {  // a partial chunk at the end of a row, element by element
                uint16_t* ah = reinterpret_cast<uint16_t*>(&v.a[k]);
                uint16_t* bh = reinterpret_cast<uint16_t*>(&v.b[k]);
                for (int j = 0; j < 8 && c + j < r.C; ++j) {
                    if (r0 < r.R) ah[j] = r.x[r0 * r.ld + c + j];
                    if (r0 + 1 < r.R) bh[j] = r.x[(r0 + 1) * r.ld + c + j];
                }
            }
        }
    }
}

// Write thread t's share into the transposed shared tile (one word per column and row pair).
__device__ __forceinline__ void col_store_smem(uint32_t* s_t, int t, const ColLoad& v) {
    const int cc = t & 15;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int rp = (t >> 4) + 16 * k;
        const uint32_t aw[4] = {v.a[k].x, v.a[k].y, v.a[k].z, v.a[k].w};
        const uint32_t bw[4] = {v.b[k].x, v.b[k].y, v.b[k].z, v.b[k].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int cl = 8 * cc + 2 * j;
            s_t[col_word(cl, rp)] = __byte_perm(aw[j], bw[j], 0x5410);      // (row r0, row r0 + 1) of column cl
            s_t[col_word(cl + 1, rp)] = __byte_perm(aw[j], bw[j], 0x7632);  // the same of column cl + 1
        }
    }
}

template <int FMT, int LAYOUT>
__global__ void __launch_bounds__(kColThreads, 3) colwise_kernel(const qz_expert* __restrict__ table, int n,
                                                                 unsigned* d_err) {
    constexpr int kBlock = FMT == QZ_FMT_MXFP8 ? 32 : 16;
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    __shared__ __align__(16) uint32_t s_t[kTileCols * 64];  // the tile transposed: [column][row pair]
    __shared__ float s_inv[16];
    if (FMT == QZ_FMT_NVFP4) fill_inv_table(s_inv);  // published by the barriers in block_prefix
    const int total = block_prefix(n, s_prefix, s_scan, ColTiles<FMT, LAYOUT>{table, d_err}, d_err);
    const int t = threadIdx.x;
    int tile = blockIdx.x;
    if (tile >= total) return;
    ColRef cur = col_ref(table, s_prefix, tile, 0);
    ColLoad v;
    col_load(cur, t, v);
    for (;;) {
        col_store_smem(s_t, t, v);
        __syncthreads();
        const int next = tile + gridDim.x;
        const bool more = next < total;
        const ColRef nxt = more ? col_ref(table, s_prefix, next, cur.expert) : cur;
        if (more) col_load(nxt, t, v);  // the next tile's loads fly while this one is quantized
        const qz_expert E = load_entry(table, cur.expert);
        const int64_t R = cur.R, C = cur.C;
        // ---- quantize: thread t takes rows 64 h .. 64 h + 63 of tile column t % 128
        const int cl = t & 127, h = t >> 7;
        const int64_t cg = (int64_t)cur.ct * kTileCols + cl;  // x column = transposed row
        const int64_t cpad = LAYOUT == QZ_SF_SWIZZLED_128x4 ? ((C + 127) & ~(int64_t)127) : C;
        const int64_t kvT = R / kBlock;                       // scale columns of the transposed matrix
        const int64_t kvs = LAYOUT == QZ_SF_SWIZZLED_128x4 ? ((kvT + 3) & ~(int64_t)3) : kvT;
        const int64_t e0 = (int64_t)cur.rt * kTileRows + 64 * h;  // first transposed column (x row) of the segment
        // NVFP4: lanes 1..15 hold RN(S / m) for the tile's expert (every lane takes part in the shuffles)
        const float qm = FMT == QZ_FMT_NVFP4 ? rcp_lane_quotient(nvfp4_encode_scale(__ldg(E.amax)), s_inv, t & 31) : 0.0f;
        // every thread decodes its segment (columns past the matrix hold zeros), so
        // that the NVFP4 shuffles see the whole warp; only the stores are guarded
        const bool inreg = cg < cpad;  // a row of the transposed SF region
        const bool live = cg < C;      // a row of the transposed payload
        uint32_t w[32];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const uint4 u = *reinterpret_cast<const uint4*>(&s_t[col_word(cl, 32 * h + 4 * m)]);
            w[4 * m] = u.x;
            w[4 * m + 1] = u.y;
            w[4 * m + 2] = u.z;
            w[4 * m + 3] = u.w;
        }
        constexpr int kBlocks = 64 / kBlock;
        uint32_t scales[kBlocks];
        if (FMT == QZ_FMT_MXFP8) {
            uint8_t* qrow = static_cast<uint8_t*>(E.q) + cg * R + e0;
            const bool q32 = ((reinterpret_cast<uintptr_t>(E.q) & 31) == 0);
#pragma unroll
            for (int i = 0; i < kBlocks; ++i) {
                uint32_t x[16], q[8];
#pragma unroll
                for (int j = 0; j < 16; ++j) x[j] = w[16 * i + j];
                scales[i] = qzq::mxfp8_block(x, q);
                if (live && e0 + 32 * i < R) {
                    const uint4 lo = make_uint4(q[0], q[1], q[2], q[3]), hi = make_uint4(q[4], q[5], q[6], q[7]);
                    if (q32) {
                        st_v8(qrow + 32 * i, lo, hi);
                    } else {
                        st_v4(qrow + 32 * i, lo);
                        st_v4(qrow + 32 * i + 16, hi);
                    }
                }
            }
        } else {
            // the tile kernels' NVFP4 arithmetic (same bytes as qzq::nvfp4_block): block
            // scales two at a time, element multipliers from 16 per-tile quotients
            const float S = nvfp4_encode_scale(__ldg(E.amax));
            uint8_t* qrow = static_cast<uint8_t*>(E.q) + cg * (R >> 1) + (e0 >> 1);
#pragma unroll
            for (int i = 0; i < kBlocks; i += 2) {
                const uint32_t two = tile_scales_nv_words(w + 8 * i, w + 8 * i + 8, S);
                scales[i] = two & 0xFFu;
                scales[i + 1] = two >> 8;
            }
            uint32_t c[2 * kBlocks];
#pragma unroll
            for (int i = 0; i < kBlocks; ++i) {
                const float rcp = nvfp4_rcp_warp(qm, scales[i]);  // all lanes
                c[2 * i] = e2m1x8_words(w[8 * i], w[8 * i + 1], w[8 * i + 2], w[8 * i + 3], rcp);
                c[2 * i + 1] = e2m1x8_words(w[8 * i + 4], w[8 * i + 5], w[8 * i + 6], w[8 * i + 7], rcp);
            }
            // the segment's 32 payload bytes: one 32-byte store when the row is 32-byte aligned
            const uintptr_t qa = reinterpret_cast<uintptr_t>(qrow);
            if (live && e0 + 64 <= R && (qa & 31) == 0) {
                st_v8(qrow, make_uint4(c[0], c[1], c[2], c[3]), make_uint4(c[4], c[5], c[6], c[7]));
            } else if (live && e0 + 64 <= R && (qa & 15) == 0) {
                st_v4(qrow, make_uint4(c[0], c[1], c[2], c[3]));
                st_v4(qrow + 16, make_uint4(c[4], c[5], c[6], c[7]));
            } else if (live) {
#pragma unroll
                for (int i = 0; i < kBlocks; ++i)
                    if (e0 + 16 * i < R) st_v2(qrow + 8 * i, c[2 * i], c[2 * i + 1]);
            }
        }
        // scale bytes; blocks past the last row hold zeros and get scale 0,
        // padded transposed rows (C <= cg < cpad) write 0x00
        if (inreg) {
            // the segment's kBlocks scale bytes are consecutive in both layouts (k0 % kBlocks == 0,
            // and a swizzled row holds 4 consecutive columns per 4-byte group): one store when aligned
            const int64_t k0 = e0 / kBlock;
            uint32_t word = 0;
#pragma unroll
            for (int i = 0; i < kBlocks; ++i) word |= (live ? scales[i] : 0u) << (8 * i);
            uint8_t* p = E.sf + qzq::sf_offset(cg, k0, kvT, LAYOUT);
            if (k0 + kBlocks <= kvs && (reinterpret_cast<uintptr_t>(p) & (kBlocks - 1)) == 0) {
                if (kBlocks == 4) *reinterpret_cast<uint32_t*>(p) = word;
                else *reinterpret_cast<uint16_t*>(p) = (uint16_t)word;
            } else {
#pragma unroll
                for (int i = 0; i < kBlocks; ++i) {
                    const int64_t k = k0 + i;
                    if (k < kvs) E.sf[qzq::sf_offset(cg, k, kvT, LAYOUT)] = (uint8_t)(word >> (8 * i));
                }
            }
        }
        __syncthreads();  // the shared tile is rewritten with the next tile
        if (!more) break;
        tile = next;
        cur = nxt;
    }
}

cudaError_t launch_colwise(const qz_expert* table, int n, int fmt, int layout, int grid, cudaStream_t s,
                           unsigned* d_err) {
    const size_t smem = (size_t)(n + 1) * sizeof(int);
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

// Resident CTAs per SM (for a one-wave persistent grid).  The 32 KB shared
// tile plus the largest prefix table exceed 48 KB, so every instantiation is
// allowed more dynamic shared memory on the current device first (this runs
// once per device before its first launch).
int colwise_blocks_per_sm(int n) {
    const int bytes = (int)((size_t)(QZ_MAX_EXPERTS + 1) * sizeof(int));
    cudaFuncSetAttribute(colwise_kernel<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    cudaFuncSetAttribute(colwise_kernel<QZ_FMT_MXFP8, QZ_SF_LINEAR>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    cudaFuncSetAttribute(colwise_kernel<QZ_FMT_NVFP4, QZ_SF_SWIZZLED_128x4>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    cudaFuncSetAttribute(colwise_kernel<QZ_FMT_NVFP4, QZ_SF_LINEAR>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    int b = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, colwise_kernel<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4>,
                                                  kColThreads, (size_t)(n + 1) * sizeof(int));
    return b > 0 ? b : 1;
}

}  // namespace qz
