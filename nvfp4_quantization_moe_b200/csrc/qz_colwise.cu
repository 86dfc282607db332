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
// tile with coalesced 16-byte loads, pairs the elements of two consecutive
// rows into one 32-bit word per column and writes the tile transposed into
// shared memory (XOR-swizzled so that both the scattered writes and the
// 16-byte row reads stay nearly conflict-free); then each thread quantizes
// 64 consecutive elements of one transposed row with the library's block
// quantizers (include/qz_quant.cuh) and writes them to the transposed
// payload.  NVFP4 takes the tensor amax as given (the row-wise computed-amax
// call of the same tensor produces it).
#include "../../include/qz_quant.cuh"

namespace qz {

constexpr int kColThreads = 256;

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

template <int FMT, int LAYOUT>
__global__ void __launch_bounds__(kColThreads, 3) colwise_kernel(const qz_expert* __restrict__ table, int n,
                                                                 unsigned* d_err) {
    constexpr int kBlock = FMT == QZ_FMT_MXFP8 ? 32 : 16;
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    __shared__ __align__(16) uint32_t s_t[kTileCols * 64];  // the tile transposed: [column][row pair]
    const int total = block_prefix(n, s_prefix, s_scan, ColTiles<FMT, LAYOUT>{table, d_err}, d_err);
    const int t = threadIdx.x;
    int e = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        while (tile >= s_prefix[e + 1]) ++e;  // tiles increase; s_prefix[n] == total > tile
        const qz_expert E = load_entry(table, e);
        const int local = tile - s_prefix[e];
        const int nct = (int)((E.cols + kTileCols - 1) / kTileCols);
        const int rt = local / nct, ct = local - rt * nct;
        const int64_t R = E.rows, C = E.cols;
        // ---- load: thread t takes 8 columns (chunk t % 16) of row pairs t / 16 + 16 k
        const int cc = t & 15;
        const int64_t c = (int64_t)ct * kTileCols + 8 * cc;
        const uint16_t* xb = static_cast<const uint16_t*>(E.x);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int rp = (t >> 4) + 16 * k;
            const int64_t r0 = (int64_t)rt * kTileRows + 2 * rp;
            uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
            if (c < C) {  // C % 8 == 0 is not required: a partial chunk is loaded element by element
                if (c + 8 <= C) {
                    if (r0 < R) a = ld_stream(xb + r0 * E.ld + c);
                    if (r0 + 1 < R) b = ld_stream(xb + (r0 + 1) * E.ld + c);
                } else {
                    uint16_t* ah = reinterpret_cast<uint16_t*>(&a);
                    uint16_t* bh = reinterpret_cast<uint16_t*>(&b);
                    for (int j = 0; j < 8 && c + j < C; ++j) {
                        if (r0 < R) ah[j] = xb[r0 * E.ld + c + j];
                        if (r0 + 1 < R) bh[j] = xb[(r0 + 1) * E.ld + c + j];
                    }
                }
            }
            const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int cl = 8 * cc + 2 * j;
                s_t[col_word(cl, rp)] = __byte_perm(aw[j], bw[j], 0x5410);      // (row r0, row r0 + 1) of column cl
                s_t[col_word(cl + 1, rp)] = __byte_perm(aw[j], bw[j], 0x7632);  // the same of column cl + 1
            }
        }
        __syncthreads();
        // ---- quantize: thread t takes rows 64 h .. 64 h + 63 of tile column t % 128
        const int cl = t & 127, h = t >> 7;
        const int64_t cg = (int64_t)ct * kTileCols + cl;  // x column = transposed row
        const int64_t cpad = LAYOUT == QZ_SF_SWIZZLED_128x4 ? ((C + 127) & ~(int64_t)127) : C;
        const int64_t kvT = R / kBlock;                   // scale columns of the transposed matrix
        const int64_t kvs = LAYOUT == QZ_SF_SWIZZLED_128x4 ? ((kvT + 3) & ~(int64_t)3) : kvT;
        const int64_t e0 = (int64_t)rt * kTileRows + 64 * h;  // first transposed column (x row) of the segment
        uint32_t w[32];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const uint4 v = *reinterpret_cast<const uint4*>(&s_t[col_word(cl, 32 * h + 4 * m)]);
            w[4 * m] = v.x;
            w[4 * m + 1] = v.y;
            w[4 * m + 2] = v.z;
            w[4 * m + 3] = v.w;
        }
        if (cg < cpad) {
            const bool live = cg < C;
            constexpr int kBlocks = 64 / kBlock;
            uint32_t scales[kBlocks];
            if (FMT == QZ_FMT_MXFP8) {
                uint8_t* qrow = static_cast<uint8_t*>(E.q) + cg * R + e0;
#pragma unroll
                for (int i = 0; i < kBlocks; ++i) {
                    uint32_t x[16], q[8];
#pragma unroll
                    for (int j = 0; j < 16; ++j) x[j] = w[16 * i + j];
                    scales[i] = qzq::mxfp8_block(x, q);
                    if (live && e0 + 32 * i < R) {
                        st_v4(qrow + 32 * i, make_uint4(q[0], q[1], q[2], q[3]));
                        st_v4(qrow + 32 * i + 16, make_uint4(q[4], q[5], q[6], q[7]));
                    }
                }
            } else {
                const float S = qzq::nvfp4_encode_scale(__ldg(E.amax));
                uint8_t* qrow = static_cast<uint8_t*>(E.q) + cg * (R >> 1) + (e0 >> 1);
#pragma unroll
                for (int i = 0; i < kBlocks; ++i) {
                    uint32_t x[8], q[2];
#pragma unroll
                    for (int j = 0; j < 8; ++j) x[j] = w[8 * i + j];
                    scales[i] = qzq::nvfp4_block(x, S, q);
                    if (live && e0 + 16 * i < R) st_v2(qrow + 8 * i, q[0], q[1]);
                }
            }
            // scale bytes; blocks past the last row hold zeros and get scale 0,
            // padded transposed rows (cg >= C) write 0x00
#pragma unroll
            for (int i = 0; i < kBlocks; ++i) {
                const int64_t k = e0 / kBlock + i;
                if (k < kvs) E.sf[qzq::sf_offset(cg, k, kvT, LAYOUT)] = live ? (uint8_t)scales[i] : (uint8_t)0;
            }
        }
        __syncthreads();  // the shared tile is rewritten by the next tile
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

int colwise_blocks_per_sm(int n) {
    int b = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, colwise_kernel<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4>,
                                                  kColThreads, (size_t)(n + 1) * sizeof(int));
    return b > 0 ? b : 1;
}

}  // namespace qz
