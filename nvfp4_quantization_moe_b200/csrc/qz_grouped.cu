// qz_grouped.cu -- persistent grouped tile kernels (sm_100a).
//
// One launch walks the whole expert table: every CTA prefix-sums the tiles of
// all experts in shared memory and then strides over the global tile index, so
// uneven and empty experts need no host round trip and no grid barrier.
//
// A tile is 128 rows x 128 bf16 columns (32 KiB of input).  Thread t of the
// 256-thread CTA owns 16-byte chunk (t % 16) of rows t/16 + 16p, p = 0..7: each
// warp reads two 256-byte row segments per instruction.  A scale block is 4
// consecutive chunks (MXFP8, 32 elements) or 2 (NVFP4, 16 elements), so its
// amax is two or one butterfly shuffle away.  Scale bytes of the swizzled
// layout are gathered in a 512-byte shared tile per 128x4 scale tile and
// leave as 16-byte stores; padded rows and scale columns are written as 0x00
// by the tile that owns them.
//
// Pages: NeMo-RL "perf(refit): batch MXFP8 expert prequantization" (Summary,
// Why: one launch for many same-shape experts instead of one per expert);
// TensorRT-LLM "MXFP8 carrier and quantize folds" (commits 3 and 6: padded SF
// rows zeroed by the kernel; commit 5: grid-shape invariance);
// Model-Optimizer "Fold fused experts' quantizers into their weights
// shard-locally" (per-expert FP32 second-level scale).
#include "qz_device.cuh"

namespace qz {

// Tiles of one expert; 0 for an empty or invalid entry (invalid entries are
// reported by block 0 only).
__device__ __forceinline__ int64_t tile_count(const qz_expert& e, unsigned bad) {
    if (bad || e.rows == 0) return 0;
    return ((e.rows + kTileRows - 1) / kTileRows) * ((e.cols + kTileCols - 1) / kTileCols);
}

template <int FMT, int LAYOUT, bool NEEDS_AMAX>
struct TableTiles {
    const qz_expert* table;
    unsigned* d_err;
    __device__ long long operator()(int i) const {
        const qz_expert e = load_entry(table, i);
        const unsigned bad = entry_errors(e, FMT, LAYOUT, NEEDS_AMAX);
        if (bad && d_err && blockIdx.x == 0) atomicOr(d_err, bad);
        return tile_count(e, bad);
    }
};

// ---------------------------------------------------------------------------
// MXFP8 tile
// ---------------------------------------------------------------------------
template <int LAYOUT>
__device__ __forceinline__ void mxfp8_tile(const qz_expert& E, int64_t rt, int64_t ct, uint8_t* s_sf) {
    const int t = threadIdx.x;
    const int chunk = t & 15;
    const int rsub = t >> 4;
    const int64_t col = ct * kTileCols + chunk * 8;
    const bool col_ok = col < E.cols;
    const int64_t kv = E.cols >> 5;
    const uint16_t* x = static_cast<const uint16_t*>(E.x);
    uint8_t* q = static_cast<uint8_t*>(E.q);

    uint4 v[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const int64_t row = rt * kTileRows + p * 16 + rsub;
        v[p] = (row < E.rows && col_ok) ? ld_stream(x + row * E.ld + col) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const int r = p * 16 + rsub;
        const int64_t row = rt * kTileRows + r;
        const bool live = row < E.rows && col_ok;
        uint32_t m = absmax_bits(v[p]);
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
        const uint32_t byte = e8m0_byte(m);
        const uint2 codes = e4m3x8_scaled(v[p], e8m0_reciprocal(byte));
        if (live) st_v2(q + row * E.cols + col, codes.x, codes.y);
        if ((chunk & 3) == 0) {
            const int kc = chunk >> 2;
            if (LAYOUT == QZ_SF_SWIZZLED_128x4) {
                s_sf[swz_in_tile(r, kc)] = live ? (uint8_t)byte : (uint8_t)0;
            } else if (live) {
                E.sf[row * kv + ct * 4 + kc] = (uint8_t)byte;
            }
        }
    }
    if (LAYOUT == QZ_SF_SWIZZLED_128x4) {
        __syncthreads();
        if (t < 32) {
            const int64_t col_tiles = (kv + 3) >> 2;
            uint8_t* dst = E.sf + ((rt * col_tiles + ct) << 9) + t * 16;
            st_v4(dst, reinterpret_cast<const uint4*>(s_sf)[t]);
        }
    }
}

template <int LAYOUT>
__global__ void __launch_bounds__(kThreads) mxfp8_grouped_kernel(const qz_expert* __restrict__ table, int n,
                                                                 unsigned* d_err) {
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    __shared__ __align__(16) uint8_t s_sf[2][512];
    const int total = block_prefix(n, s_prefix, s_scan, TableTiles<QZ_FMT_MXFP8, LAYOUT, false>{table, d_err}, d_err);
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
        const int e = find_owner(s_prefix, n, tile);
        const qz_expert E = load_entry(table, e);
        const int64_t local = tile - s_prefix[e];
        const int64_t nct = (E.cols + kTileCols - 1) / kTileCols;
        mxfp8_tile<LAYOUT>(E, local / nct, local % nct, s_sf[it & 1]);
    }
}

// ---------------------------------------------------------------------------
// NVFP4 tile, per-tensor second-level scale (amax[0] of the expert)
// ---------------------------------------------------------------------------
template <int LAYOUT>
__device__ __forceinline__ void nvfp4_tile(const qz_expert& E, int64_t rt, int64_t ct, uint8_t* s_sf) {
    const int t = threadIdx.x;
    const int chunk = t & 15;
    const int rsub = t >> 4;
    const int64_t col = ct * kTileCols + chunk * 8;
    const bool col_ok = col < E.cols;
    const int64_t kv = E.cols >> 4;
    const uint16_t* x = static_cast<const uint16_t*>(E.x);
    uint8_t* q = static_cast<uint8_t*>(E.q);
    const float S = nvfp4_encode_scale(*E.amax);

    uint4 v[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const int64_t row = rt * kTileRows + p * 16 + rsub;
        v[p] = (row < E.rows && col_ok) ? ld_stream(x + row * E.ld + col) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const int r = p * 16 + rsub;
        const int64_t row = rt * kTileRows + r;
        const bool live = row < E.rows && col_ok;
        uint32_t m = absmax_bits(v[p]);
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        const Nvfp4Block blk = nvfp4_block(bits_to_float_bf16(m), S);
        const uint32_t codes = e2m1x8_scaled(v[p], blk.rcp);
        if (live) st_u32(q + row * (E.cols >> 1) + (col >> 1), codes);
        if ((chunk & 1) == 0) {
            const int kk = chunk >> 1;  // 0..7: two 4-column scale tiles per tile
            if (LAYOUT == QZ_SF_SWIZZLED_128x4) {
                s_sf[((kk >> 2) << 9) + swz_in_tile(r, kk & 3)] = live ? (uint8_t)blk.scale : (uint8_t)0;
            } else if (live) {
                E.sf[row * kv + ct * 8 + kk] = (uint8_t)blk.scale;
            }
        }
    }
    if (LAYOUT == QZ_SF_SWIZZLED_128x4) {
        __syncthreads();
        if (t < 64) {
            const int64_t col_tiles = (kv + 3) >> 2;
            const int64_t ctile = ct * 2 + (t >> 5);
            if (ctile < col_tiles) {
                uint8_t* dst = E.sf + ((rt * col_tiles + ctile) << 9) + (t & 31) * 16;
                st_v4(dst, reinterpret_cast<const uint4*>(s_sf)[t]);
            }
        }
    }
}

template <int LAYOUT>
__global__ void __launch_bounds__(kThreads) nvfp4_tensor_grouped_kernel(const qz_expert* __restrict__ table, int n,
                                                                        unsigned* d_err) {
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    __shared__ __align__(16) uint8_t s_sf[2][1024];
    const int total = block_prefix(n, s_prefix, s_scan, TableTiles<QZ_FMT_NVFP4, LAYOUT, true>{table, d_err}, d_err);
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
        const int e = find_owner(s_prefix, n, tile);
        const qz_expert E = load_entry(table, e);
        const int64_t local = tile - s_prefix[e];
        const int64_t nct = (E.cols + kTileCols - 1) / kTileCols;
        nvfp4_tile<LAYOUT>(E, local / nct, local % nct, s_sf[it & 1]);
    }
}

// ---------------------------------------------------------------------------
// per-tensor amax pass (NVFP4 PER_TENSOR_COMPUTE)
// ---------------------------------------------------------------------------

// amax[0] = 0 for every valid non-empty entry, before the atomic max pass.
__global__ void amax_clear_kernel(const qz_expert* __restrict__ table, int n, int layout) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const qz_expert e = load_entry(table, i);
        if (e.rows > 0 && entry_errors(e, QZ_FMT_NVFP4, layout, true) == 0) *e.amax = 0.0f;
    }
}

__global__ void __launch_bounds__(kThreads) amax_grouped_kernel(const qz_expert* __restrict__ table, int n,
                                                                int layout, unsigned* d_err) {
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    __shared__ uint32_t s_max[kThreads / 32];
    // the table check uses the caller's layout so that invalid entries are
    // skipped identically by this pass and the quantize pass
    int total;
    if (layout == QZ_SF_SWIZZLED_128x4)
        total = block_prefix(n, s_prefix, s_scan, TableTiles<QZ_FMT_NVFP4, QZ_SF_SWIZZLED_128x4, true>{table, d_err}, d_err);
    else
        total = block_prefix(n, s_prefix, s_scan, TableTiles<QZ_FMT_NVFP4, QZ_SF_LINEAR, true>{table, d_err}, d_err);
    const int t = threadIdx.x, chunk = t & 15, rsub = t >> 4;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const int e = find_owner(s_prefix, n, tile);
        const qz_expert E = load_entry(table, e);
        const int64_t local = tile - s_prefix[e];
        const int64_t nct = (E.cols + kTileCols - 1) / kTileCols;
        const int64_t rt = local / nct, ct = local % nct;
        const int64_t col = ct * kTileCols + chunk * 8;
        const uint16_t* x = static_cast<const uint16_t*>(E.x);
        uint4 v[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const int64_t row = rt * kTileRows + p * 16 + rsub;
            v[p] = (row < E.rows && col < E.cols) ? ld_stream(x + row * E.ld + col) : make_uint4(0, 0, 0, 0);
        }
        uint32_t m = 0;
#pragma unroll
        for (int p = 0; p < 8; ++p) m = max(m, absmax_bits(v[p]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if ((t & 31) == 0) s_max[t >> 5] = m;
        __syncthreads();
        if (t == 0) {
            uint32_t mm = 0;
            for (int w = 0; w < kThreads / 32; ++w) mm = max(mm, s_max[w]);
            // non-negative floats order like their bit patterns
            atomicMax(reinterpret_cast<unsigned int*>(E.amax), mm << 16);
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// standalone linear -> swizzled conversion
// ---------------------------------------------------------------------------

struct PairTiles {
    const qz_sf_pair* table;
    unsigned* d_err;
    __device__ long long operator()(int i) const {
        const qz_sf_pair p = table[i];
        unsigned bad = 0;
        if (p.rows < 0 || p.kv < 1) bad |= QZ_DERR_SHAPE;
        if (p.rows > 0 && (!p.src || !p.dst)) bad |= QZ_DERR_NULL;
        if (p.rows > 0 && !aligned(p.dst, 16)) bad |= QZ_DERR_ALIGN;
        if (bad && d_err && blockIdx.x == 0) atomicOr(d_err, bad);
        if (bad || p.rows == 0) return 0;
        return ((p.rows + 127) / 128) * ((p.kv + 3) / 4);
    }
};

// One 128x4 scale tile per iteration: thread t < 128 gathers the 4 bytes of
// tile row t, the tile leaves as 32 16-byte stores.
__global__ void __launch_bounds__(kThreads) swizzle_kernel(const qz_sf_pair* __restrict__ table, int n, unsigned* d_err) {
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    __shared__ __align__(16) uint8_t s_tile[2][512];
    const int total = block_prefix(n, s_prefix, s_scan, PairTiles{table, d_err}, d_err);
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
        const int e = find_owner(s_prefix, n, tile);
        const qz_sf_pair P = table[e];
        const int64_t local = tile - s_prefix[e];
        const int64_t col_tiles = (P.kv + 3) / 4;
        const int64_t rt = local / col_tiles, ct = local % col_tiles;
        uint8_t* s = s_tile[it & 1];
        const int t = threadIdx.x;
        if (t < 128) {
            const int64_t row = rt * 128 + t;
#pragma unroll
            for (int kc = 0; kc < 4; ++kc) {
                const int64_t k = ct * 4 + kc;
                s[swz_in_tile(t, kc)] = (row < P.rows && k < P.kv) ? __ldg(P.src + row * P.kv + k) : (uint8_t)0;
            }
        }
        __syncthreads();
        if (t < 32) st_v4(P.dst + ((rt * col_tiles + ct) << 9) + t * 16, reinterpret_cast<const uint4*>(s)[t]);
    }
}

// ---------------------------------------------------------------------------
// host-side launchers (called from qz_api.cu)
// ---------------------------------------------------------------------------

size_t prefix_smem(int n) { return (size_t)(n + 1) * sizeof(int); }

cudaError_t launch_mxfp8(const qz_expert* table, int n, int layout, int grid, cudaStream_t s, unsigned* d_err) {
    if (layout == QZ_SF_SWIZZLED_128x4)
        mxfp8_grouped_kernel<QZ_SF_SWIZZLED_128x4><<<grid, kThreads, prefix_smem(n), s>>>(table, n, d_err);
    else
        mxfp8_grouped_kernel<QZ_SF_LINEAR><<<grid, kThreads, prefix_smem(n), s>>>(table, n, d_err);
    return cudaGetLastError();
}

cudaError_t launch_nvfp4_tensor(const qz_expert* table, int n, int layout, bool compute_amax, int grid,
                                cudaStream_t s, unsigned* d_err) {
    if (compute_amax) {
        amax_clear_kernel<<<(n + kThreads - 1) / kThreads, kThreads, 0, s>>>(table, n, layout);
        amax_grouped_kernel<<<grid, kThreads, prefix_smem(n), s>>>(table, n, layout, d_err);
    }
    if (layout == QZ_SF_SWIZZLED_128x4)
        nvfp4_tensor_grouped_kernel<QZ_SF_SWIZZLED_128x4><<<grid, kThreads, prefix_smem(n), s>>>(table, n, d_err);
    else
        nvfp4_tensor_grouped_kernel<QZ_SF_LINEAR><<<grid, kThreads, prefix_smem(n), s>>>(table, n, d_err);
    return cudaGetLastError();
}

cudaError_t launch_swizzle(const qz_sf_pair* table, int n, int grid, cudaStream_t s, unsigned* d_err) {
    swizzle_kernel<<<grid, kThreads, prefix_smem(n), s>>>(table, n, d_err);
    return cudaGetLastError();
}

// Resident CTAs per SM of each grouped kernel, for sizing a one-wave grid.
int grouped_blocks_per_sm(int which, int n) {
    int b = 1;
    const size_t smem = prefix_smem(n);
    switch (which) {
        case 0: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, mxfp8_grouped_kernel<QZ_SF_SWIZZLED_128x4>, kThreads, smem); break;
        case 1: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, nvfp4_tensor_grouped_kernel<QZ_SF_SWIZZLED_128x4>, kThreads, smem); break;
        case 2: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, swizzle_kernel, kThreads, smem); break;
        default: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, amax_grouped_kernel, kThreads, smem); break;
    }
    return b > 0 ? b : 1;
}

}  // namespace qz
