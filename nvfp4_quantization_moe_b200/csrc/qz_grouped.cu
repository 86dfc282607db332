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
// tile walk with a register prefetch ring
//
// Pass p (0..7) of warp w covers tile rows (p & 3) * 32 + 4w + 2 (p >> 2) +
// lane / 16: the warp owns rows r with r % 32 in [4w, 4w + 4), i.e. exactly
// four 16-byte chunks of every 512-byte swizzled scale tile, which it
// assembles in its own 64 bytes of shared memory (no CTA barrier).  As soon
// as pass p of the current tile is consumed, slot p is refilled with pass p
// of the CTA's next tile, so about eight 16-byte loads per thread are always
// in flight.
// ---------------------------------------------------------------------------

// One thread's view of a tile: pointers to its first row (tile row r0 =
// 4w + lane/16) at its chunk's column; pass p adds kPassRow[p] rows, so the
// per-pass address and bounds arithmetic is 32-bit.
struct TileRef {
    const uint16_t* xp;  // x of (rt*128 + r0, ct*128 + chunk*8)
    uint8_t* qp;         // payload byte of the same element
    uint8_t* sfp;        // linear SF byte of (rt*128 + r0, block of the chunk); swizzled: region base
    const float* amax;
    int ld;              // x row stride, elements
    int qld;             // payload row bytes
    int kv;              // scale columns
    int rows_left;       // pass p is live iff kPassRow[p] < rows_left (and col_ok)
    bool col_ok;
    int rt, ct;
    int expert;
};

__device__ __forceinline__ constexpr int pass_row(int p) { return (p & 3) * 32 + 2 * (p >> 2); }

template <int FMT, int LAYOUT>
__device__ __forceinline__ TileRef tile_ref(const qz_expert* table, const int* s_prefix, int n, int tile, int w,
                                            int lane) {
    const int e = find_owner(s_prefix, n, tile);
    const qz_expert E = load_entry(table, e);
    const int local = tile - s_prefix[e];
    const int nct = (int)((E.cols + kTileCols - 1) / kTileCols);
    TileRef t;
    t.rt = local / nct;
    t.ct = local - t.rt * nct;
    const int chunk = lane & 15;
    const int r0 = 4 * w + (lane >> 4);
    const int64_t row0 = (int64_t)t.rt * kTileRows + r0;
    const int64_t col = (int64_t)t.ct * kTileCols + chunk * 8;
    t.ld = (int)E.ld;
    t.qld = (int)(FMT == QZ_FMT_MXFP8 ? E.cols : E.cols >> 1);
    t.kv = (int)(FMT == QZ_FMT_MXFP8 ? E.cols >> 5 : E.cols >> 4);
    t.xp = static_cast<const uint16_t*>(E.x) + row0 * E.ld + col;
    t.qp = static_cast<uint8_t*>(E.q) + row0 * t.qld + (FMT == QZ_FMT_MXFP8 ? col : col >> 1);
    t.sfp = LAYOUT == QZ_SF_SWIZZLED_128x4 ? E.sf : E.sf + row0 * t.kv + (FMT == QZ_FMT_MXFP8 ? col >> 5 : col >> 4);
    t.amax = E.amax;
    const int64_t left = E.rows - row0;
    t.rows_left = left > kTileRows ? kTileRows : (int)left;
    t.col_ok = col < E.cols;
    t.expert = e;
    return t;
}

__device__ __forceinline__ uint4 tile_load(const TileRef& t, int p) {
    const int pr = pass_row(p);
    return (t.col_ok && pr < t.rows_left) ? ld_stream(t.xp + pr * t.ld) : make_uint4(0, 0, 0, 0);
}

// Quantize pass p of tile t (8 elements per thread in v).  MXFP8 blocks span
// 4 lanes, NVFP4 blocks 2.  Swizzled scale bytes go to the warp's staging
// area s (64 bytes per 4-column scale tile), linear ones straight to memory.
template <int FMT, int LAYOUT>
__device__ __forceinline__ void tile_pass(const TileRef& t, int p, int lane, uint4 v, float S, uint8_t* s,
                                          const float* inv) {
    const int chunk = lane & 15;
    const int pr = pass_row(p);
    const bool live = t.col_ok && pr < t.rows_left;
    const int stage = (2 * (p >> 2) + (lane >> 4)) * 16 + (p & 3) * 4;  // byte of this row in the warp's chunks
    uint32_t m = absmax_bits(v);
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    if (FMT == QZ_FMT_MXFP8) {
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
        const uint32_t byte = e8m0_byte(m);
        const uint2 codes = e4m3x8_scaled(v, e8m0_reciprocal(byte));
        if (live) st_v2(t.qp + pr * t.qld, codes.x, codes.y);
        if ((chunk & 3) == 0) {
            if (LAYOUT == QZ_SF_SWIZZLED_128x4) s[stage + (chunk >> 2)] = live ? (uint8_t)byte : (uint8_t)0;
            else if (live) t.sfp[pr * t.kv] = (uint8_t)byte;
        }
    } else {
        const Nvfp4Block blk = nvfp4_block(bits_to_float_bf16(m), S, inv);
        const uint32_t codes = e2m1x8_scaled(v, blk.rcp);
        if (live) st_u32(t.qp + pr * t.qld, codes);
        if ((chunk & 1) == 0) {
            const int kk = chunk >> 1;  // 0..7: two 4-column scale tiles per tile
            if (LAYOUT == QZ_SF_SWIZZLED_128x4) s[(kk >> 2) * 64 + stage + (kk & 3)] = live ? (uint8_t)blk.scale : (uint8_t)0;
            else if (live) t.sfp[pr * t.kv] = (uint8_t)blk.scale;
        }
    }
}

// Store the warp's staged chunks of the tile's swizzled scale tile(s).
template <int FMT>
__device__ __forceinline__ void tile_flush_sf(const TileRef& t, int w, int lane, const uint8_t* s) {
    __syncwarp();
    const int col_tiles = (t.kv + 3) >> 2;
    constexpr int kTilesPerTile = FMT == QZ_FMT_MXFP8 ? 1 : 2;
    if (lane < 4 * kTilesPerTile) {
        const int j = lane >> 2, c = lane & 3;
        const int ctile = t.ct * kTilesPerTile + j;
        if (ctile < col_tiles)
            st_v4(t.sfp + (((int64_t)t.rt * col_tiles + ctile) << 9) + (4 * w + c) * 16,
                  *reinterpret_cast<const uint4*>(s + j * 64 + c * 16));
    }
    __syncwarp();
}

template <int FMT, int LAYOUT>
__global__ void __launch_bounds__(kThreads, 3) grouped_tile_kernel(const qz_expert* __restrict__ table, int n,
                                                                unsigned* d_err) {
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    constexpr int kStage = FMT == QZ_FMT_MXFP8 ? 64 : 128;
    __shared__ __align__(16) uint8_t s_sf[kThreads / 32][kStage];
    __shared__ float s_inv[16];
    constexpr bool kAmax = FMT == QZ_FMT_NVFP4;
    if (kAmax) fill_inv_table(s_inv);  // published by the barriers in block_prefix
    const int total = block_prefix(n, s_prefix, s_scan, TableTiles<FMT, LAYOUT, kAmax>{table, d_err}, d_err);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int tile = blockIdx.x;
    if (tile >= total) return;
    TileRef cur = tile_ref<FMT, LAYOUT>(table, s_prefix, n, tile, w, lane);
    uint4 v[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) v[p] = tile_load(cur, p);
    for (;;) {
        const int next = tile + gridDim.x;
        const bool more = next < total;
        const TileRef nxt = more ? tile_ref<FMT, LAYOUT>(table, s_prefix, n, next, w, lane) : cur;
        const float S = kAmax ? nvfp4_encode_scale(*cur.amax) : 0.0f;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            tile_pass<FMT, LAYOUT>(cur, p, lane, v[p], S, s_sf[w], s_inv);
            if (more) v[p] = tile_load(nxt, p);
        }
        if (LAYOUT == QZ_SF_SWIZZLED_128x4) tile_flush_sf<FMT>(cur, w, lane, s_sf[w]);
        if (!more) break;
        cur = nxt;
        tile = next;
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

// Same tile walk and prefetch ring as the quantize kernel; each warp keeps a
// running maximum while its tiles stay in one expert and publishes it with
// one atomic max (non-negative floats order like their bit patterns).
template <int LAYOUT>
__global__ void __launch_bounds__(kThreads) amax_grouped_kernel(const qz_expert* __restrict__ table, int n,
                                                                unsigned* d_err) {
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    const int total = block_prefix(n, s_prefix, s_scan, TableTiles<QZ_FMT_NVFP4, LAYOUT, true>{table, d_err}, d_err);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int tile = blockIdx.x;
    if (tile >= total) return;
    TileRef cur = tile_ref<QZ_FMT_NVFP4, LAYOUT>(table, s_prefix, n, tile, w, lane);
    uint4 v[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) v[p] = tile_load(cur, p);
    uint32_t run = 0;
    for (;;) {
        const int next = tile + gridDim.x;
        const bool more = next < total;
        const TileRef nxt = more ? tile_ref<QZ_FMT_NVFP4, LAYOUT>(table, s_prefix, n, next, w, lane) : cur;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            run = max(run, absmax_bits(v[p]));
            if (more) v[p] = tile_load(nxt, p);
        }
        if (!more || nxt.expert != cur.expert) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) run = max(run, __shfl_xor_sync(0xFFFFFFFFu, run, o));
            if (lane == 0) atomicMax(reinterpret_cast<unsigned int*>(const_cast<float*>(cur.amax)), run << 16);
            run = 0;
        }
        if (!more) break;
        cur = nxt;
        tile = next;
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
        grouped_tile_kernel<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4><<<grid, kThreads, prefix_smem(n), s>>>(table, n, d_err);
    else
        grouped_tile_kernel<QZ_FMT_MXFP8, QZ_SF_LINEAR><<<grid, kThreads, prefix_smem(n), s>>>(table, n, d_err);
    return cudaGetLastError();
}

cudaError_t launch_nvfp4_tensor(const qz_expert* table, int n, int layout, bool compute_amax, int grid,
                                cudaStream_t s, unsigned* d_err) {
    if (compute_amax) {
        amax_clear_kernel<<<(n + kThreads - 1) / kThreads, kThreads, 0, s>>>(table, n, layout);
        if (layout == QZ_SF_SWIZZLED_128x4)
            amax_grouped_kernel<QZ_SF_SWIZZLED_128x4><<<grid, kThreads, prefix_smem(n), s>>>(table, n, d_err);
        else
            amax_grouped_kernel<QZ_SF_LINEAR><<<grid, kThreads, prefix_smem(n), s>>>(table, n, d_err);
    }
    if (layout == QZ_SF_SWIZZLED_128x4)
        grouped_tile_kernel<QZ_FMT_NVFP4, QZ_SF_SWIZZLED_128x4><<<grid, kThreads, prefix_smem(n), s>>>(table, n, d_err);
    else
        grouped_tile_kernel<QZ_FMT_NVFP4, QZ_SF_LINEAR><<<grid, kThreads, prefix_smem(n), s>>>(table, n, d_err);
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
        case 0: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, grouped_tile_kernel<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4>, kThreads, smem); break;
        case 1: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, grouped_tile_kernel<QZ_FMT_NVFP4, QZ_SF_SWIZZLED_128x4>, kThreads, smem); break;
        case 2: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, swizzle_kernel, kThreads, smem); break;
        default: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, amax_grouped_kernel<QZ_SF_SWIZZLED_128x4>, kThreads, smem); break;
    }
    return b > 0 ? b : 1;
}

}  // namespace qz
