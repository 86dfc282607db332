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
#include <mutex>

#include "qz_device.cuh"

namespace qz {

constexpr int kStaticWsMaxExperts = QZ_STATIC_WS_MAX_EXPERTS;  // table limit of the allocation-free entry point
constexpr int kStaticWsMaxDevices = 64;

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
// tile walk: one lane per scale block, register prefetch ring
//
// A tile is 128 rows x 128 bf16 columns.  Each lane owns one whole scale
// block per pass (MXFP8: 32 elements, 64 bytes; NVFP4: 16 elements, 32 bytes),
// so the block amax, the scale and its reciprocal are computed once per block
// with no shuffles.  LPR lanes cover a row of the tile, a warp covers RPP rows
// per pass, and pass p of warp w covers the rows r with r % 32 = 4w + (l & 3)
// and r / 32 = l >> 2, l = p * RPP + lane / LPR: the warp owns exactly four
// 16-byte chunks of every 512-byte swizzled scale tile and assembles them in
// its own shared-memory staging area (no CTA barrier).  As soon as pass p of
// the current tile is consumed, its registers are refilled with pass p of the
// CTA's next tile, so about 32 bytes of loads per lane stay in flight.
// ---------------------------------------------------------------------------

template <int FMT>
struct TileGeo {
    static constexpr int kBlock = FMT == QZ_FMT_MXFP8 ? 32 : 16;  // elements per scale block
    static constexpr int kLpr = kTileCols / kBlock;                // lanes per tile row: 4 / 8
    static constexpr int kRpp = 32 / kLpr;                         // rows per warp pass: 8 / 4
    static constexpr int kPasses = 16 / kRpp;                      // passes per tile: 2 / 4
    static constexpr int kWords = kBlock / 2;                      // bf16x2 words per lane per pass
    static constexpr int kSfTiles = kTileCols / (4 * kBlock);      // 4-column scale tiles per tile: 1 / 2
};

// One thread's view of a tile: pointers for pass 0; pass p adds p * kRpp * 8 rows.
struct TileRef {
    const uint16_t* xp;  // x of (rt*128 + r(0), ct*128 + kb*block)
    uint8_t* qp;         // payload byte of the same element
    uint8_t* sfp;        // linear SF byte of (row(0), block); swizzled: region base
    const float* amax;
    int ld;              // x row stride, elements
    int qld;             // payload row bytes
    int kv;              // scale columns
    int rows_left;       // pass p is live iff p * kRpp * 8 < rows_left (and col_ok)
    bool col_ok;
    bool a32;            // rows are 32-byte aligned: one 256-bit load per 16 elements
    bool q32;            // payload rows 32-byte aligned (MXFP8): one 256-bit store per block
    int rt, ct;
    int expert;
};

template <int FMT>
__device__ __forceinline__ int local_row(int p, int lane) { return p * TileGeo<FMT>::kRpp + lane / TileGeo<FMT>::kLpr; }

template <int FMT>
__device__ __forceinline__ int tile_row(int p, int w, int lane) {
    const int l = local_row<FMT>(p, lane);
    return (l >> 2) * 32 + 4 * w + (l & 3);
}

template <int FMT, int LAYOUT>
__device__ __forceinline__ TileRef tile_ref(const qz_expert* table, const int* s_prefix, int n, int tile, int w,
                                            int lane, int hint = -1) {
    using G = TileGeo<FMT>;
    int e = hint;
    if (e < 0) {
        e = find_owner(s_prefix, n, tile);
    } else {
        while (tile >= s_prefix[e + 1]) ++e;  // hint owns a tile <= this one; s_prefix[n] = total > tile
    }
    const qz_expert E = load_entry(table, e);
    const int local = tile - s_prefix[e];
    const int nct = (int)((E.cols + kTileCols - 1) / kTileCols);
    TileRef t;
    // (the MXFP8 tiles measured faster with the plain division and search)
    t.rt = FMT == QZ_FMT_NVFP4 ? div_nonneg(local, nct) : local / nct;
    t.ct = local - t.rt * nct;
    const int kb = lane % G::kLpr;
    const int64_t row0 = (int64_t)t.rt * kTileRows + tile_row<FMT>(0, w, lane);
    const int64_t col = (int64_t)t.ct * kTileCols + kb * G::kBlock;
    t.ld = (int)E.ld;
    t.qld = (int)(FMT == QZ_FMT_MXFP8 ? E.cols : E.cols >> 1);
    t.kv = (int)(E.cols / G::kBlock);
    t.xp = static_cast<const uint16_t*>(E.x) + row0 * E.ld + col;
    t.qp = static_cast<uint8_t*>(E.q) + row0 * t.qld + (FMT == QZ_FMT_MXFP8 ? col : col >> 1);
    t.sfp = LAYOUT == QZ_SF_SWIZZLED_128x4 ? E.sf : E.sf + row0 * t.kv + col / G::kBlock;
    t.amax = E.amax;
    const int64_t left = E.rows - row0;
    t.rows_left = left > kTileRows ? kTileRows : (int)left;
    t.col_ok = col < E.cols;
    t.a32 = ((reinterpret_cast<uintptr_t>(E.x) & 31) == 0) && ((E.ld & 15) == 0);
    t.q32 = (reinterpret_cast<uintptr_t>(E.q) & 31) == 0;  // MXFP8 rows are cols bytes, a multiple of 32
    t.expert = e;
    return t;
}

template <int FMT>
__device__ __forceinline__ bool pass_live(const TileRef& t, int p) {
    return t.col_ok && p * TileGeo<FMT>::kRpp * 8 < t.rows_left;
}

// The lane's block of pass p (zeros outside the matrix).
template <int FMT, int HINT = kL2Normal>
__device__ __forceinline__ void tile_load(const TileRef& t, int p, uint32_t* w) {
    using G = TileGeo<FMT>;
    uint32_t (&a)[8] = *reinterpret_cast<uint32_t(*)[8]>(w);
    uint32_t (&b)[8] = *reinterpret_cast<uint32_t(*)[8]>(w + 8 * (G::kWords / 8 - 1));
    if (pass_live<FMT>(t, p)) {
        const uint16_t* src = t.xp + p * G::kRpp * 8 * t.ld;
        if (t.a32) {
            ld_stream_32<HINT>(src, a);
            if (G::kWords == 16) ld_stream_32<HINT>(src + 16, b);
        } else {
            ld_pair_16<HINT>(src, a);
            if (G::kWords == 16) ld_pair_16<HINT>(src + 16, b);
        }
    } else {
#pragma unroll
        for (int i = 0; i < G::kWords; ++i) w[i] = 0u;
    }
}

// Scale byte of the lane's block of pass p: swizzled bytes go to the warp's
// staging area s (64 bytes per 4-column scale tile), linear ones to memory.
template <int FMT, int LAYOUT>
__device__ __forceinline__ void tile_scale_store(const TileRef& t, int p, int lane, uint32_t scale, uint8_t* s) {
    using G = TileGeo<FMT>;
    const bool live = pass_live<FMT>(t, p);
    const int l = local_row<FMT>(p, lane);
    const int kb = lane % G::kLpr;
    if (LAYOUT == QZ_SF_SWIZZLED_128x4) {
        s[(kb >> 2) * 64 + (l & 3) * 16 + (l >> 2) * 4 + (kb & 3)] = live ? (uint8_t)scale : (uint8_t)0;
    } else if (live) {
        t.sfp[p * G::kRpp * 8 * t.kv] = (uint8_t)scale;
    }
}

// MXFP8: quantize the lane's 32-element block of pass p.
template <int LAYOUT>
__device__ __forceinline__ void tile_pass_mx(const TileRef& t, int p, int lane, const uint32_t* w, uint8_t* s) {
    using G = TileGeo<QZ_FMT_MXFP8>;
    const uint32_t scale = e8m0_byte(absmax_words<G::kWords>(w));
    const float r = e8m0_reciprocal(scale);
    uint4 c0, c1;
    c0.x = e4m3x4_words(w[0], w[1], r);
    c0.y = e4m3x4_words(w[2], w[3], r);
    c0.z = e4m3x4_words(w[4], w[5], r);
    c0.w = e4m3x4_words(w[6], w[7], r);
    c1.x = e4m3x4_words(w[8], w[9], r);
    c1.y = e4m3x4_words(w[10], w[11], r);
    c1.z = e4m3x4_words(w[12], w[13], r);
    c1.w = e4m3x4_words(w[14], w[15], r);
    if (pass_live<QZ_FMT_MXFP8>(t, p)) {
        uint8_t* dst = t.qp + p * G::kRpp * 8 * t.qld;
        if (t.q32) {
            st_v8(dst, c0, c1);  // four lanes fill 128 contiguous bytes in one store
        } else {
            st_v4(dst, c0);
            st_v4(dst + 16, c1);
        }
    }
    tile_scale_store<QZ_FMT_MXFP8, LAYOUT>(t, p, lane, scale, s);
}

// NVFP4: quantize the lane's 16-element block of pass p with scale code
// `scale` and element multiplier rcp.
template <int LAYOUT>
__device__ __forceinline__ void tile_pass_nv(const TileRef& t, int p, int lane, const uint32_t* w, uint32_t scale,
                                             float rcp, uint8_t* s) {
    using G = TileGeo<QZ_FMT_NVFP4>;
    const uint32_t c0 = e2m1x8_words(w[0], w[1], w[2], w[3], rcp);
    const uint32_t c1 = e2m1x8_words(w[4], w[5], w[6], w[7], rcp);
    if (pass_live<QZ_FMT_NVFP4>(t, p)) st_v2(t.qp + p * G::kRpp * 8 * t.qld, c0, c1);
    tile_scale_store<QZ_FMT_NVFP4, LAYOUT>(t, p, lane, scale, s);
}

// NVFP4 block scale codes of passes p and p + 1 (one packed pair).
__device__ __forceinline__ uint32_t tile_scales_nv(const uint32_t* w0, const uint32_t* w1, float S) {
    return nvfp4_scale_pair(bits_to_float_bf16(absmax_words<8>(w0)), bits_to_float_bf16(absmax_words<8>(w1)), S);
}

// Store the warp's staged chunks of the tile's swizzled scale tile(s).
template <int FMT>
__device__ __forceinline__ void tile_flush_sf(const TileRef& t, int w, int lane, const uint8_t* s) {
    __syncwarp();
    const int col_tiles = (t.kv + 3) >> 2;
    constexpr int kT = TileGeo<FMT>::kSfTiles;
    if (lane < 4 * kT) {
        const int j = lane >> 2, c = lane & 3;
        const int ctile = t.ct * kT + j;
        if (ctile < col_tiles)
            st_v4(t.sfp + (((int64_t)t.rt * col_tiles + ctile) << 9) + (4 * w + c) * 16,
                  *reinterpret_cast<const uint4*>(s + j * 64 + c * 16));
    }
    __syncwarp();
}

template <int FMT, int LAYOUT>
__global__ void __launch_bounds__(kThreads, 3) grouped_tile_kernel(const qz_expert* __restrict__ table, int n,
                                                                   unsigned* d_err) {
    using G = TileGeo<FMT>;
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    __shared__ __align__(16) uint8_t s_sf[kThreads / 32][64 * G::kSfTiles];
    __shared__ float s_inv[16];
    constexpr bool kAmax = FMT == QZ_FMT_NVFP4;
    if (kAmax) fill_inv_table(s_inv);  // published by the barriers in block_prefix
    const int total = block_prefix(n, s_prefix, s_scan, TableTiles<FMT, LAYOUT, kAmax>{table, d_err}, d_err);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int tile = blockIdx.x;
    if (tile >= total) return;
    TileRef cur = tile_ref<FMT, LAYOUT>(table, s_prefix, n, tile, w, lane);
    uint32_t v[G::kPasses][G::kWords];
#pragma unroll
    for (int p = 0; p < G::kPasses; ++p) tile_load<FMT>(cur, p, v[p]);
    for (;;) {
        const int next = tile + gridDim.x;
        const bool more = next < total;
        const TileRef nxt = more ? tile_ref<FMT, LAYOUT>(table, s_prefix, n, next, w, lane, FMT == QZ_FMT_NVFP4 ? cur.expert : -1) : cur;
        const float S = kAmax ? nvfp4_encode_scale(*cur.amax) : 0.0f;
        if (FMT == QZ_FMT_MXFP8) {
#pragma unroll
            for (int p = 0; p < G::kPasses; ++p) {
                tile_pass_mx<LAYOUT>(cur, p, lane, v[p], s_sf[w]);
                if (more) tile_load<FMT>(nxt, p, v[p]);
            }
        } else {
            const float qm = rcp_lane_quotient(S, s_inv, lane);
#pragma unroll
            for (int p = 0; p < G::kPasses; p += 2) {
                const uint32_t sc = tile_scales_nv(v[p], v[p + 1], S);
                const uint32_t sc0 = sc & 0xFFu, sc1 = sc >> 8;
                tile_pass_nv<LAYOUT>(cur, p, lane, v[p], sc0, nvfp4_rcp_warp(qm, sc0), s_sf[w]);
                if (more) tile_load<FMT>(nxt, p, v[p]);
                tile_pass_nv<LAYOUT>(cur, p + 1, lane, v[p + 1], sc1, nvfp4_rcp_warp(qm, sc1), s_sf[w]);
                if (more) tile_load<FMT>(nxt, p + 1, v[p + 1]);
            }
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
__global__ void __launch_bounds__(kThreads, 3) amax_grouped_kernel(const qz_expert* __restrict__ table, int n,
                                                                   unsigned* d_err) {
    using G = TileGeo<QZ_FMT_NVFP4>;
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    const int total = block_prefix(n, s_prefix, s_scan, TableTiles<QZ_FMT_NVFP4, LAYOUT, true>{table, d_err}, d_err);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int tile = blockIdx.x;
    if (tile >= total) return;
    TileRef cur = tile_ref<QZ_FMT_NVFP4, LAYOUT>(table, s_prefix, n, tile, w, lane);
    uint32_t v[G::kPasses][G::kWords];
#pragma unroll
    for (int p = 0; p < G::kPasses; ++p) tile_load<QZ_FMT_NVFP4>(cur, p, v[p]);
    uint32_t run = 0;
    for (;;) {
        const int next = tile + gridDim.x;
        const bool more = next < total;
        const TileRef nxt = more ? tile_ref<QZ_FMT_NVFP4, LAYOUT>(table, s_prefix, n, next, w, lane, cur.expert) : cur;
#pragma unroll
        for (int p = 0; p < G::kPasses; ++p) {
            run = max(run, absmax_words<G::kWords>(v[p]));
            if (more) tile_load<QZ_FMT_NVFP4>(nxt, p, v[p]);
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
// NVFP4 with a computed per-tensor amax in one launch (L2-chunked)
//
// The experts are cut into chunks of consecutive experts holding about
// kChunkTiles tiles (~16 MB of bf16).  Work items are runs of up to
// kItemTiles tiles of one chunk, fetched from an atomic counter in segment
// order: segment s holds A(s) then Q(s - kLag) (the last kLag segments hold
// only Q items).  An A item folds its tiles' amax into their experts' slots
// (atomic max) and adds its tile count to its chunk's done counter; a Q item
// quantizes tiles of chunk s - kLag once that chunk's A tiles are all done,
// re-reading the input from L2 where the A pass left it.  kLag chunks of A
// items (more than the items in flight on the whole GPU) separate a chunk's
// A and Q items, so Q items rarely wait, while the kLag + 1 live chunks stay
// well inside L2.  Every item waits only on items fetched before it and A
// items never wait, so all items finish whatever the number of resident CTAs;
// the wait is still bounded (QZ_DERR_TIMEOUT).  A CTA consumes each fetched
// item index one item later, so the atomic's latency is hidden.
//
// Workspace (caller's device memory, zeroed by the call):
//   ws[0] next item, ws[8 + k] done A tiles of chunk k, then one amax word per
//   expert (bf16 magnitude bits << 16).
// ---------------------------------------------------------------------------

constexpr int kChunkTiles = 512;       // ~16 MB of bf16 input per chunk
constexpr int kItemTiles = 2;          // tiles per work item
constexpr int kLag = 2;                // chunks between a chunk's A items and its Q items
constexpr int kMaxChunks = 4096;
constexpr int kWsHeader = 8;
static_assert(kLag >= 1, "Q items of a chunk must follow all of its A items");

__host__ __device__ constexpr size_t workspace_words(int n) { return (size_t)kWsHeader + kMaxChunks + (size_t)n; }

struct ItemRef {
    int first_tile;  // first tile of the run
    int ntiles;      // tiles in the run (1..kItemTiles)
    int chunk;
    bool is_a;
};

template <int LAYOUT>
__global__ void __launch_bounds__(kThreads, 3) nvfp4_compute_l2_kernel(const qz_expert* __restrict__ table, int n,
                                                                       unsigned* __restrict__ ws, unsigned* d_err) {
    using G = TileGeo<QZ_FMT_NVFP4>;
    extern __shared__ int s_dyn[];
    int* s_prefix = s_dyn;                 // n + 1: first tile of each expert
    int* s_cf = s_dyn + (n + 1);           // nchunks + 1: first tile of each chunk
    int* s_seg = s_cf + (kMaxChunks + 1);  // nchunks + kLag + 1: first item of each segment
    __shared__ long long s_scan[33];
    __shared__ __align__(16) uint8_t s_sf[kThreads / 32][64 * G::kSfTiles];
    __shared__ float s_inv[16];
    __shared__ int s_item[4];
    __shared__ unsigned s_ok[2];
    fill_inv_table(s_inv);
    const int total = block_prefix(n, s_prefix, s_scan, TableTiles<QZ_FMT_NVFP4, LAYOUT, true>{table, d_err}, d_err);
    if (total == 0) return;
    const int tpc = max(kChunkTiles, (total + kMaxChunks - 1) / kMaxChunks);  // tiles per chunk
    const int nchunks = (total + tpc - 1) / tpc;
    // chunk k starts at the first expert whose first tile is >= k * tpc
    for (int k = threadIdx.x; k <= nchunks; k += blockDim.x) {
        const int target = k * tpc;
        int lo = 0, hi = n;  // first e in [0, n] with s_prefix[e] >= target (s_prefix[n] = total)
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (s_prefix[mid] >= target) hi = mid; else lo = mid + 1;
        }
        s_cf[k] = s_prefix[lo];
    }
    __syncthreads();
    // items of chunk k: ceil(T(k) / kItemTiles); segment s = A(s) then Q(s - kLag)
    auto chunk_items = [&](int k) {
        return (k >= 0 && k < nchunks) ? (s_cf[k + 1] - s_cf[k] + kItemTiles - 1) / kItemTiles : 0;
    };
    const int nseg = nchunks + kLag;
    if (threadIdx.x == 0) {
        int run = 0;
        for (int k = 0; k < nseg; ++k) {
            s_seg[k] = run;
            run += chunk_items(k) + chunk_items(k - kLag);
        }
        s_seg[nseg] = run;
    }
    unsigned* next_item = ws;
    unsigned* done = ws + kWsHeader;
    unsigned* amax_ws = ws + kWsHeader + kMaxChunks;
    unsigned pending = 0;  // thread 0: an item index fetched one iteration ahead
    if (threadIdx.x == 0) {
        s_item[0] = (int)atomicAdd(next_item, 1u);
        pending = atomicAdd(next_item, 1u);
    }
    __syncthreads();
    const int items = s_seg[nseg];
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;

    auto decode = [&](int j) {
        int lo = 0, hi = nseg - 1;  // last s with s_seg[s] <= j
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_seg[mid] <= j) lo = mid; else hi = mid - 1;
        }
        const int off = j - s_seg[lo];
        const int a_items = chunk_items(lo);
        ItemRef r;
        r.is_a = off < a_items;
        r.chunk = r.is_a ? lo : lo - kLag;
        const int idx = r.is_a ? off : off - a_items;
        r.first_tile = s_cf[r.chunk] + idx * kItemTiles;
        r.ntiles = min(kItemTiles, s_cf[r.chunk + 1] - r.first_tile);
        return r;
    };

    // A reads keep their lines in L2 for the Q re-read; Q reads release them
    auto load_tile = [&](const TileRef& t, bool a_item, uint32_t (&v)[G::kPasses][G::kWords]) {
        if (a_item) {
#pragma unroll
            for (int p = 0; p < G::kPasses; ++p) tile_load<QZ_FMT_NVFP4, kL2Last>(t, p, v[p]);
        } else {
#pragma unroll
            for (int p = 0; p < G::kPasses; ++p) tile_load<QZ_FMT_NVFP4, kL2First>(t, p, v[p]);
        }
    };
    int j = s_item[0];
    if (j >= items) return;
    ItemRef item = decode(j);
    TileRef cur = tile_ref<QZ_FMT_NVFP4, LAYOUT>(table, s_prefix, n, item.first_tile, w, lane);
    uint32_t v[G::kPasses][G::kWords];
    load_tile(cur, item.is_a, v);
    for (int it = 0;; ++it) {
        // publish the index fetched during the previous item, fetch another
        if (threadIdx.x == 0) {
            s_item[(it + 1) & 3] = (int)pending;
            pending = atomicAdd(next_item, 1u);
            unsigned ok = 1;
            if (!item.is_a) {
                // wait until every A tile of this item's chunk is done
                const unsigned need = (unsigned)(s_cf[item.chunk + 1] - s_cf[item.chunk]);
                const long long t0 = clock64();
                while (ld_acquire_gpu(done + item.chunk) < need) {
                    if (clock64() - t0 > (1LL << 31)) {
                        if (d_err) atomicOr(d_err, QZ_DERR_TIMEOUT);
                        ok = 0;
                        break;
                    }
                }
            }
            s_ok[it & 1] = ok;
        }
        __syncthreads();
        const int jn = s_item[(it + 1) & 3];
        const bool more_items = jn < items;
        const ItemRef nitem = more_items ? decode(jn) : item;
        uint32_t run = 0;  // A: running max of this warp over the item's tiles of one expert
        for (int k = 0; k < item.ntiles; ++k) {
            const bool last = k + 1 == item.ntiles;
            const bool more = !last || more_items;
            const int ntile = last ? nitem.first_tile : item.first_tile + k + 1;
            const bool next_a = last ? nitem.is_a : item.is_a;
            const TileRef nxt = more ? tile_ref<QZ_FMT_NVFP4, LAYOUT>(table, s_prefix, n, ntile, w, lane) : cur;
            if (item.is_a) {
#pragma unroll
                for (int p = 0; p < G::kPasses; ++p) run = max(run, absmax_words<G::kWords>(v[p]));
                if (more) load_tile(nxt, next_a, v);
                if (last || nxt.expert != cur.expert) {
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) run = max(run, __shfl_xor_sync(0xFFFFFFFFu, run, o));
                    if (lane == 0) atomicMax(amax_ws + cur.expert, run << 16);
                    run = 0;
                }
            } else {
                // ordered after thread 0's acquire of the chunk count by the barrier above
                const float A = __uint_as_float(ld_relaxed_gpu(amax_ws + cur.expert));
                const float S = nvfp4_encode_scale(A);
                const float qm = rcp_lane_quotient(S, s_inv, lane);
#pragma unroll
                for (int p = 0; p < G::kPasses; p += 2) {
                    const uint32_t sc = tile_scales_nv(v[p], v[p + 1], S);
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const uint32_t scq = (sc >> (8 * q)) & 0xFFu;
                        tile_pass_nv<LAYOUT>(cur, p + q, lane, v[p + q], scq, nvfp4_rcp_warp(qm, scq), s_sf[w]);
                        if (more) {
                            if (next_a) tile_load<QZ_FMT_NVFP4, kL2Last>(nxt, p + q, v[p + q]);
                            else tile_load<QZ_FMT_NVFP4, kL2First>(nxt, p + q, v[p + q]);
                        }
                    }
                }
                if (LAYOUT == QZ_SF_SWIZZLED_128x4) tile_flush_sf<QZ_FMT_NVFP4>(cur, w, lane, s_sf[w]);
                if (threadIdx.x == 0) *const_cast<float*>(cur.amax) = A;
            }
            cur = nxt;
        }
        if (item.is_a) {
            // every warp's atomic max precedes the barrier; thread 0's fence
            // then releases them all before the count (the grid-barrier idiom)
            __syncthreads();
            if (threadIdx.x == 0) {
                __threadfence();
                atomicAdd(done + item.chunk, (unsigned)item.ntiles);
            }
        }
        if (!more_items) break;
        item = nitem;
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

size_t workspace_bytes(int n) { return workspace_words(n) * sizeof(unsigned); }

size_t compute_l2_smem(int n) { return (size_t)(n + 1 + kMaxChunks + 1 + kMaxChunks + kLag + 1) * sizeof(int); }

// One launch of the L2-chunked computed-amax path on a zeroed workspace.
cudaError_t launch_nvfp4_compute_l2(const qz_expert* table, int n, int layout, int grid, unsigned* ws,
                                    cudaStream_t s, unsigned* d_err) {
    cudaError_t e = cudaMemsetAsync(ws, 0, workspace_bytes(n), s);
    if (e != cudaSuccess) return e;
    const size_t smem = compute_l2_smem(n);
    if (layout == QZ_SF_SWIZZLED_128x4)
        nvfp4_compute_l2_kernel<QZ_SF_SWIZZLED_128x4><<<grid, kThreads, smem, s>>>(table, n, ws, d_err);
    else
        nvfp4_compute_l2_kernel<QZ_SF_LINEAR><<<grid, kThreads, smem, s>>>(table, n, ws, d_err);
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
        case 3: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, amax_grouped_kernel<QZ_SF_SWIZZLED_128x4>, kThreads, smem); break;
        default: {
            const size_t big = compute_l2_smem(n);
            cudaFuncSetAttribute(nvfp4_compute_l2_kernel<QZ_SF_SWIZZLED_128x4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)big);
            cudaFuncSetAttribute(nvfp4_compute_l2_kernel<QZ_SF_LINEAR>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)big);
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, nvfp4_compute_l2_kernel<QZ_SF_SWIZZLED_128x4>, kThreads, big);
            break;
        }
    }
    return b > 0 ? b : 1;
}

}  // namespace qz

// ---------------------------------------------------------------------------
// Allocation-free variant of the L2-chunked computed-amax launch: its scratch
// is this file-scope device array instead of a caller workspace.  Every GPU
// that loads the library holds it until the process exits.
// ---------------------------------------------------------------------------
namespace qz {

static __device__ __align__(256) unsigned g_static_ws[workspace_words(kStaticWsMaxExperts)];

namespace {
std::mutex g_static_mu;
unsigned* g_static_ws_dev[kStaticWsMaxDevices] = {};
}  // namespace

// Device address of g_static_ws on the current device, looked up once per
// device (the host-side name is only a stand-in for the device copy).
cudaError_t static_workspace(unsigned** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kStaticWsMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ws_dev[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_ws);
        if (e != cudaSuccess) return e;
        g_static_ws_dev[dev] = static_cast<unsigned*>(p);
    }
    *out = g_static_ws_dev[dev];
    return cudaSuccess;
}

cudaError_t launch_nvfp4_compute_l2_static(const qz_expert* table, int n, int layout, int grid, cudaStream_t s,
                                           unsigned* d_err) {
    unsigned* ws = nullptr;
    cudaError_t e = static_workspace(&ws);
    if (e != cudaSuccess) return e;
    return launch_nvfp4_compute_l2(table, n, layout, grid, ws, s, d_err);
}

}  // namespace qz
