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

// Programmatic dependent launch (PTX griddepcontrol, sm_90+).  The tile
// kernels are launched with programmatic stream serialization: each CTA
// allows the next such launch on the stream to start as soon as it begins,
// and -- unless the call was declared independent of the work before it --
// waits for the preceding grid to complete (and its writes to be visible)
// before it reads anything.  Without a preceding trigger both are no-ops.
__device__ __forceinline__ void pdl_allow_next() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_prior() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <int FMT, int LAYOUT>
__global__ void __launch_bounds__(kThreads, 3) grouped_tile_kernel(const qz_expert* __restrict__ table, int n,
                                                                   unsigned* d_err, int wait_prior) {
    using G = TileGeo<FMT>;
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    __shared__ __align__(16) uint8_t s_sf[kThreads / 32][64 * G::kSfTiles];
    __shared__ float s_inv[16];
    constexpr bool kAmax = FMT == QZ_FMT_NVFP4;
    pdl_allow_next();
    if (wait_prior) pdl_wait_prior();
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
// running maximum while its tiles stay in one expert and folds it into the
// CTA's per-expert maximum in shared memory; at the end the CTA publishes one
// atomic max per expert it touched (non-negative floats order like their bit
// patterns).  Folding in shared memory first keeps the global atomics to one
// per CTA and expert: amax slots of many experts often share a few cache
// lines, where atomics from every warp would serialize.
template <int LAYOUT>
__global__ void __launch_bounds__(kThreads, 3) amax_grouped_kernel(const qz_expert* __restrict__ table, int n,
                                                                   unsigned* d_err) {
    using G = TileGeo<QZ_FMT_NVFP4>;
    extern __shared__ int s_prefix[];
    unsigned* s_amax = reinterpret_cast<unsigned*>(s_prefix + (n + 1));  // n words
    __shared__ long long s_scan[33];
    for (int i = threadIdx.x; i < n; i += blockDim.x) s_amax[i] = 0u;  // published by block_prefix's barriers
    const int total = block_prefix(n, s_prefix, s_scan, TableTiles<QZ_FMT_NVFP4, LAYOUT, true>{table, d_err}, d_err);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int tile = blockIdx.x;
    if (tile < total) {
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
                if (lane == 0 && run != 0u) atomicMax(s_amax + cur.expert, run << 16);
                run = 0;
            }
            if (!more) break;
            cur = nxt;
            tile = next;
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const unsigned m = s_amax[i];
        if (m != 0u) atomicMax(reinterpret_cast<unsigned int*>(load_entry(table, i).amax), m);
    }
}

// ---------------------------------------------------------------------------
// NVFP4 with a computed per-tensor amax in one launch: bulk copies feed the
// amax side from HBM ahead of the quantize warps, which re-read from L2
//
// A tensor's encode scale needs the amax of the whole tensor, so no element
// of an expert can be quantized before all of it has been read.  Every CTA
// (one per SM, all resident: a cooperative launch) runs
//  - a producer warp whose lane i feeds stage i of a ring of kStages
//    shared-memory stages: it walks its share of this CTA's amax units (units
//    b, b + grid, ... of the call; a unit is up to 32 KB of one expert: a
//    block of whole rows, or one 16384-column segment of a row) and copies
//    each into the stage with cp.async.bulk (the copy engine moves the bytes;
//    no register holds them in flight), completion counted in bytes on the
//    stage's mbarrier -- the lanes work independently, so no unit waits for
//    another stage's bookkeeping;
//  - kStages consumer warps (consumer i takes stage i): the unit's largest
//    magnitude from shared memory, folded into the CTA's maximum of its
//    expert (shared memory); the consumer that folds the CTA's last unit of
//    an expert queues the expert for
//  - a publisher warp, which takes the finished experts in batches of up to
//    32: the CTA's maxima into the experts' amax words (atomic max of bf16
//    magnitude bits), one fence, then the CTA's unit counts -- so no stage
//    ever waits for a fence;
//  - kQWarps quantize warps (the tile walk of the grouped kernel: 8 warps own
//    the row groups of a 128 x 128 tile) that take tiles b, b + grid, ... and
//    quantize each once its expert's unit counter is complete (a bounded
//    acquire wait), re-reading the input from L2 with loads that release the
//    lines.
// The producer copies a unit only while its expert starts within kWindowTiles
// tiles of this CTA's quantize front, so about kWindowTiles tiles plus one
// expert stay live in L2 (an expert whose first tile is inside the window is
// always admitted whole, so the quantize warps can never wait on a unit the
// window holds back).  Every wait is bounded by a time limit; when one runs
// out the kernel reports QZ_DERR_TIMEOUT, raises an abort word that ends the
// other waits early, lets the copies it issued land, and returns.
//
// Workspace (caller's device memory, zeroed by the call):
//   ws[0] abort word; ws[8 + e] units of expert e folded into its amax;
//   ws[8 + kMaxChunks + e] expert e's amax (bf16 magnitude bits << 16).
// ---------------------------------------------------------------------------

constexpr int kQGroups = 2;            // quantize groups: each walks its own tiles
constexpr int kQWarps = 8 * kQGroups;  // quantize warps: 8 per group (the 8 row groups of a tile)
constexpr int kStages = 4;             // shared-memory stages of the amax ring (one consumer warp each)
constexpr int kUnitBytes = 32768;      // bytes of one amax unit (one stage)
constexpr int kWindowTiles = 1536;     // how far (in tiles, ~48 MB) the copies may run ahead
constexpr int kPipeThreads = 32 * (kQWarps + 1 + kStages + 1);  // + producer, consumers, publisher
constexpr int kMaxChunks = 4096;       // workspace words reserved for the per-expert unit counters
constexpr int kWsHeader = 8;
constexpr long long kDefaultWaitNs = 20LL * 1000 * 1000;  // 20 ms: far above any legitimate wait
static_assert(QZ_MAX_EXPERTS <= kMaxChunks, "one unit counter per expert");

__host__ __device__ constexpr size_t workspace_words(int n) { return (size_t)kWsHeader + kMaxChunks + (size_t)n; }

__device__ __forceinline__ long long global_ns() {
    long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// --- mbarrier and bulk-copy primitives (PTX ISA: mbarrier, cp.async.bulk) ---

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// true once the phase with the given parity has completed
__device__ __forceinline__ bool mbar_test(uint64_t* bar, unsigned parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// global -> shared bulk copy completing `bytes` on bar (16-byte aligned
// addresses, bytes a multiple of 16; the CTA is its own cluster)
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// --- amax units ---

// How an expert is cut into units of at most kUnitBytes: row blocks of krows
// whole rows, or (rows wider than a unit) row segments of seg columns.
struct UnitGeo {
    int seg;    // columns per segment (cols, or kUnitBytes / 2 for wider rows)
    int nseg;   // segments per row
    int krows;  // rows per unit
};

__device__ __forceinline__ UnitGeo unit_geo(const qz_expert& E) {
    UnitGeo g;
    const int64_t wide = kUnitBytes / 2;
    g.seg = (int)(E.cols < wide ? E.cols : wide);
    g.nseg = (int)((E.cols + g.seg - 1) / g.seg);
    g.krows = max(1, kUnitBytes / (2 * g.seg));
    return g;
}

__device__ __forceinline__ long long unit_count(const qz_expert& E) {
    const UnitGeo g = unit_geo(E);
    return ((E.rows + g.krows - 1) / g.krows) * g.nseg;
}

template <int LAYOUT>
struct TableUnits {
    const qz_expert* table;
    __device__ long long operator()(int i) const {
        const qz_expert e = load_entry(table, i);
        if (e.rows == 0 || entry_errors(e, QZ_FMT_NVFP4, LAYOUT, true)) return 0;
        return unit_count(e);
    }
};

// Warp-uniform bounded wait until every lane sees `ready()`; false when the
// time limit ran out (QZ_DERR_TIMEOUT, abort raised) or the kernel aborted.
// The CTA's abort flag (shared memory) is checked on every poll; the global
// abort word and the timer only on every 64th, so that a poll costs no
// L2 round trip of its own.
template <typename Ready>
__device__ __forceinline__ bool bounded_wait(Ready ready, volatile unsigned* abort_word, volatile int* s_abort,
                                             long long limit, unsigned* d_err, int lane, unsigned sleep_ns) {
    const long long t0 = global_ns();
    for (unsigned it = 1;; ++it) {
        if (__all_sync(0xFFFFFFFFu, ready())) return true;
        const bool rare = (it & 63u) == 0u;
        const bool aborted = *s_abort != 0 || (rare && *abort_word != 0u);
        const bool late = rare && global_ns() - t0 > limit;
        if (__any_sync(0xFFFFFFFFu, aborted || late)) {
            if (!__any_sync(0xFFFFFFFFu, aborted) && lane == 0) {
                if (d_err) atomicOr(d_err, QZ_DERR_TIMEOUT);
                *abort_word = 1u;
                *s_abort = 1;
            }
            return false;
        }
        if (sleep_ns) __nanosleep(sleep_ns);
    }
}

template <int LAYOUT>
__global__ void __launch_bounds__(kPipeThreads, 1) nvfp4_compute_pipe_kernel(
    const qz_expert* __restrict__ table, int n, unsigned* __restrict__ ws, unsigned* d_err, long long wait_ns,
    unsigned test_flags) {
    using G = TileGeo<QZ_FMT_NVFP4>;
    extern __shared__ __align__(128) unsigned char s_dyn[];
    unsigned char* s_ring = s_dyn;                                           // kStages x kUnitBytes
    int* s_prefix = reinterpret_cast<int*>(s_dyn + kStages * kUnitBytes);   // n + 1: first tile of each expert
    int* s_uprefix = s_prefix + (n + 1);                                     // n + 1: first unit of each expert
    unsigned* s_emax = reinterpret_cast<unsigned*>(s_uprefix + (n + 1));     // n: this CTA's maximum per expert
    unsigned* s_ecnt = s_emax + n;                                           // n: this CTA's units folded per expert
    volatile int* s_pubq = reinterpret_cast<volatile int*>(s_ecnt + n);      // n: experts this CTA has finished, in order
    __shared__ long long s_scan[33];
    __shared__ __align__(16) uint8_t s_sf[kQWarps][64 * G::kSfTiles];
    __shared__ float s_inv[16];
    __shared__ __align__(8) uint64_t s_full[kStages], s_empty[kStages];
    __shared__ int s_unit_expert[kStages];
    __shared__ unsigned s_unit_bytes[kStages];
    __shared__ volatile int s_qtile[kQWarps];  // quantize warp w has done this CTA's tiles below this
    __shared__ volatile int s_abort;
    __shared__ unsigned s_pubtail;  // entries pushed to s_pubq
    fill_inv_table(s_inv);
    if (threadIdx.x < kQWarps) s_qtile[threadIdx.x] = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {  // published by block_prefix's barriers
        s_emax[i] = s_ecnt[i] = 0u;
        s_pubq[i] = -1;
    }
    if (threadIdx.x == 0) s_pubtail = 0u;
    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_empty[i], 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    const int total = block_prefix(n, s_prefix, s_scan, TableTiles<QZ_FMT_NVFP4, LAYOUT, true>{table, d_err}, d_err);
    const int units = block_prefix(n, s_uprefix, s_scan, TableUnits<LAYOUT>{table}, d_err);
    if (total == 0 || units == 0) return;

    volatile unsigned* abort_word = ws;
    unsigned* counted = ws + kWsHeader;
    unsigned* amax_ws = ws + kWsHeader + kMaxChunks;
    const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grid = gridDim.x, b = blockIdx.x;
    const long long limit = wait_ns > 0 ? wait_ns : kDefaultWaitNs;

    if (wid < kQWarps) {
        // ---------------- quantize warps: group q takes tiles b + (q + kQGroups i) grid ----------------
        const int w = wid & 7;              // row group within the tile
        const int qg = wid >> 3;            // quantize group
        const int stride = grid * kQGroups;
        int t = b + qg * grid;
        if (t >= total) {
            s_qtile[wid] = total;
            return;
        }
        s_qtile[wid] = t;
        TileRef cur = tile_ref<QZ_FMT_NVFP4, LAYOUT>(table, s_prefix, n, t, w, lane);
        uint32_t v[G::kPasses][G::kWords];
#pragma unroll
        for (int p = 0; p < G::kPasses; ++p) tile_load<QZ_FMT_NVFP4, kL2First>(cur, p, v[p]);
        int ready = -1;  // the last expert whose amax is known complete
        for (;;) {
            const int t2 = t + stride;
            const bool more = t2 < total;
            const TileRef nxt = more ? tile_ref<QZ_FMT_NVFP4, LAYOUT>(table, s_prefix, n, t2, w, lane, cur.expert) : cur;
            if (cur.expert != ready) {
                const unsigned need = (unsigned)(s_uprefix[cur.expert + 1] - s_uprefix[cur.expert]);
                const unsigned* cnt = counted + cur.expert;
                if (!bounded_wait([&] { return ld_acquire_gpu(cnt) >= need; }, abort_word, &s_abort, limit, d_err,
                                  lane, 32))
                    return;
                ready = cur.expert;
            }
            // ordered after this lane's acquire of the expert's unit count
            const float A = __uint_as_float(ld_relaxed_gpu(amax_ws + cur.expert));
            const float S = nvfp4_encode_scale(A);
            const float qm = rcp_lane_quotient(S, s_inv, lane);
#pragma unroll
            for (int p = 0; p < G::kPasses; p += 2) {
                const uint32_t sc = tile_scales_nv(v[p], v[p + 1], S);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const uint32_t scq = (sc >> (8 * q)) & 0xFFu;
                    tile_pass_nv<LAYOUT>(cur, p + q, lane, v[p + q], scq, nvfp4_rcp_warp(qm, scq), s_sf[wid]);
                    if (more) tile_load<QZ_FMT_NVFP4, kL2First>(nxt, p + q, v[p + q]);
                }
            }
            if (LAYOUT == QZ_SF_SWIZZLED_128x4) tile_flush_sf<QZ_FMT_NVFP4>(cur, w, lane, s_sf[wid]);
            if (w == 0 && lane == 0) *const_cast<float*>(cur.amax) = A;
            s_qtile[wid] = more ? t2 : total;
            if (!more) return;
            cur = nxt;
            t = t2;
        }
    }

    if (wid == kQWarps) {
        // ---------------- producer: lane i < kStages feeds stage i with this CTA's units
        //                  k = i, i + kStages, ... (unit b + k grid of the call) ----------------
        const bool feeds = lane < kStages;
        int k = lane;  // this lane's next unit, counted among the CTA's units
        long long t_last = global_ns();
        bool stop = false;
        for (unsigned it = 1;; ++it) {
            const int u = b + k * grid;
            const bool pending = feeds && u < units;
            if (!__any_sync(0xFFFFFFFFu, pending)) break;
            bool issued = false;
            if (pending) {
                const int use = k / kStages;
                bool ready = use == 0 || mbar_test(&s_empty[lane], (unsigned)((use - 1) & 1));
                int e = 0;
                if (ready) {
                    e = find_owner(s_uprefix, n, u);
                    int lo = total;
#pragma unroll
                    for (int q = 0; q < kQWarps; ++q) lo = min(lo, s_qtile[q]);
                    ready = s_prefix[e] - lo <= kWindowTiles;  // the expert starts within the window
                }
                if (ready) {
                    const qz_expert E = load_entry(table, e);
                    const UnitGeo g = unit_geo(E);
                    const int j = u - s_uprefix[e];
                    const int rb = g.nseg == 1 ? j : j / g.nseg;
                    const int64_t r0 = (int64_t)rb * g.krows;
                    const int64_t c0 = (int64_t)(j - rb * g.nseg) * g.seg;
                    const int nr = (int)min((int64_t)g.krows, E.rows - r0);
                    const int nc = (int)min((int64_t)g.seg, E.cols - c0);
                    const unsigned bytes = (unsigned)(nr * nc * 2);
                    const uint16_t* src = static_cast<const uint16_t*>(E.x) + r0 * E.ld + c0;
                    unsigned char* dst = s_ring + lane * kUnitBytes;
                    s_unit_expert[lane] = e;
                    s_unit_bytes[lane] = bytes;
                    mbar_arrive_expect_tx(&s_full[lane], bytes);  // releases the two words above
                    if (g.nseg == 1 && E.ld == E.cols) {
                        bulk_copy_g2s(dst, src, bytes, &s_full[lane]);  // whole rows, contiguous
                    } else {
                        for (int r = 0; r < nr; ++r)
                            bulk_copy_g2s(dst + r * nc * 2, src + (int64_t)r * E.ld, (unsigned)(nc * 2), &s_full[lane]);
                    }
                    k += kStages;
                    issued = true;
                }
            }
            if (__any_sync(0xFFFFFFFFu, issued)) {
                t_last = global_ns();  // the limit counts from the last progress
            } else {
                const bool rare = (it & 63u) == 0u;
                const bool aborted = s_abort != 0 || (rare && *abort_word != 0u);
                const bool late = rare && global_ns() - t_last > limit;
                if (__any_sync(0xFFFFFFFFu, aborted || late)) {
                    if (!__any_sync(0xFFFFFFFFu, aborted) && lane == 0) {
                        if (d_err) atomicOr(d_err, QZ_DERR_TIMEOUT);
                        *abort_word = 1u;
                        s_abort = 1;
                    }
                    stop = true;
                    break;
                }
                __nanosleep(32);
            }
        }
        // the copies already issued must land before the CTA can retire
        if (stop && feeds && k >= kStages) {
            const int last = k - kStages;  // this lane's last issued unit
            const long long t0 = global_ns();
            while (!mbar_test(&s_full[lane], (unsigned)((last / kStages) & 1)) && global_ns() - t0 < limit) {
            }
        }
        return;
    }

    // this CTA's units of expert e: units b + k grid inside [s_uprefix[e], s_uprefix[e + 1])
    auto mine_of = [&](int e) {
        const int u0 = s_uprefix[e] - b, u1 = s_uprefix[e + 1] - b;
        return (unsigned)(max(0, (u1 + grid - 1) / grid) - max(0, (u0 + grid - 1) / grid));
    };
    const bool withhold = (test_flags & QZ_TEST_WITHHOLD_ARRIVALS) != 0u;

    if (wid == kQWarps + 1 + kStages) {
        // ---------------- publisher: the experts this CTA has finished, in batches of up
        //                  to 32: every maximum, one fence, then every count ----------------
        int expect = 0;  // experts with at least one unit of this CTA
        for (int e = lane; e < n; e += 32) expect += mine_of(e) != 0u ? 1 : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) expect += __shfl_xor_sync(0xFFFFFFFFu, expect, o);
        int head = 0;
        long long t_last = global_ns();
        for (unsigned it = 1; head < expect; ++it) {
            const int e = head + lane < expect ? s_pubq[head + lane] : -1;
            const unsigned have = __ballot_sync(0xFFFFFFFFu, e >= 0);
            const int nb = have == 0xFFFFFFFFu ? 32 : __ffs(~have) - 1;  // the leading run of finished experts
            if (nb == 0) {
                const bool rare = (it & 63u) == 0u;
                const bool aborted = s_abort != 0 || (rare && *abort_word != 0u);
                const bool late = rare && global_ns() - t_last > limit;
                if (__any_sync(0xFFFFFFFFu, aborted || late)) {
                    if (!__any_sync(0xFFFFFFFFu, aborted) && lane == 0) {
                        if (d_err) atomicOr(d_err, QZ_DERR_TIMEOUT);
                        *abort_word = 1u;
                        s_abort = 1;
                    }
                    return;
                }
                __nanosleep(64);
                continue;
            }
            __threadfence_block();  // the queue entries were written after the experts' last folds
            if (lane < nb) {
                const unsigned m = atomicMax(s_emax + e, 0u);  // every fold of this CTA is in
                if (m != 0u) atomicMax(amax_ws + e, m);
            }
            __threadfence();  // the maxima are visible before the counts that release them
            if (lane < nb && !withhold) atomicAdd(counted + e, mine_of(e));
            __syncwarp();
            head += nb;
            t_last = global_ns();
        }
        return;
    }

    // ---------------- consumers: consumer i takes stage i (units k = i, i + kStages, ...) ----------------
    const int ci = wid - kQWarps - 1;
    const int mine = (units - b + grid - 1) / grid;  // units of this CTA
    for (int k = ci; k < mine; k += kStages) {
        uint64_t* fb = &s_full[ci];
        const unsigned par = (unsigned)((k / kStages) & 1);
        if (!bounded_wait([&] { return mbar_test(fb, par); }, abort_word, &s_abort, limit, d_err, lane, 0)) return;
        const int e = s_unit_expert[ci];
        const unsigned bytes = s_unit_bytes[ci];
        const uint4* src = reinterpret_cast<const uint4*>(s_ring + ci * kUnitBytes);
        uint32_t m0 = 0u, m1 = 0u;
        const unsigned chunks = bytes >> 4;  // 16-byte chunks (bytes is a multiple of 32)
        unsigned i = lane;
        for (; i + 32 < chunks; i += 64) {
            const uint4 a = src[i], c = src[i + 32];
            m0 = max_abs_bf16x2(max_abs_bf16x2(m0, a.x), max_abs_bf16x2(a.y, max_abs_bf16x2(a.z, a.w)));
            m1 = max_abs_bf16x2(max_abs_bf16x2(m1, c.x), max_abs_bf16x2(c.y, max_abs_bf16x2(c.z, c.w)));
        }
        if (i < chunks) {
            const uint4 a = src[i];
            m0 = max_abs_bf16x2(max_abs_bf16x2(m0, a.x), max_abs_bf16x2(a.y, max_abs_bf16x2(a.z, a.w)));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[ci]);  // the stage may be refilled
        uint32_t r = larger_half(max_abs_bf16x2(m0, m1));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) r = max(r, __shfl_xor_sync(0xFFFFFFFFu, r, o));
        if (lane == 0) {
            // fold into this CTA's maximum of expert e; the consumer that folds
            // the CTA's last unit of e hands the expert to the publisher
            atomicMax(s_emax + e, r << 16);
            __threadfence_block();
            if (atomicAdd(s_ecnt + e, 1u) + 1u == mine_of(e)) {
                __threadfence_block();
                s_pubq[atomicAdd(&s_pubtail, 1u)] = e;
            }
        }
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
size_t amax_smem(int n) { return (size_t)(2 * n + 1) * sizeof(int); }

// A tile-kernel launch with programmatic stream serialization (see
// pdl_allow_next); wait_prior = 0 only for calls declared independent.
template <int FMT, int LAYOUT>
cudaError_t launch_tiles(const qz_expert* table, int n, int grid, cudaStream_t s, unsigned* d_err, int wait_prior) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = prefix_smem(n);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, grouped_tile_kernel<FMT, LAYOUT>, table, n, d_err, wait_prior);
}

cudaError_t launch_mxfp8(const qz_expert* table, int n, int layout, int grid, cudaStream_t s, unsigned* d_err,
                         bool independent) {
    const int wait = independent ? 0 : 1;
    if (layout == QZ_SF_SWIZZLED_128x4)
        return launch_tiles<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4>(table, n, grid, s, d_err, wait);
    return launch_tiles<QZ_FMT_MXFP8, QZ_SF_LINEAR>(table, n, grid, s, d_err, wait);
}

cudaError_t launch_nvfp4_tensor(const qz_expert* table, int n, int layout, bool compute_amax, int grid,
                                cudaStream_t s, unsigned* d_err, bool independent) {
    if (compute_amax) {
        amax_clear_kernel<<<(n + kThreads - 1) / kThreads, kThreads, 0, s>>>(table, n, layout);
        if (layout == QZ_SF_SWIZZLED_128x4)
            amax_grouped_kernel<QZ_SF_SWIZZLED_128x4><<<grid, kThreads, amax_smem(n), s>>>(table, n, d_err);
        else
            amax_grouped_kernel<QZ_SF_LINEAR><<<grid, kThreads, amax_smem(n), s>>>(table, n, d_err);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // the quantize pass of a computed-amax call depends on the amax pass before it
    const int wait = (independent && !compute_amax) ? 0 : 1;
    if (layout == QZ_SF_SWIZZLED_128x4)
        return launch_tiles<QZ_FMT_NVFP4, QZ_SF_SWIZZLED_128x4>(table, n, grid, s, d_err, wait);
    return launch_tiles<QZ_FMT_NVFP4, QZ_SF_LINEAR>(table, n, grid, s, d_err, wait);
}

size_t workspace_bytes(int n) { return workspace_words(n) * sizeof(unsigned); }

size_t compute_pipe_smem(int n) { return (size_t)kStages * kUnitBytes + (size_t)(5 * n + 2) * sizeof(int); }

// One cooperative launch of the computed-amax pipeline on a zeroed workspace
// (every CTA resident: a quantize warp waits on amax warps of every CTA).
cudaError_t launch_nvfp4_compute_l2(const qz_expert* table, int n, int layout, int grid, unsigned* ws,
                                    cudaStream_t s, unsigned* d_err, long long wait_ns, unsigned test_flags) {
    cudaError_t e = cudaMemsetAsync(ws, 0, workspace_bytes(n), s);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kPipeThreads);
    cfg.dynamicSmemBytes = compute_pipe_smem(n);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (layout == QZ_SF_SWIZZLED_128x4)
        return cudaLaunchKernelEx(&cfg, nvfp4_compute_pipe_kernel<QZ_SF_SWIZZLED_128x4>, table, n, ws, d_err, wait_ns,
                                  test_flags);
    return cudaLaunchKernelEx(&cfg, nvfp4_compute_pipe_kernel<QZ_SF_LINEAR>, table, n, ws, d_err, wait_ns, test_flags);
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
        case 3: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, amax_grouped_kernel<QZ_SF_SWIZZLED_128x4>, kThreads, amax_smem(n)); break;
        default: {
            const size_t big = compute_pipe_smem(n);
            cudaFuncSetAttribute(nvfp4_compute_pipe_kernel<QZ_SF_SWIZZLED_128x4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)big);
            cudaFuncSetAttribute(nvfp4_compute_pipe_kernel<QZ_SF_LINEAR>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)big);
            int b2 = 1;
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, nvfp4_compute_pipe_kernel<QZ_SF_SWIZZLED_128x4>, kPipeThreads, big);
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b2, nvfp4_compute_pipe_kernel<QZ_SF_LINEAR>, kPipeThreads, big);
            b = min(b, b2);  // a cooperative grid must fit resident for both instantiations
            break;
        }
    }
    return b > 0 ? b : 1;
}

}  // namespace qz

// ---------------------------------------------------------------------------
// Allocation-free variant of the single-launch computed-amax path: its scratch
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
                                           unsigned* d_err, long long wait_ns, unsigned test_flags) {
    unsigned* ws = nullptr;
    cudaError_t e = static_workspace(&ws);
    if (e != cudaSuccess) return e;
    return launch_nvfp4_compute_l2(table, n, layout, grid, ws, s, d_err, wait_ns, test_flags);
}

}  // namespace qz
