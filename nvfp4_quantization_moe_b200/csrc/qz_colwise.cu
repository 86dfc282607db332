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
// One persistent launch walks all experts' 128 x 128 tiles, each CTA (MXFP8)
// or each group of 8 warps (NVFP4) a contiguous run of them (so its expert --
// the entry and the NVFP4 scale -- changes rarely), down the rows of x
// first: consecutive tiles fill consecutive pieces of the same 128
// transposed output rows, so the output leaves L2 in whole lines of few DRAM
// pages instead of 64- or 128-byte pieces of 128 different rows per tile.
// Asynchronous 16-byte copies (cp.async, zero-filled past the matrix) bring
// a tile row-major into a shared-memory stage while the tile before it is
// quantized: MXFP8 runs two CTAs per SM with three stages each and one CTA
// barrier per tile; NVFP4 runs one CTA per SM of three independent 8-warp
// groups (24 warps) with two stages each and a named barrier per group.
//   MXFP8: a thread reads one 32-bit word per row -- two neighbouring
//   columns -- for 32 rows, pairs consecutive rows of each column into bf16x2
//   words and quantizes the two 32-element column segments with the
//   library's block quantizers (include/qz_quant.cuh).
//   NVFP4: the transpose is done by ldmatrix.trans from a swizzled stage,
//   which hands each thread two whole 16-row column blocks in the same bf16x2
//   word form, four instructions for 32 elements.
// The quantized blocks go straight to the transposed payload.  NVFP4 takes
// the tensor amax as given (the row-wise computed-amax call of the same
// tensor produces it).
#include "../../include/qz_quant.cuh"
#include "qz_async.cuh"

namespace qz {

constexpr int kColThreads = 256;
constexpr int kColStages = 3;  // tiles in flight per CTA

// Per format: tile columns, CTAs per SM, and whether the stage is swizzled.
template <int FMT>
struct ColGeo {
    static constexpr int kTC = 128;
    static constexpr int kCtas = 2;
    static constexpr int kStageBytes = kTileRows * kTC * 2;  // one bf16 tile, row-major (32 / 16 KB)
    static constexpr int kBlock = FMT == QZ_FMT_MXFP8 ? 32 : 16;
};

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

// Column tiles of an expert with C columns: whole 128-column groups, so that
// the tiles also cover the swizzled layout's padded scale rows up to the next
// multiple of 128 (with 64-column tiles a group past the last column is a
// tile of zeros that writes only padding).
template <int TC>
__device__ __forceinline__ int64_t col_tiles_c(int64_t C) { return (C + 127) / 128 * (128 / TC); }

template <int FMT, int LAYOUT, int TC>
struct ColTiles {
    const qz_expert* table;
    unsigned* d_err;
    __device__ long long operator()(int i) const {
        const qz_expert e = load_entry(table, i);
        const unsigned bad = colwise_entry_errors(e, FMT, LAYOUT);
        if (bad && d_err && blockIdx.x == 0) atomicOr(d_err, bad);
        if (bad || e.rows == 0) return 0;
        return ((e.rows + kTileRows - 1) / kTileRows) * col_tiles_c<TC>(e.cols);
    }
};

// A walk over consecutive tiles of the call: the tile's expert (its entry)
// and its row / column tile, row tiles fastest.  Moving to the next tile
// reloads the entry only when the expert changes.
struct ColRef {
    const uint16_t* x;
    int64_t R, C, ld;
    uint8_t* q;
    uint8_t* sf;
    const float* amax;
    int rt, ct, nrt;
    int expert;
};

template <int TC>
__device__ __forceinline__ ColRef col_ref(const qz_expert* table, const int* s_prefix, int tile, int e) {
    while (tile >= s_prefix[e + 1]) ++e;  // tiles increase; s_prefix[n] == total > tile
    const qz_expert E = load_entry(table, e);
    const int local = tile - s_prefix[e];
    ColRef r;
    r.nrt = (int)((E.rows + kTileRows - 1) / kTileRows);
    r.ct = local / r.nrt;
    r.rt = local - r.ct * r.nrt;
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
template <int TC>
__device__ __forceinline__ void col_next(ColRef& r, const qz_expert* table, const int* s_prefix, int tile) {
    if (tile < s_prefix[r.expert + 1]) {
        if (++r.rt == r.nrt) {
            r.rt = 0;
            ++r.ct;
        }
    } else {
        r = col_ref<TC>(table, s_prefix, tile, r.expert + 1);
    }
}

// NVFP4 stages hold a tile row-major with its 16-byte chunks permuted per
// row: chunk cc of row r sits at chunk position cc ^ swz(r), swz(r) = bit 0
// of r and bits 4-5 of r as bits 1-2.  The eight rows that one ldmatrix
// reads (below) then fall into eight different bank groups.
__device__ __forceinline__ int nv_stage_swz(int r) { return (r & 1) | (((r >> 4) & 3) << 1); }

// Issue thread t's copies of a tile into a stage: chunk t % (TC / 8) (8
// columns) of rows t / (TC / 8) + (2048 / TC) k.  Rows past the matrix and
// columns past its last one are zero-filled without reading.
template <int TC, bool SWZ>
__device__ __forceinline__ void col_issue(const ColRef& r, uint32_t stage, int t) {
    constexpr int kChunks = TC / 8;                  // 16-byte chunks per tile row
    constexpr int kRowsPer = kColThreads / kChunks;  // rows per round of the CTA's threads
    const int cc = t % kChunks;
    const int64_t c = (int64_t)r.ct * TC + 8 * cc;
    const int64_t cols_left = r.C - c;
    const int cbytes = cols_left >= 8 ? 16 : (cols_left > 0 ? (int)cols_left * 2 : 0);
#pragma unroll
    for (int k = 0; k < kTileRows / kRowsPer; ++k) {
        const int row = t / kChunks + kRowsPer * k;
        const int64_t rg = (int64_t)r.rt * kTileRows + row;
        const bool in = rg < r.R && cbytes > 0;
        const void* src = in ? static_cast<const void*>(r.x + rg * r.ld + c) : static_cast<const void*>(r.x);
        const int pc = SWZ ? (cc ^ nv_stage_swz(row)) : cc;
        cp_async_16(stage + (uint32_t)(row * (TC * 2) + 16 * pc), src, in ? cbytes : 0);
    }
}

// Four 8x8 bf16 matrices from shared memory, transposed: lanes 8 m .. 8 m + 7
// give the 16-byte source rows of matrix m; register m of lane l receives the
// elements of source rows 2 (l % 4) and + 1 in column l / 4 (low half first).
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
                 : "r"(addr)
                 : "memory");
}

// MXFP8: the tile in stage s_words (128 x 128, row-major); thread (warp w,
// lane l) quantizes tile columns 64 (w % 2) + 2 l and + 1, rows 32 (w / 2) ..
// + 31 of each: one word per row holds both columns.
template <int LAYOUT>
__device__ __forceinline__ void col_tile_mx(const ColRef& cur, const uint32_t* s_words, int w, int lane) {
    constexpr int kTC = 128, kBlock = 32;
    const int ch = w & 1, rs = w >> 1;
    const int64_t R = cur.R, C = cur.C;
    const uint32_t* tw = s_words + (32 * rs) * (kTC / 2) + 32 * ch + lane;
    uint32_t xa[16], xb[16];  // column pairs (row 2i low, row 2i + 1 high) of the two columns
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t r0 = tw[(2 * i) * (kTC / 2)], r1 = tw[(2 * i + 1) * (kTC / 2)];
        xa[i] = __byte_perm(r0, r1, 0x5410);
        xb[i] = __byte_perm(r0, r1, 0x7632);
    }
    const int64_t cg = (int64_t)cur.ct * kTC + 64 * ch + 2 * lane;  // x column = transposed row
    const int64_t e0 = (int64_t)cur.rt * kTileRows + 32 * rs;       // first x row of the segment
    const int64_t cpad = LAYOUT == QZ_SF_SWIZZLED_128x4 ? ((C + 127) & ~(int64_t)127) : C;
    const int64_t kvT = R / kBlock;  // scale columns of the transposed matrix
    const int64_t kvs = LAYOUT == QZ_SF_SWIZZLED_128x4 ? ((kvT + 3) & ~(int64_t)3) : kvT;
    const int64_t k0 = e0 / kBlock;  // the segment's scale column
    uint32_t qa[8], qb[8];
    const uint32_t sa = qzq::mxfp8_block(xa, qa);
    const uint32_t sb = qzq::mxfp8_block(xb, qb);
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
    // scale bytes (a block past the last row holds zeros and gets scale 0;
    // padded transposed rows C <= cg < cpad get 0x00)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int64_t row = cg + j;
        if (row >= cpad || k0 >= kvs) continue;
        cur.sf[qzq::sf_offset(row, k0, kvT, LAYOUT)] = row < C ? (uint8_t)(j ? sb : sa) : (uint8_t)0;
    }
}

// NVFP4: the tile at stage address st (128 x TC, swizzled).  Lane 4 c + j of
// warp w holds column 8 (w + 8 u) + c of the tile (u < TC / 64) and the
// blocks of rows 16 j + 64 h .. + 15 (h = 0, 1) as 8 bf16x2 words each (word
// m = rows 2m, 2m + 1 of the block, low half first).  Matrix m of half h
// reads, in source row i (supplied by lane 8 (m % 4) + i of the x4 that
// covers it), tile row 64 h + 16 (i / 2) + 2 m + i % 2, whose swizzle is i:
// the 8 rows hit 8 bank groups.
template <int LAYOUT, int TC>
__device__ __forceinline__ void col_tile_nv(const ColRef& cur, uint32_t st, int w, int lane, float S, float qm) {
    constexpr int kBlock = 16;
    const int mi = lane & 7, mm = lane >> 3;
    const uint32_t base = st + (uint32_t)((16 * (mi >> 1) + 2 * mm + (mi & 1)) * (TC * 2) + 16 * (w ^ mi));
    const int64_t R = cur.R, C = cur.C;
    const int64_t cpad = LAYOUT == QZ_SF_SWIZZLED_128x4 ? ((C + 127) & ~(int64_t)127) : C;
    const int64_t kvT = R / kBlock;  // scale columns of the transposed matrix
    const int64_t kvs = LAYOUT == QZ_SF_SWIZZLED_128x4 ? ((kvT + 3) & ~(int64_t)3) : kvT;
    // This thread's four blocks: transposed rows cg0 + 64 u (u = 0, 1), blocks
    // starting at x row e00 + 64 h (h = 0, 1).  Their payload bytes and scale
    // bytes are affine in (u, h): payload + 64 u rows of the transposed payload
    // + 32 h bytes; scale + 8 u + 512 h (swizzled: cg0 % 128 < 64, so + 64 rows
    // stays in the 128-row group and moves two 4-row slices; + 4 scale columns
    // is the next 512-byte tile) or + 64 u kvT + 4 h (linear).
    const int64_t cg0 = (int64_t)cur.ct * TC + 8 * w + (lane >> 2);
    const int64_t e00 = (int64_t)cur.rt * kTileRows + 16 * (lane & 3);
    const int64_t k00 = e00 / kBlock;
    const int64_t qrow = R >> 1;  // payload bytes per transposed row
    uint8_t* const q0 = cur.q + cg0 * qrow + (e00 >> 1);
    int64_t s0, su, sh;
    if (LAYOUT == QZ_SF_SWIZZLED_128x4) {
        const int r = (int)(cg0 & 127);
        s0 = (((cg0 >> 7) * ((kvT + 3) >> 2) + (k00 >> 2)) << 9) + ((((r & 31) << 2) + (r >> 5)) << 2) + (k00 & 3);
        su = 8;
        sh = 512;
    } else {
        s0 = cg0 * kvT + k00;
        su = 64 * kvT;
        sh = 4;
    }
#pragma unroll
    for (int u = 0; u < TC / 64; ++u) {  // chunk w + 8 u: (w + 8 u) ^ mi == (w ^ mi) + 8 u
        uint32_t v[2][8];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int qd = 0; qd < 2; ++qd)
                ldsm_x4_trans(base + (uint32_t)(128 * u + 64 * (TC * 2) * h + 8 * (TC * 2) * qd), v[h][4 * qd],
                              v[h][4 * qd + 1], v[h][4 * qd + 2], v[h][4 * qd + 3]);
        // the tile kernels' NVFP4 arithmetic (same bytes as qzq::nvfp4_block): both
        // blocks' scales at once, element multipliers from 16 per-tile quotients
        const uint32_t two = tile_scales_nv_words(v[0], v[1], S);
        const uint32_t sc[2] = {two & 0xFFu, two >> 8};
        uint32_t c[2][2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float rcp = nvfp4_rcp_warp(qm, sc[h]);
            c[h][0] = e2m1x8_words(v[h][0], v[h][1], v[h][2], v[h][3], rcp);
            c[h][1] = e2m1x8_words(v[h][4], v[h][5], v[h][6], v[h][7], rcp);
        }
        const int64_t cg = cg0 + 64 * u;  // x column = transposed row
        if (cg < cpad) {
            const bool live = cg < C;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (live && e00 + 64 * h < R) st_v2(q0 + u * (qrow << 6) + 32 * h, c[h][0], c[h][1]);
                // scale byte (a block past the last row holds zeros and gets scale 0;
                // padded transposed rows C <= cg < cpad get 0x00)
                if (k00 + 4 * h < kvs) cur.sf[s0 + u * su + h * sh] = live ? (uint8_t)sc[h] : (uint8_t)0;
            }
        }
    }
}

template <int FMT, int LAYOUT>
__global__ void __launch_bounds__(kColThreads, ColGeo<FMT>::kCtas) colwise_kernel(const qz_expert* __restrict__ table,
                                                                                 int n, unsigned* d_err) {
    using G = ColGeo<FMT>;
    extern __shared__ __align__(16) int s_prefix[];  // [n + 1] prefix, then the stages (16-byte aligned)
    __shared__ long long s_scan[33];
    __shared__ float s_inv[16];
    if (FMT == QZ_FMT_NVFP4) fill_inv_table(s_inv);  // published by the barriers in block_prefix
    const int total = block_prefix(n, s_prefix, s_scan, ColTiles<FMT, LAYOUT, G::kTC>{table, d_err}, d_err);
    const int t = threadIdx.x;
    const uint32_t stages = (uint32_t)__cvta_generic_to_shared(s_prefix + ((n + 4) & ~3));
    const uint32_t* s_words = reinterpret_cast<const uint32_t*>(s_prefix + ((n + 4) & ~3));

    // this CTA's tiles: a contiguous run [beg, end) of the call's tiles, so the
    // expert (entry, NVFP4 scale) changes at most a few times per CTA
    const int beg = (int)((int64_t)total * blockIdx.x / gridDim.x);
    const int end = (int)((int64_t)total * (blockIdx.x + 1) / gridDim.x);
    if (beg >= end) return;
    ColRef iss = col_ref<G::kTC>(table, s_prefix, beg, find_owner(s_prefix, n, beg));  // the walk issuing copies
    ColRef cur = iss;                                                                 // the walk quantizing
    // prologue: the first kColStages - 1 tiles in flight
#pragma unroll
    for (int s = 0; s < kColStages - 1; ++s) {
        if (beg + s < end) {
            if (s > 0) col_next<G::kTC>(iss, table, s_prefix, beg + s);
            col_issue<G::kTC, FMT == QZ_FMT_NVFP4>(iss, stages + s * G::kStageBytes, t);
        }
        cp_async_commit();
    }
    const int w = t >> 5, lane = t & 31;
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
                col_next<G::kTC>(iss, table, s_prefix, ahead);
                col_issue<G::kTC, FMT == QZ_FMT_NVFP4>(iss, stages + ((k + kColStages - 1) % kColStages) * G::kStageBytes,
                                                       t);
            }
            cp_async_commit();
        }
        if (k > 0) col_next<G::kTC>(cur, table, s_prefix, tile);
        if constexpr (FMT == QZ_FMT_MXFP8) {
            col_tile_mx<LAYOUT>(cur, s_words + cur_s * (G::kStageBytes / 4), w, lane);
        } else {
            if (cur.expert != scale_expert) {
                scale_expert = cur.expert;
                S = nvfp4_encode_scale(__ldg(cur.amax));
                qm = rcp_lane_quotient(S, s_inv, lane);  // every lane: the shuffles below need all
            }
            col_tile_nv<LAYOUT, G::kTC>(cur, stages + cur_s * G::kStageBytes, w, lane, S, qm);
        }
    }
    cp_async_wait<0>();  // nothing is left in flight at exit
}

// NVFP4: one CTA per SM of three independent groups of 8 warps (24 warps per
// SM) that share the prefix table.  Each group walks its own contiguous run
// of tiles through two 32 KB stages of its own (one tile copied while the
// previous one is quantized) and synchronizes on its own named barrier, so
// the groups never wait for one another; a thread quantizes as in the
// two-CTA form, one 64-column half at a time.
constexpr int kNvGroups = 3;
constexpr int kNvGroupStages = 2;
constexpr int kNvStageBytes = kTileRows * 128 * 2;

__device__ __forceinline__ void group_barrier(int g) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "r"(kColThreads) : "memory");
}

template <int LAYOUT>
__global__ void __launch_bounds__(kColThreads * kNvGroups, 1) colwise_nv_kernel(const qz_expert* __restrict__ table,
                                                                               int n, unsigned* d_err) {
    constexpr int kTC = 128;
    extern __shared__ __align__(16) int s_prefix[];  // [n + 1] prefix, then the groups' stages
    __shared__ long long s_scan[33];
    __shared__ float s_inv[16];
    fill_inv_table(s_inv);  // published by the barriers in block_prefix
    const int total = block_prefix(n, s_prefix, s_scan, ColTiles<QZ_FMT_NVFP4, LAYOUT, kTC>{table, d_err}, d_err);
    const int g = threadIdx.x / kColThreads, t = threadIdx.x % kColThreads;
    const uint32_t stages = (uint32_t)__cvta_generic_to_shared(s_prefix + ((n + 4) & ~3)) +
                            (uint32_t)(g * kNvGroupStages * kNvStageBytes);
    // this group's tiles: a contiguous run [beg, end) of the call's tiles
    const int64_t groups = (int64_t)gridDim.x * kNvGroups, gi = (int64_t)blockIdx.x * kNvGroups + g;
    const int beg = (int)((int64_t)total * gi / groups);
    const int end = (int)((int64_t)total * (gi + 1) / groups);
    if (beg >= end) return;  // only group barriers follow
    ColRef iss = col_ref<kTC>(table, s_prefix, beg, find_owner(s_prefix, n, beg));  // the walk issuing copies
    ColRef cur = iss;                                                             // the walk quantizing
    col_issue<kTC, true>(iss, stages, t);
    cp_async_commit();
    const int w = t >> 5, lane = t & 31;
    int scale_expert = -1;
    float S = 0.0f, qm = 0.0f;
    for (int k = 0;; ++k) {
        const int tile = beg + k;
        if (tile >= end) break;
        cp_async_wait<0>();  // this thread's copies of tile k have landed
        group_barrier(g);    // ... and the group's; tile k - 1's stage is free again
        if (tile + 1 < end) {
            col_next<kTC>(iss, table, s_prefix, tile + 1);
            col_issue<kTC, true>(iss, stages + ((k + 1) & 1) * kNvStageBytes, t);
        }
        cp_async_commit();
        if (k > 0) col_next<kTC>(cur, table, s_prefix, tile);
        if (cur.expert != scale_expert) {
            scale_expert = cur.expert;
            S = nvfp4_encode_scale(__ldg(cur.amax));
            qm = rcp_lane_quotient(S, s_inv, lane);  // every lane: the shuffles below need all
        }
        col_tile_nv<LAYOUT, kTC>(cur, stages + (k & 1) * kNvStageBytes, w, lane, S, qm);
    }
    cp_async_wait<0>();  // nothing is left in flight at exit
}

size_t colwise_nv_smem(int n) {
    return (size_t)((n + 4) & ~3) * sizeof(int) + (size_t)kNvGroups * kNvGroupStages * kNvStageBytes;
}

template <int FMT>
size_t colwise_smem(int n) {
    return (size_t)((n + 4) & ~3) * sizeof(int) + (size_t)kColStages * ColGeo<FMT>::kStageBytes;
}

cudaError_t launch_colwise(const qz_expert* table, int n, int fmt, int layout, int grid, cudaStream_t s,
                           unsigned* d_err) {
    if (fmt == QZ_FMT_MXFP8) {
        const size_t smem = colwise_smem<QZ_FMT_MXFP8>(n);
        if (layout == QZ_SF_SWIZZLED_128x4)
            colwise_kernel<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4><<<grid, kColThreads, smem, s>>>(table, n, d_err);
        else
            colwise_kernel<QZ_FMT_MXFP8, QZ_SF_LINEAR><<<grid, kColThreads, smem, s>>>(table, n, d_err);
    } else {
        const size_t smem = colwise_nv_smem(n);
        if (layout == QZ_SF_SWIZZLED_128x4)
            colwise_nv_kernel<QZ_SF_SWIZZLED_128x4><<<grid, kColThreads * kNvGroups, smem, s>>>(table, n, d_err);
        else
            colwise_nv_kernel<QZ_SF_LINEAR><<<grid, kColThreads * kNvGroups, smem, s>>>(table, n, d_err);
    }
    return cudaGetLastError();
}

// Resident CTAs per SM of the format's kernel (for a one-wave persistent
// grid).  The stages plus the largest prefix table exceed 48 KB, so both
// layouts are allowed more dynamic shared memory on the current device first
// (this runs once per device and format before the first launch).
int colwise_blocks_per_sm(int n, int fmt) {
    int b = 1;
    if (fmt == QZ_FMT_MXFP8) {
        const int bytes = (int)colwise_smem<QZ_FMT_MXFP8>(QZ_MAX_EXPERTS);
        cudaFuncSetAttribute(colwise_kernel<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        cudaFuncSetAttribute(colwise_kernel<QZ_FMT_MXFP8, QZ_SF_LINEAR>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, colwise_kernel<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4>, kColThreads,
                                                      colwise_smem<QZ_FMT_MXFP8>(n));
    } else {
        const int bytes = (int)colwise_nv_smem(QZ_MAX_EXPERTS);
        cudaFuncSetAttribute(colwise_nv_kernel<QZ_SF_SWIZZLED_128x4>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        cudaFuncSetAttribute(colwise_nv_kernel<QZ_SF_LINEAR>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, colwise_nv_kernel<QZ_SF_SWIZZLED_128x4>, kColThreads * kNvGroups,
                                                      colwise_nv_smem(n));
    }
    return b > 0 ? b : 1;
}

}  // namespace qz
