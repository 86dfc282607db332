// qz_rows.cu -- row-scaled NVFP4 over a split activation (sm_100a).
//
// TransformerEngine PR #3800 (Description, Changes): the concatenated
// activation is quantized once, each row with its own FP32 amax, and the
// payload, row amax and scale factors land in per-expert storage whose
// swizzled padding is independent per expert (uneven and empty splits).
//
// One warp works on one row at a time (four independent warps per CTA, a
// persistent grid); each warp takes a contiguous run of rows, so consecutive
// rows mostly share an expert and its table entry.  Lane l owns the
// 16-element blocks l + 32i of the row (a row of up to 4096 elements is eight
// 32-byte loads per lane), held in registers: the row amax is a warp
// reduction and each block's scale is computed once, by its owner.  As soon
// as a block is quantized its registers are refilled with the same block of
// the warp's next row, so the next row streams in while this one is
// processed.
//
// Per row, the element multipliers RN(S / value(s)) of all 127 finite e4m3
// scale codes s are tabulated once in the warp's shared memory (four exact
// quotients per lane), so a block's multiplier is one table read.  Block
// amaxes use the packed bf16 magnitude maximum; the block scales and the
// element products run on packed f32 pairs.  The row's scale
// bytes are gathered in shared memory and leave as 32-bit stores.
// Rows longer than 4096 elements take a two-pass path (amax pass, then a
// quantize pass re-reading the row from L2).
//
// Units of work are "virtual rows": an expert owns rows (linear layout) or
// pad(rows, 128) virtual rows (swizzled); a virtual row past the last live row
// writes its zero scale bytes, so no memset of the SF region is needed
// (TensorRT-LLM "MXFP8 carrier and quantize folds", commits 3 and 6).
#include "qz_device.cuh"

namespace qz {

constexpr int kRowThreads = 128;                          // four independent warps
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kRowBlocksPerLane = 8;                      // register-resident blocks per lane
constexpr int kRowMaxResident = 32 * kRowBlocksPerLane;   // blocks of a register-resident row (4096 elements)
constexpr int kRcpCodes = 128;                            // e4m3 codes 0..127 (0x7F is never produced)

template <int LAYOUT>
struct RowUnits {
    const qz_expert* table;
    unsigned* d_err;
    __device__ long long operator()(int i) const {
        const qz_expert e = load_entry(table, i);
        const unsigned bad = entry_errors(e, QZ_FMT_NVFP4, LAYOUT, true);
        if (bad && d_err && blockIdx.x == 0) atomicOr(d_err, bad);
        if (bad || e.rows == 0) return 0;
        return LAYOUT == QZ_SF_SWIZZLED_128x4 ? pad_to(e.rows, 128) : e.rows;
    }
};

// ---------------------------------------------------------------------------
// rows
// ---------------------------------------------------------------------------

// Where a warp reads one virtual row from (all a prefetch needs).
struct RowSrc {
    const uint16_t* x;  // row start
    int kv;             // blocks per row
    bool resident;      // live row with kv <= 256: read into registers
    bool a32;           // 32-byte aligned rows
};

// One warp's view of one virtual row.
struct RowRef {
    RowSrc src;
    uint8_t* q;         // payload row start
    uint8_t* sfrow;     // swizzled: the row's byte of scale column 0; linear: the row's first SF byte
    float* amax;        // the row's amax slot
    int kv;             // blocks per row
    bool live;          // row < rows (else a padded row of the swizzled region)
    bool q8;            // payload row 8-byte aligned
};

// Row `row` of expert entry E, read side.
__device__ __forceinline__ RowSrc row_src_of(const qz_expert& E, int64_t row) {
    RowSrc r;
    r.x = static_cast<const uint16_t*>(E.x) + row * E.ld;
    r.kv = (int)(E.cols >> 4);
    r.resident = row < E.rows && r.kv <= kRowMaxResident;
    r.a32 = ((reinterpret_cast<uintptr_t>(E.x) & 31) == 0) && ((E.ld & 15) == 0);
    return r;
}

__device__ __forceinline__ RowSrc row_src_at(const qz_expert* table, int e, int64_t row) {
    return row_src_of(load_entry(table, e), row);
}

// Row `row` of expert e.
template <int LAYOUT>
__device__ __forceinline__ RowRef row_ref_at(const qz_expert* table, int e, int64_t row) {
    const qz_expert E = load_entry(table, e);
    RowRef r;
    r.src = row_src_of(E, row);
    r.live = row < E.rows;
    r.q = static_cast<uint8_t*>(E.q) + row * (E.cols >> 1);
    r.kv = r.src.kv;
    if (LAYOUT == QZ_SF_SWIZZLED_128x4) {
        const int64_t col_tiles = (r.kv + 3) >> 2;
        const int rr = (int)(row & 127);
        r.sfrow = E.sf + (((row >> 7) * col_tiles) << 9) + ((((rr & 31) << 2) + (rr >> 5)) << 2);
    } else {
        r.sfrow = E.sf + row * r.kv;
    }
    r.amax = E.amax + row;
    r.q8 = ((reinterpret_cast<uintptr_t>(r.q)) & 7) == 0;
    return r;
}

// Block b of the row (zeros past the row).
__device__ __forceinline__ void row_block_load(const RowSrc& r, int b, uint32_t (&w)[8]) {
    if (b < r.kv) {
        if (r.a32) ld_stream_32(r.x + b * 16, w);
        else ld_pair_16(r.x + b * 16, w);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = 0u;
    }
}

// The lane's register-resident block i (lane + 32 i) of a live row with kv <= 256.
__device__ __forceinline__ void row_load_resident(const RowSrc& r, int i, int lane, uint32_t (&w)[8]) {
    if (r.resident) {
        row_block_load(r, lane + 32 * i, w);
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) w[k] = 0u;
    }
}

// Payload bytes of block b (codes c0: elements 0-7, c1: 8-15).
__device__ __forceinline__ void row_payload_store(const RowRef& r, int b, uint32_t c0, uint32_t c1) {
    if (b < r.kv) {
        if (r.q8) {
            st_v2(r.q + b * 8, c0, c1);
        } else {
            st_u32(r.q + b * 8, c0);
            st_u32(r.q + b * 8 + 4, c1);
        }
    }
}

// The row's scale bytes, gathered in the warp's shared buffer `bytes`
// (pad(kv, 4) of them; entries past kv are zero), to their layout.
template <int LAYOUT>
__device__ __forceinline__ void row_scales_store(const RowRef& r, const uint32_t* words, int lane) {
    if (LAYOUT == QZ_SF_SWIZZLED_128x4) {
        // word j holds scale columns 4j..4j+3: one 32-bit store per column tile
        const int nw = (r.kv + 3) >> 2;
        for (int j = lane; j < nw; j += 32) st_u32(r.sfrow + (j << 9), words[j]);
    } else {
        const uint8_t* bytes = reinterpret_cast<const uint8_t*>(words);
        int k0 = 0;
        if ((reinterpret_cast<uintptr_t>(r.sfrow) & 3) == 0) {
            for (int j = lane; j < (r.kv >> 2); j += 32) st_u32(r.sfrow + 4 * j, words[j]);
            k0 = r.kv & ~3;
        }
        for (int k = k0 + lane; k < r.kv; k += 32) r.sfrow[k] = bytes[k];
    }
}

// Block b's quantization for the long-row path, scale bytes gathered from
// four consecutive lanes by shuffles (all lanes call this).
template <int LAYOUT>
__device__ __forceinline__ void row_block_quant(const RowRef& r, int b, const uint32_t (&w)[8], float S,
                                                const float* inv, int lane) {
    const Nvfp4Block blk = nvfp4_block(bits_to_float_bf16(absmax_words<8>(w)), S, inv);
    row_payload_store(r, b, e2m1x8_words(w[0], w[1], w[2], w[3], blk.rcp), e2m1x8_words(w[4], w[5], w[6], w[7], blk.rcp));
    const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, blk.scale, 1);
    const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, blk.scale, 2);
    const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, blk.scale, 3);
    if ((lane & 3) == 0) {
        const uint32_t word = blk.scale | (s1 << 8) | (s2 << 16) | (s3 << 24);
        if (LAYOUT == QZ_SF_SWIZZLED_128x4) {
            if (b < ((r.kv + 3) & ~3)) st_u32(r.sfrow + ((b >> 2) << 9), word);
        } else {
            uint8_t* p = r.sfrow + b;
            if (b + 4 <= r.kv && (((uintptr_t)p) & 3) == 0) {
                st_u32(p, word);
            } else {
                for (int j = 0; j < 4 && b + j < r.kv; ++j) p[j] = (uint8_t)(word >> (8 * j));
            }
        }
    }
}

__device__ __forceinline__ uint32_t warp_max(uint32_t m) { return __reduce_max_sync(0xFFFFFFFFu, m); }

// Encode scale S = RN(1 / RN(A / 2688)) of a row amax A (a bf16 value),
// zero when the decode scale is zero.  RN(A / 2688) uses the quotient
// correction of Markstein (IBM J. Res. Dev. 34(1), 1990): q0 = RN(A * RN(1/2688)),
// r = A - 2688 q0 exactly (one FMA), RN(q0 + r * RN(1/2688)).  A has 8
// significant bits and 2688 = 21 * 2^7, so A / 2688 is a multiple of an odd
// fraction k/21 of an ulp away from the representable grid and never within
// 1/42 ulp of a rounding midpoint: the correction returns the correctly
// rounded quotient (checked against IEEE division for every bf16 A >= 2^-100
// in the test suite).
__device__ __forceinline__ float row_encode_scale(float A) {
    const float c = 1.0f / 2688.0f;
    const float q0 = __fmul_rn(A, c);
    const float r = __fmaf_rn(-q0, 2688.0f, A);
    const float g = __fmaf_rn(r, c, q0);
    return g == 0.0f ? 0.0f : __frcp_rn(g);
}

// The element multiplier of every e4m3 code for encode scale S: code 0 (a
// zero block) gets 0, a subnormal quotient is flushed to zero.  Code 0x7F is
// NaN in e4m3 and never produced by the saturating conversion; its entry is
// unused.
__device__ __forceinline__ void fill_rcp_table(float* tab, float S, const float* inv, int lane) {
#pragma unroll
    for (int j = 0; j < kRcpCodes / 32; ++j) {
        const uint32_t c = (uint32_t)(lane + 32 * j);
        tab[c] = nvfp4_rcp(S, c, inv);
    }
}

template <int LAYOUT>
__global__ void __launch_bounds__(kRowThreads) nvfp4_rows_kernel(const qz_expert* __restrict__ table, int n,
                                                                 unsigned* d_err) {
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    __shared__ float s_inv[16];
    __shared__ float s_rcp[kRowWarps][kRcpCodes];
    __shared__ uint32_t s_sfw[kRowWarps][kRowMaxResident / 4];
    fill_inv_table(s_inv);
    const int total = block_prefix(n, s_prefix, s_scan, RowUnits<LAYOUT>{table, d_err}, d_err);  // has barriers
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // the warp's contiguous run of virtual rows [u, u_end)
    const long long W = (long long)gridDim.x * kRowWarps, g = (long long)blockIdx.x * kRowWarps + warp;
    int u = (int)(g * total / W);
    const int u_end = (int)((g + 1) * total / W);
    if (u >= u_end) return;  // no CTA barrier follows
    float* rcp_tab = s_rcp[warp];
    uint32_t* sfw = s_sfw[warp];
    uint8_t* sfb = reinterpret_cast<uint8_t*>(sfw);
    int e = find_owner(s_prefix, n, u);
    RowRef cur = row_ref_at<LAYOUT>(table, e, u - s_prefix[e]);
    uint32_t w[kRowBlocksPerLane][8];
#pragma unroll
    for (int i = 0; i < kRowBlocksPerLane; ++i) row_load_resident(cur.src, i, lane, w[i]);
    for (;;) {
        const int un = u + 1;
        const bool more = un < u_end;
        int en = e;
        if (more) {
            while (un >= s_prefix[en + 1]) ++en;  // s_prefix[n] == total > un
        }
        const RowSrc nxt = more ? row_src_at(table, en, un - s_prefix[en]) : cur.src;
        if (!cur.live) {
            // padded row of the swizzled region: zero scale bytes only
            const int nw = (cur.kv + 3) >> 2;
            for (int j = lane; j < nw; j += 32) st_u32(cur.sfrow + (j << 9), 0u);
            if (more) {
#pragma unroll
                for (int i = 0; i < kRowBlocksPerLane; ++i) row_load_resident(nxt, i, lane, w[i]);
            }
        } else if (cur.kv <= kRowMaxResident) {
            uint32_t bm[kRowBlocksPerLane];
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < kRowBlocksPerLane; ++i) {
                bm[i] = absmax_words<8>(w[i]);
                m = max(m, bm[i]);
            }
            const float A = bits_to_float_bf16(warp_max(m));
            if (lane == 0) *cur.amax = A;
            const float S = row_encode_scale(A);
            const int nbp = (cur.kv + 3) & ~3;
            __syncwarp();  // the previous row's table and scale-byte reads are done
            fill_rcp_table(rcp_tab, S, s_inv, lane);
            uint32_t code[kRowBlocksPerLane];
#pragma unroll
            for (int i = 0; i < kRowBlocksPerLane; i += 2) {
                const uint32_t two =
                    nvfp4_scale_pair(bits_to_float_bf16(bm[i]), bits_to_float_bf16(bm[i + 1]), S);
                code[i] = two & 0xFFu;
                code[i + 1] = two >> 8;
            }
#pragma unroll
            for (int i = 0; i < kRowBlocksPerLane; ++i)
                if (32 * i < nbp) sfb[lane + 32 * i] = (uint8_t)code[i];  // uniform
            __syncwarp();  // table and scale bytes complete
            row_scales_store<LAYOUT>(cur, sfw, lane);
#pragma unroll
            for (int i = 0; i < kRowBlocksPerLane; ++i) {
                if (32 * i < nbp) {  // uniform
                    const float rcp = rcp_tab[code[i]];
                    const uint32_t c0 = e2m1x8_words(w[i][0], w[i][1], w[i][2], w[i][3], rcp);
                    const uint32_t c1 = e2m1x8_words(w[i][4], w[i][5], w[i][6], w[i][7], rcp);
                    row_payload_store(cur, lane + 32 * i, c0, c1);
                }
                // refill with the next row's block as soon as this one is consumed
                if (more) row_load_resident(nxt, i, lane, w[i]);
            }
        } else {
            // long row: amax pass, then a quantize pass re-reading the row
            uint32_t m = 0;
            for (int b = lane; b < cur.kv; b += 32) {
                uint32_t v[8];
                row_block_load(cur.src, b, v);
                m = max(m, absmax_words<8>(v));
            }
            const float A = bits_to_float_bf16(warp_max(m));
            if (lane == 0) *cur.amax = A;
            const float S = row_encode_scale(A);
            const int nbp = (cur.kv + 3) & ~3;
            for (int b0 = 0; b0 < nbp; b0 += 32) {
                uint32_t v[8];
                row_block_load(cur.src, b0 + lane, v);
                row_block_quant<LAYOUT>(cur, b0 + lane, v, S, s_inv, lane);
            }
            if (more) {
#pragma unroll
                for (int i = 0; i < kRowBlocksPerLane; ++i) row_load_resident(nxt, i, lane, w[i]);
            }
        }
        if (!more) break;
        u = un;
        e = en;
        cur = row_ref_at<LAYOUT>(table, e, u - s_prefix[e]);
    }
}

cudaError_t launch_nvfp4_rows(const qz_expert* table, int n, int layout, int grid, cudaStream_t s, unsigned* d_err) {
    const size_t smem = (size_t)(n + 1) * sizeof(int);
    if (layout == QZ_SF_SWIZZLED_128x4)
        nvfp4_rows_kernel<QZ_SF_SWIZZLED_128x4><<<grid, kRowThreads, smem, s>>>(table, n, d_err);
    else
        nvfp4_rows_kernel<QZ_SF_LINEAR><<<grid, kRowThreads, smem, s>>>(table, n, d_err);
    return cudaGetLastError();
}

// Resident CTAs per SM (for a one-wave persistent grid).
int rows_blocks_per_sm(int n) {
    int b = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, nvfp4_rows_kernel<QZ_SF_SWIZZLED_128x4>, kRowThreads,
                                                  (size_t)(n + 1) * sizeof(int));
    return b > 0 ? b : 1;
}

}  // namespace qz
