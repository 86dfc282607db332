// qz_rows.cu -- row-scaled NVFP4 over a split activation (sm_100a).
//
// TransformerEngine PR #3800 (Description, Changes): the concatenated
// activation is quantized once, each row with its own FP32 amax, and the
// payload, row amax and scale factors land in per-expert storage whose
// swizzled padding is independent per expert (uneven and empty splits).
//
// One warp works on one row at a time (four independent warps per CTA, a
// persistent grid).  Lane l owns the 16-element blocks l + 32i of the row (a
// row of up to 4096 elements is eight 32-byte loads per lane), held in
// registers: the row amax is a warp reduction and each block's scale is
// computed once, by its owner.  As soon as a block is quantized its registers
// are refilled with the same block of the warp's next row, so the next row
// streams in while this one is processed.  The scale bytes of four
// consecutive blocks (four consecutive lanes) leave as one 32-bit store.
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

// One warp's view of one virtual row.
struct RowRef {
    const uint16_t* x;  // row start
    uint8_t* q;         // payload row start
    uint8_t* sfrow;     // swizzled: the row's byte of scale column 0; linear: the row's first SF byte
    float* amax;        // the row's amax slot
    int kv;             // blocks per row
    bool live;          // row < rows (else a padded row of the swizzled region)
    bool a32;           // 32-byte aligned rows
    bool q8;            // payload row 8-byte aligned
};

template <int LAYOUT>
__device__ __forceinline__ RowRef row_ref(const qz_expert* table, const int* s_prefix, int n, int u) {
    const int e = find_owner(s_prefix, n, u);
    const qz_expert E = load_entry(table, e);
    RowRef r;
    const int64_t row = u - s_prefix[e];
    r.live = row < E.rows;
    r.x = static_cast<const uint16_t*>(E.x) + row * E.ld;
    r.q = static_cast<uint8_t*>(E.q) + row * (E.cols >> 1);
    r.kv = (int)(E.cols >> 4);
    if (LAYOUT == QZ_SF_SWIZZLED_128x4) {
        const int64_t col_tiles = (r.kv + 3) >> 2;
        const int rr = (int)(row & 127);
        r.sfrow = E.sf + (((row >> 7) * col_tiles) << 9) + ((((rr & 31) << 2) + (rr >> 5)) << 2);
    } else {
        r.sfrow = E.sf + row * r.kv;
    }
    r.amax = E.amax + row;
    r.a32 = ((reinterpret_cast<uintptr_t>(E.x) & 31) == 0) && ((E.ld & 15) == 0);
    r.q8 = ((reinterpret_cast<uintptr_t>(r.q)) & 7) == 0;
    return r;
}

// Block b of the row (zeros past the row).
__device__ __forceinline__ void row_block_load(const RowRef& r, int b, uint32_t (&w)[8]) {
    if (b < r.kv) {
        if (r.a32) ld_stream_32(r.x + b * 16, w);
        else ld_pair_16(r.x + b * 16, w);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = 0u;
    }
}

// The lane's register-resident block i (lane + 32 i) of a live row with kv <= 256.
__device__ __forceinline__ void row_load_resident(const RowRef& r, int i, int lane, uint32_t (&w)[8]) {
    if (r.live && r.kv <= kRowMaxResident) {
        row_block_load(r, lane + 32 * i, w);
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) w[k] = 0u;
    }
}

// Store the scale group of blocks k0..k0+3 (k0 % 4 == 0), bytes in `word`.
template <int LAYOUT>
__device__ __forceinline__ void store_scale_group(const RowRef& r, int k0, uint32_t word) {
    if (LAYOUT == QZ_SF_SWIZZLED_128x4) {
        if (k0 < ((r.kv + 3) & ~3)) st_u32(r.sfrow + ((k0 >> 2) << 9), word);
    } else {
        uint8_t* p = r.sfrow + k0;
        if (k0 + 4 <= r.kv && (((uintptr_t)p) & 3) == 0) {
            st_u32(p, word);
        } else {
            for (int j = 0; j < 4 && k0 + j < r.kv; ++j) p[j] = (uint8_t)(word >> (8 * j));
        }
    }
}

// Quantize block b (words w) with its scale blk; four consecutive lanes'
// scale bytes leave as one store (all lanes call this).
template <int LAYOUT>
__device__ __forceinline__ void row_block_store(const RowRef& r, int b, const uint32_t (&w)[8], Nvfp4Block blk,
                                                int lane) {
    const uint32_t c0 = e2m1x8_words(w[0], w[1], w[2], w[3], blk.rcp);
    const uint32_t c1 = e2m1x8_words(w[4], w[5], w[6], w[7], blk.rcp);
    if (b < r.kv) {
        if (r.q8) {
            st_v2(r.q + b * 8, c0, c1);
        } else {
            st_u32(r.q + b * 8, c0);
            st_u32(r.q + b * 8 + 4, c1);
        }
    }
    const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, blk.scale, 1);
    const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, blk.scale, 2);
    const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, blk.scale, 3);
    if ((lane & 3) == 0) store_scale_group<LAYOUT>(r, b, blk.scale | (s1 << 8) | (s2 << 16) | (s3 << 24));
}

template <int LAYOUT>
__device__ __forceinline__ void row_block_quant(const RowRef& r, int b, const uint32_t (&w)[8], uint32_t m, float S,
                                                const float* inv, int lane) {
    row_block_store<LAYOUT>(r, b, w, nvfp4_block(bits_to_float_bf16(m), S, inv), lane);
}

__device__ __forceinline__ uint32_t warp_max(uint32_t m) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    return m;
}

template <int LAYOUT>
__global__ void __launch_bounds__(kRowThreads) nvfp4_rows_kernel(const qz_expert* __restrict__ table, int n,
                                                                 unsigned* d_err) {
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    __shared__ float s_inv[16];
    fill_inv_table(s_inv);
    const int total = block_prefix(n, s_prefix, s_scan, RowUnits<LAYOUT>{table, d_err}, d_err);  // has barriers
    const int lane = threadIdx.x & 31;
    const int stride = gridDim.x * kRowWarps;
    int u = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
    if (u >= total) return;
    RowRef cur = row_ref<LAYOUT>(table, s_prefix, n, u);
    uint32_t w[kRowBlocksPerLane][8];
#pragma unroll
    for (int i = 0; i < kRowBlocksPerLane; ++i) row_load_resident(cur, i, lane, w[i]);
    for (;;) {
        const int un = u + stride;
        const bool more = un < total;
        const RowRef nxt = more ? row_ref<LAYOUT>(table, s_prefix, n, un) : cur;
        if (!cur.live) {
            // padded row of the swizzled region: zero scale bytes only
            const int kvp = (cur.kv + 3) & ~3;
            for (int k0 = 4 * lane; k0 < kvp; k0 += 128) st_u32(cur.sfrow + ((k0 >> 2) << 9), 0u);
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
            const float S = nvfp4_encode_scale(A);
            const int nbp = (cur.kv + 3) & ~3;
            // all block scales first: eight independent chains for the scheduler
            Nvfp4Block blk[kRowBlocksPerLane];
#pragma unroll
            for (int i = 0; i < kRowBlocksPerLane; ++i) blk[i] = nvfp4_block(bits_to_float_bf16(bm[i]), S, s_inv);
#pragma unroll
            for (int i = 0; i < kRowBlocksPerLane; ++i) {
                if (32 * i < nbp) row_block_store<LAYOUT>(cur, lane + 32 * i, w[i], blk[i], lane);  // uniform
                // refill with the next row's block as soon as this one is consumed
                if (more) row_load_resident(nxt, i, lane, w[i]);
            }
        } else {
            // long row: amax pass, then a quantize pass re-reading the row
            uint32_t m = 0;
            for (int b = lane; b < cur.kv; b += 32) {
                uint32_t v[8];
                row_block_load(cur, b, v);
                m = max(m, absmax_words<8>(v));
            }
            const float A = bits_to_float_bf16(warp_max(m));
            if (lane == 0) *cur.amax = A;
            const float S = nvfp4_encode_scale(A);
            const int nbp = (cur.kv + 3) & ~3;
            for (int b0 = 0; b0 < nbp; b0 += 32) {
                uint32_t v[8];
                row_block_load(cur, b0 + lane, v);
                row_block_quant<LAYOUT>(cur, b0 + lane, v, absmax_words<8>(v), S, s_inv, lane);
            }
            if (more) {
#pragma unroll
                for (int i = 0; i < kRowBlocksPerLane; ++i) row_load_resident(nxt, i, lane, w[i]);
            }
        }
        if (!more) break;
        cur = nxt;
        u = un;
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
