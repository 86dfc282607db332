// qz_rows.cu -- row-scaled NVFP4 over a split activation (sm_100a).
//
// TransformerEngine PR #3800 (Description, Changes): the concatenated
// activation is quantized once, each row with its own FP32 amax, and the
// payload, row amax and scale factors land in per-expert storage whose
// swizzled padding is independent per expert (uneven and empty splits).
//
// One persistent 128-thread CTA works on one row at a time.  Thread t owns
// the 16-element blocks t and t + 128 of the row (a row of up to 4096
// elements is two 32-byte loads per thread), held in registers: the row amax
// is a warp reduction plus a four-word exchange in shared memory, and each
// block's scale is computed once, by its owner.  While a row is quantized,
// the CTA's next row is already being loaded into the same registers, block
// by block as they are consumed.  The scale bytes of four consecutive blocks
// (four consecutive threads) leave as one 32-bit store.  Rows longer than
// 4096 elements take a two-pass path (amax pass, then a quantize pass
// re-reading the row from L2).
//
// Units of work are "virtual rows": an expert owns rows (linear layout) or
// pad(rows, 128) virtual rows (swizzled); a virtual row past the last live row
// writes its zero scale bytes, so no memset of the SF region is needed
// (TensorRT-LLM "MXFP8 carrier and quantize folds", commits 3 and 6).
#include "qz_device.cuh"

namespace qz {

constexpr int kRowThreads = 128;
constexpr int kRowBlocksPerThread = 2;                              // register-resident blocks per thread
constexpr int kRowMaxResident = kRowThreads * kRowBlocksPerThread;  // blocks of a register-resident row

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

// Store the scale group starting at block k0 (k0 % 4 == 0), bytes in `word`.
template <int LAYOUT>
__device__ __forceinline__ void store_scale_group(uint8_t* sf, int64_t row, int64_t k0, int64_t kv, uint32_t word) {
    if (LAYOUT == QZ_SF_SWIZZLED_128x4) {
        if (k0 < pad_to(kv, 4)) st_u32(sf + swz_offset(row, k0, kv), word);
    } else {
        const int64_t base = row * kv + k0;
        if (k0 + 4 <= kv && (base & 3) == 0 && (((uintptr_t)sf) & 3) == 0) {
            st_u32(sf + base, word);
        } else {
            for (int j = 0; j < 4 && k0 + j < kv; ++j) sf[base + j] = (uint8_t)(word >> (8 * j));
        }
    }
}

// One thread's view of one virtual row.
struct RowRef {
    const uint16_t* x;  // row start
    uint8_t* q;         // payload row start
    uint8_t* sf;        // expert's SF region
    float* amax;        // expert's row amax array
    int64_t row;        // row inside the expert
    int kv;             // blocks per row
    bool live;          // row < rows (else a padded row of the swizzled region)
    bool a32;           // 32-byte aligned rows
};

__device__ __forceinline__ RowRef row_ref(const qz_expert* table, const int* s_prefix, int n, int u) {
    const int e = find_owner(s_prefix, n, u);
    const qz_expert E = load_entry(table, e);
    RowRef r;
    r.row = u - s_prefix[e];
    r.live = r.row < E.rows;
    r.x = static_cast<const uint16_t*>(E.x) + r.row * E.ld;
    r.q = static_cast<uint8_t*>(E.q) + r.row * (E.cols >> 1);
    r.sf = E.sf;
    r.amax = E.amax;
    r.kv = (int)(E.cols >> 4);
    r.a32 = ((reinterpret_cast<uintptr_t>(E.x) & 31) == 0) && ((E.ld & 15) == 0);
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

// The thread's register-resident blocks (t + 128 i) of a live row with kv <= 256.
__device__ __forceinline__ void row_load_resident(const RowRef& r, int i, uint32_t (&w)[8]) {
    if (r.live && r.kv <= kRowMaxResident) {
        row_block_load(r, (int)threadIdx.x + kRowThreads * i, w);
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) w[k] = 0u;
    }
}

// Quantize block b (words w, amax bits m) with encode scale S; four
// consecutive threads' scale bytes leave as one store (all threads call this).
template <int LAYOUT>
__device__ __forceinline__ void row_block_quant(const RowRef& r, int b, const uint32_t (&w)[8], uint32_t m, float S,
                                                const float* inv, bool q8) {
    const Nvfp4Block blk = nvfp4_block(bits_to_float_bf16(m), S, inv);
    const uint32_t c0 = e2m1x8_words(w[0], w[1], w[2], w[3], blk.rcp);
    const uint32_t c1 = e2m1x8_words(w[4], w[5], w[6], w[7], blk.rcp);
    if (b < r.kv) {
        if (q8) {
            st_v2(r.q + b * 8, c0, c1);
        } else {
            st_u32(r.q + b * 8, c0);
            st_u32(r.q + b * 8 + 4, c1);
        }
    }
    const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, blk.scale, 1);
    const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, blk.scale, 2);
    const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, blk.scale, 3);
    if ((threadIdx.x & 3) == 0)
        store_scale_group<LAYOUT>(r.sf, r.row, b, r.kv, blk.scale | (s1 << 8) | (s2 << 16) | (s3 << 24));
}

// CTA-wide maximum of m (bf16 magnitude bits): one shared word per warp,
// alternating between two sets on successive calls (`parity`), so that each
// call needs a single barrier: a set is rewritten only after the next call's
// barrier, which every thread reaches after reading it.
__device__ __forceinline__ uint32_t cta_max(uint32_t m, uint32_t (*s_max)[kRowThreads / 32], int parity) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0) s_max[parity][threadIdx.x >> 5] = m;
    __syncthreads();
    uint32_t r = 0;
#pragma unroll
    for (int k = 0; k < kRowThreads / 32; ++k) r = max(r, s_max[parity][k]);
    return r;
}

template <int LAYOUT>
__global__ void __launch_bounds__(kRowThreads) nvfp4_rows_kernel(const qz_expert* __restrict__ table, int n,
                                                                 unsigned* d_err) {
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    __shared__ float s_inv[16];
    __shared__ uint32_t s_max[2][kRowThreads / 32];
    fill_inv_table(s_inv);
    const int total = block_prefix(n, s_prefix, s_scan, RowUnits<LAYOUT>{table, d_err}, d_err);  // has barriers
    const int t = threadIdx.x;
    int u = blockIdx.x;
    if (u >= total) return;
    RowRef cur = row_ref(table, s_prefix, n, u);
    uint32_t w[kRowBlocksPerThread][8];
#pragma unroll
    for (int i = 0; i < kRowBlocksPerThread; ++i) row_load_resident(cur, i, w[i]);
    int reductions = 0;  // CTA reductions so far: their shared words alternate
    for (;;) {
        const int un = u + gridDim.x;
        const bool more = un < total;
        const RowRef nxt = more ? row_ref(table, s_prefix, n, un) : cur;
        if (!cur.live) {
            // padded row of the swizzled region: zero scale bytes only
            const int kvp = (int)pad_to(cur.kv, 4);
            for (int k0 = 4 * t; k0 < kvp; k0 += 4 * kRowThreads) st_u32(cur.sf + swz_offset(cur.row, k0, cur.kv), 0u);
            if (more) {
#pragma unroll
                for (int i = 0; i < kRowBlocksPerThread; ++i) row_load_resident(nxt, i, w[i]);
            }
        } else if (cur.kv <= kRowMaxResident) {
            uint32_t bm[kRowBlocksPerThread];
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < kRowBlocksPerThread; ++i) {
                bm[i] = absmax_words<8>(w[i]);
                m = max(m, bm[i]);
            }
            const uint32_t rowm = cta_max(m, s_max, (reductions++) & 1);
            const float A = bits_to_float_bf16(rowm);
            if (t == 0) cur.amax[cur.row] = A;
            const float S = nvfp4_encode_scale(A);
            const bool q8 = (((uintptr_t)cur.q) & 7) == 0;
            const int nbp = (int)pad_to(cur.kv, 4);
#pragma unroll
            for (int i = 0; i < kRowBlocksPerThread; ++i) {
                const int b0 = kRowThreads * i;
                if (b0 < nbp) row_block_quant<LAYOUT>(cur, b0 + t, w[i], bm[i], S, s_inv, q8);  // uniform
                // refill with the next row's block as soon as this one is consumed
                if (more) row_load_resident(nxt, i, w[i]);
            }
        } else {
            // long row: amax pass, then a quantize pass re-reading the row
            uint32_t m = 0;
            for (int b = t; b < cur.kv; b += kRowThreads) {
                uint32_t v[8];
                row_block_load(cur, b, v);
                m = max(m, absmax_words<8>(v));
            }
            const uint32_t rowm = cta_max(m, s_max, (reductions++) & 1);
            const float A = bits_to_float_bf16(rowm);
            if (t == 0) cur.amax[cur.row] = A;
            const float S = nvfp4_encode_scale(A);
            const bool q8 = (((uintptr_t)cur.q) & 7) == 0;
            const int nbp = (int)pad_to(cur.kv, 4);
            for (int b0 = 0; b0 < nbp; b0 += kRowThreads) {
                uint32_t v[8];
                row_block_load(cur, b0 + t, v);
                row_block_quant<LAYOUT>(cur, b0 + t, v, absmax_words<8>(v), S, s_inv, q8);
            }
            if (more) {
#pragma unroll
                for (int i = 0; i < kRowBlocksPerThread; ++i) row_load_resident(nxt, i, w[i]);
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
