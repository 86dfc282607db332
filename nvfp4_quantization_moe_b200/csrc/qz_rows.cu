// qz_rows.cu -- row-scaled NVFP4 over a split activation (sm_100a).
//
// TransformerEngine PR #3800 (Description, Changes): the concatenated
// activation is quantized once, each row with its own FP32 amax, and the
// payload, row amax and scale factors land in per-expert storage whose
// swizzled padding is independent per expert (uneven and empty splits).
//
// One warp per row.  Rows of up to 4096 elements are brought into shared
// memory by one bulk (TMA) copy each: each of the 12 warps of a CTA keeps
// kRowDepth rows in flight in its own ring of shared-memory slots, each slot
// with an mbarrier that the copy completes, so HBM streams while the warp
// quantizes.  The warp reads the slot twice (row amax, then quantization), so
// few registers are live and many warps fit on an SM.  In the quantize pass a
// lane takes one 16-element block at a time, so each block scale is computed
// once, and the scale bytes of four consecutive blocks (four consecutive
// lanes) leave as one 32-bit store.  Longer rows take a two-pass path
// straight from global memory.
//
// Units of work are "virtual rows": an expert owns rows (linear layout) or
// pad(rows, 128) virtual rows (swizzled); a virtual row past the last live row
// writes its zero scale bytes, so no memset of the SF region is needed
// (TensorRT-LLM "MXFP8 carrier and quantize folds", commits 3 and 6).
#include "qz_device.cuh"

namespace qz {

constexpr int kRowChunks = 16;                  // 16-byte chunks per lane for a 4096-element row
constexpr int kRowSlot = 32 * kRowChunks * 16;  // bytes of one shared-memory row slot (8 KiB)
constexpr int kRowDepth = 2;                    // rows in flight per warp
constexpr int kRowWarps = 12;                   // warps per CTA
constexpr int kRowThreads = 32 * kRowWarps;
constexpr int kRowBarBytes = 1024;              // mbarrier area at the start of shared memory
constexpr size_t kRowRingBytes = (size_t)kRowWarps * kRowDepth * kRowSlot;
constexpr size_t kRowStashBytes = (size_t)kRowWarps * (kRowSlot / 32) * sizeof(uint16_t);  // block amax per warp

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
__device__ __forceinline__ void store_scale_group(const qz_expert& E, int64_t row, int64_t k0, int64_t kv,
                                                  uint32_t word) {
    if (LAYOUT == QZ_SF_SWIZZLED_128x4) {
        if (k0 < pad_to(kv, 4)) st_u32(E.sf + swz_offset(row, k0, kv), word);
    } else {
        const int64_t base = row * kv + k0;
        if (k0 + 4 <= kv && (base & 3) == 0 && (((uintptr_t)E.sf) & 3) == 0) {
            st_u32(E.sf + base, word);
        } else {
            for (int j = 0; j < 4 && k0 + j < kv; ++j) E.sf[base + j] = (uint8_t)(word >> (8 * j));
        }
    }
}

// Quantize blocks b0 .. b0+31 of a row, lane l taking block b = b0 + l whose
// two chunks are v0, v1 (zeros past the row) and whose amax has bf16 bits m.
// The scale bytes of four consecutive blocks (lanes 4g .. 4g+3) leave as one
// 32-bit store.
template <int LAYOUT>
__device__ __forceinline__ void row_blocks(const qz_expert& E, int64_t row, uint8_t* qrow, bool q8, int64_t b,
                                           int64_t kv, uint4 v0, uint4 v1, uint32_t m, float S, const float* inv,
                                           int lane) {
    const Nvfp4Block blk = nvfp4_block(bits_to_float_bf16(m), S, inv);
    const uint32_t c0 = e2m1x8_scaled(v0, blk.rcp);
    const uint32_t c1 = e2m1x8_scaled(v1, blk.rcp);
    if (b < kv) {
        if (q8) {
            st_v2(qrow + b * 8, c0, c1);
        } else {
            st_u32(qrow + b * 8, c0);
            st_u32(qrow + b * 8 + 4, c1);
        }
    }
    const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, blk.scale, 1);
    const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, blk.scale, 2);
    const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, blk.scale, 3);
    if ((lane & 3) == 0) store_scale_group<LAYOUT>(E, row, b, kv, blk.scale | (s1 << 8) | (s2 << 16) | (s3 << 24));
}

// A row of at most 4096 elements staged in shared memory.  Amax pass: lane l
// reads chunks l + 32i (conflict-free), pairs of lanes combine a block's two
// chunks and the block amax goes to the warp's stash (bf16 bits per block).
// Quantize pass: one 16-element block per lane, its amax from the stash.
template <int LAYOUT>
__device__ __forceinline__ void row_from_slot(const qz_expert& E, int64_t row, const uint8_t* slot, uint16_t* stash,
                                              const float* inv, int lane) {
    const int nch = (int)(E.cols >> 3), kv = (int)(E.cols >> 4);
    const int nbp = (int)pad_to(kv, 4);  // blocks whose scale bytes exist (incl. padding)
    uint32_t m = 0;
#pragma unroll 4
    for (int c0 = 0; c0 < nch; c0 += 32) {  // nch is even: a block's chunks are both live or both not
        const int c = c0 + lane;
        uint32_t cm = c < nch ? absmax_bits(lds128(slot + c * 16)) : 0u;
        cm = max(cm, __shfl_xor_sync(0xFFFFFFFFu, cm, 1));
        if ((lane & 1) == 0 && c < nch) stash[c >> 1] = (uint16_t)cm;
        m = max(m, cm);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __syncwarp();
    const float A = bits_to_float_bf16(m);
    if (lane == 0) E.amax[row] = A;
    const float S = nvfp4_encode_scale(A);
    uint8_t* qrow = static_cast<uint8_t*>(E.q) + row * (E.cols >> 1);
    const bool q8 = (((uintptr_t)qrow) & 7) == 0;
#pragma unroll 2
    for (int b0 = 0; b0 < nbp; b0 += 32) {
        const int b = b0 + lane;
        uint4 v0 = make_uint4(0, 0, 0, 0), v1 = make_uint4(0, 0, 0, 0);
        uint32_t bm = 0;
        if (b < kv) {
            v0 = lds128(slot + b * 32);
            v1 = lds128(slot + b * 32 + 16);
            bm = stash[b];
        }
        row_blocks<LAYOUT>(E, row, qrow, q8, b, kv, v0, v1, bm, S, inv, lane);
    }
}

// A row of any length straight from global memory: amax pass, then a
// quantize pass re-reading the row (served by L2).
template <int LAYOUT>
__device__ __forceinline__ void row_two_pass(const qz_expert& E, int64_t row, const float* inv, int lane) {
    const int64_t nch = E.cols >> 3, kv = E.cols >> 4, nbp = pad_to(kv, 4);
    const uint16_t* xr = static_cast<const uint16_t*>(E.x) + row * E.ld;
    uint32_t m = 0;
    for (int64_t c = lane; c < nch; c += 32) m = max(m, absmax_bits(ld_stream(xr + c * 8)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const float A = bits_to_float_bf16(m);
    if (lane == 0) E.amax[row] = A;
    const float S = nvfp4_encode_scale(A);
    uint8_t* qrow = static_cast<uint8_t*>(E.q) + row * (E.cols >> 1);
    const bool q8 = (((uintptr_t)qrow) & 7) == 0;
    for (int64_t b0 = 0; b0 < nbp; b0 += 32) {
        const int64_t b = b0 + lane;
        uint4 v0 = make_uint4(0, 0, 0, 0), v1 = make_uint4(0, 0, 0, 0);
        if (b < kv) {
            v0 = ld_stream(xr + b * 16);
            v1 = ld_stream(xr + b * 16 + 8);
        }
        row_blocks<LAYOUT>(E, row, qrow, q8, b, kv, v0, v1, max(absmax_bits(v0), absmax_bits(v1)), S, inv, lane);
    }
}

// Zero scale bytes of a padded row of the swizzled region.
__device__ __forceinline__ void row_zero_scales(const qz_expert& E, int64_t row, int lane) {
    const int64_t kv = E.cols >> 4;
    for (int64_t k0 = 4 * lane; k0 < pad_to(kv, 4); k0 += 128) st_u32(E.sf + swz_offset(row, k0, kv), 0u);
}

struct RowRef {
    qz_expert E;
    int64_t row;
};

__device__ __forceinline__ RowRef row_ref(const qz_expert* table, const int* s_prefix, int n, int u) {
    const int e = find_owner(s_prefix, n, u);
    RowRef r;
    r.E = load_entry(table, e);
    r.row = u - s_prefix[e];
    return r;
}

template <int LAYOUT>
__global__ void __launch_bounds__(kRowThreads, 1) nvfp4_rows_kernel(const qz_expert* __restrict__ table, int n,
                                                                 unsigned* d_err) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    uint8_t* ring = smem + kRowBarBytes;
    uint16_t* stash_all = reinterpret_cast<uint16_t*>(ring + kRowRingBytes);
    int* s_prefix = reinterpret_cast<int*>(ring + kRowRingBytes + kRowStashBytes);
    __shared__ long long s_scan[33];
    __shared__ float s_inv[16];
    fill_inv_table(s_inv);
    if (threadIdx.x < kRowWarps * kRowDepth) mbar_init(&bars[threadIdx.x], 1);
    mbar_init_fence();
    const int total = block_prefix(n, s_prefix, s_scan, RowUnits<LAYOUT>{table, d_err}, d_err);  // has barriers
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int stride = gridDim.x * kRowWarps;
    const int first = blockIdx.x * kRowWarps + w;
    uint8_t* slots = ring + (size_t)w * kRowDepth * kRowSlot;
    uint64_t* my_bars = bars + w * kRowDepth;
    uint16_t* stash = stash_all + w * (kRowSlot / 32);
    unsigned issued = 0, phase = 0;  // per-slot bits, identical in every lane

    // start the copy of unit u into slot s when it is a live row that fits a slot
    auto issue = [&](long long u, int s) {
        issued &= ~(1u << s);
        if (u >= total) return;
        const RowRef r = row_ref(table, s_prefix, n, (int)u);
        const uint32_t bytes = (uint32_t)(r.E.cols * 2);
        if (r.row >= r.E.rows || bytes > (uint32_t)kRowSlot) return;
        if (lane == 0) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&my_bars[s], bytes);
            bulk_load(slots + s * kRowSlot, static_cast<const uint16_t*>(r.E.x) + r.row * r.E.ld, bytes, &my_bars[s]);
        }
        issued |= 1u << s;
    };

#pragma unroll
    for (int s = 0; s < kRowDepth; ++s) issue((long long)first + (long long)s * stride, s);

    for (int i = 0;; ++i) {
        const long long u = (long long)first + (long long)i * stride;
        if (u >= total) break;
        const int s = i % kRowDepth;
        const RowRef r = row_ref(table, s_prefix, n, (int)u);
        if (r.row >= r.E.rows) {
            row_zero_scales(r.E, r.row, lane);
        } else if ((issued >> s) & 1u) {
            if (!mbar_wait_bounded(&my_bars[s], (phase >> s) & 1u)) {
                if (lane == 0 && d_err) atomicOr(d_err, QZ_DERR_TIMEOUT);
                break;
            }
            phase ^= 1u << s;
            row_from_slot<LAYOUT>(r.E, r.row, slots + s * kRowSlot, stash, s_inv, lane);
        } else {
            row_two_pass<LAYOUT>(r.E, r.row, s_inv, lane);
        }
        __syncwarp();  // every lane is done with slot s before it is refilled
        issue(u + (long long)kRowDepth * stride, s);
    }
    // drain: copies still in flight (units past a timeout) complete before exit
#pragma unroll
    for (int s = 0; s < kRowDepth; ++s)
        if ((issued >> s) & 1u) {
            if (!mbar_wait_bounded(&my_bars[s], (phase >> s) & 1u) && lane == 0 && d_err) atomicOr(d_err, QZ_DERR_TIMEOUT);
            phase ^= 1u << s;
            issued &= ~(1u << s);
        }
}

size_t rows_smem_bytes(int n) {
    return kRowBarBytes + kRowRingBytes + kRowStashBytes + (size_t)(n + 1) * sizeof(int);
}

cudaError_t launch_nvfp4_rows(const qz_expert* table, int n, int layout, int grid, cudaStream_t s, unsigned* d_err) {
    const size_t smem = rows_smem_bytes(n);
    if (layout == QZ_SF_SWIZZLED_128x4)
        nvfp4_rows_kernel<QZ_SF_SWIZZLED_128x4><<<grid, kRowThreads, smem, s>>>(table, n, d_err);
    else
        nvfp4_rows_kernel<QZ_SF_LINEAR><<<grid, kRowThreads, smem, s>>>(table, n, d_err);
    return cudaGetLastError();
}

// Opt the row kernels into their shared-memory size; returns resident CTAs per SM.
int rows_blocks_per_sm(int n) {
    const size_t smem = rows_smem_bytes(QZ_MAX_EXPERTS);
    cudaFuncSetAttribute(nvfp4_rows_kernel<QZ_SF_SWIZZLED_128x4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(nvfp4_rows_kernel<QZ_SF_LINEAR>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int b = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, nvfp4_rows_kernel<QZ_SF_SWIZZLED_128x4>, kRowThreads,
                                                  rows_smem_bytes(n));
    return b > 0 ? b : 1;
}

}  // namespace qz
