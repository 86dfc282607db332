// qz_rows.cu -- row-scaled NVFP4 over a split activation (sm_100a).
//
// TransformerEngine PR #3800 (Description, Changes): the concatenated
// activation is quantized once, each row with its own FP32 amax, and the
// payload, row amax and scale factors land in per-expert storage whose
// swizzled padding is independent per expert (uneven and empty splits).
//
// One warp per row.  A row of up to 4096 elements stays in registers (16
// chunks of 8 bf16 per lane), so the row amax and the block scales come from a
// single read of HBM; longer rows take a second pass over the row (served by
// L2).  Lane l holds chunks l + 32i: the two chunks of a 16-element block sit
// in lanes (2j, 2j+1) and the four blocks of one 4-byte scale group in eight
// consecutive lanes, so a scale group leaves as one 32-bit store.
//
// Units of work are "virtual rows": an expert owns rows (linear layout) or
// pad(rows, 128) virtual rows (swizzled); a virtual row past the last live row
// writes its zero scale bytes, so no memset of the SF region is needed
// (TensorRT-LLM "MXFP8 carrier and quantize folds", commits 3 and 6).
#include "qz_device.cuh"

namespace qz {

constexpr int kRowChunks = 16;  // chunks of 8 elements per lane held in registers

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

// Quantize the 16 chunks of pass i held in v (chunk index c = lane + 32 i + c0).
template <int LAYOUT>
__device__ __forceinline__ void row_pass(const qz_expert& E, int64_t row, int64_t c, int64_t nch, int64_t kv,
                                         uint4 v, float S, int lane) {
    uint32_t m = absmax_bits(v);
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    const Nvfp4Block blk = nvfp4_block(bits_to_float_bf16(m), S);
    const uint32_t codes = e2m1x8_scaled(v, blk.rcp);
    if (c < nch) st_u32(static_cast<uint8_t*>(E.q) + row * (E.cols >> 1) + c * 4, codes);
    // gather the scale bytes of blocks k0..k0+3 (lanes base, base+2, base+4, base+6)
    const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, blk.scale, 2);
    const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, blk.scale, 4);
    const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, blk.scale, 6);
    if ((lane & 7) == 0) {
        const int64_t k0 = c >> 1;
        store_scale_group<LAYOUT>(E, row, k0, kv, blk.scale | (s1 << 8) | (s2 << 16) | (s3 << 24));
    }
}

template <int LAYOUT>
__global__ void __launch_bounds__(kThreads) nvfp4_rows_kernel(const qz_expert* __restrict__ table, int n,
                                                              unsigned* d_err) {
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    const int total = block_prefix(n, s_prefix, s_scan, RowUnits<LAYOUT>{table, d_err}, d_err);
    const int lane = threadIdx.x & 31;
    const int warps = kThreads / 32;
    for (int u = blockIdx.x * warps + (threadIdx.x >> 5); u < total; u += gridDim.x * warps) {
        const int e = find_owner(s_prefix, n, u);
        const qz_expert E = load_entry(table, e);
        const int64_t row = u - s_prefix[e];
        const int64_t nch = E.cols >> 3;   // 16-byte chunks in the row
        const int64_t kv = E.cols >> 4;    // scale columns
        const int64_t nsc = 2 * pad_to(kv, 4);  // chunks whose scale bytes exist (incl. padding)
        if (row >= E.rows) {
            // padded row of the swizzled region: zero scale bytes only
            for (int64_t k0 = 4 * lane; k0 < pad_to(kv, 4); k0 += 128) st_u32(E.sf + swz_offset(row, k0, kv), 0u);
            continue;
        }
        const uint16_t* xr = static_cast<const uint16_t*>(E.x) + row * E.ld;
        if (nsc <= 32 * kRowChunks) {
            uint4 v[kRowChunks];
#pragma unroll
            for (int i = 0; i < kRowChunks; ++i) {
                const int64_t c = lane + 32 * i;
                v[i] = (c < nch) ? ld_stream(xr + c * 8) : make_uint4(0, 0, 0, 0);
            }
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < kRowChunks; ++i) m = max(m, absmax_bits(v[i]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
            const float A = bits_to_float_bf16(m);
            if (lane == 0) E.amax[row] = A;
            const float S = nvfp4_encode_scale(A);
#pragma unroll
            for (int i = 0; i < kRowChunks; ++i) {
                const int64_t c0 = 32 * i;
                if (c0 < nsc) row_pass<LAYOUT>(E, row, c0 + lane, nch, kv, v[i], S, lane);
            }
        } else {
            // long row: amax pass, then a quantize pass re-reading the row
            uint32_t m = 0;
            for (int64_t c = lane; c < nch; c += 32) m = max(m, absmax_bits(ld_stream(xr + c * 8)));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
            const float A = bits_to_float_bf16(m);
            if (lane == 0) E.amax[row] = A;
            const float S = nvfp4_encode_scale(A);
            for (int64_t c0 = 0; c0 < nsc; c0 += 32) {
                const int64_t c = c0 + lane;
                const uint4 v = (c < nch) ? ld_stream(xr + c * 8) : make_uint4(0, 0, 0, 0);
                row_pass<LAYOUT>(E, row, c, nch, kv, v, S, lane);
            }
        }
    }
}

cudaError_t launch_nvfp4_rows(const qz_expert* table, int n, int layout, int grid, cudaStream_t s, unsigned* d_err) {
    const size_t smem = (size_t)(n + 1) * sizeof(int);
    if (layout == QZ_SF_SWIZZLED_128x4)
        nvfp4_rows_kernel<QZ_SF_SWIZZLED_128x4><<<grid, kThreads, smem, s>>>(table, n, d_err);
    else
        nvfp4_rows_kernel<QZ_SF_LINEAR><<<grid, kThreads, smem, s>>>(table, n, d_err);
    return cudaGetLastError();
}

int rows_blocks_per_sm(int n) {
    int b = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, nvfp4_rows_kernel<QZ_SF_SWIZZLED_128x4>, kThreads,
                                                  (size_t)(n + 1) * sizeof(int));
    return b > 0 ? b : 1;
}

}  // namespace qz
