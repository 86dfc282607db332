// qz_merge.cu -- attention decode merge that also writes its MXFP8 form (sm_100a).
//
// TensorRT-LLM "MXFP8 carrier and quantize folds", commit 3: the kernel that
// finishes flash-decoding holds the merged attention output in registers, and
// the projection consuming it immediately quantizes it to MXFP8; the merge
// writes both forms, and the scale-factor rows that swizzling invents past the
// last live row, spread over the live CTAs a few bytes each, so the caller
// can pass a plain per-step allocation.  A producer kernel of this library
// using the device functions of include/qz_quant.cuh.
//
// Merge (flash-decoding split combine): S partial outputs O[s, t, :] with
// log-sum-exps lse[s, t] give y[t, :] = sum_s w_s O[s, t, :] / sum_s w_s,
// w_s = exp(lse[s, t] - max_s lse[s, t]), accumulated in binary64 (partial
// outputs of opposite signs cancel, and a binary32 sum would lose the
// result's low bits) and rounded once to bf16.
//
// CTA (t, c) owns 1024 columns of token t: thread i holds 8 consecutive
// outputs, four consecutive threads one MXFP8 block.
#include "../../include/qz_quant.cuh"

namespace qz {

constexpr int kMergeCols = 1024;               // columns per CTA
constexpr int kMergeThreads = kMergeCols / 8;  // 8 outputs per thread

__global__ void __launch_bounds__(kMergeThreads) attention_merge_kernel(const float* __restrict__ O,
                                                                        const float* __restrict__ lse, int S,
                                                                        int64_t T, int64_t H, uint16_t* y, uint8_t* q,
                                                                        uint8_t* sf, int layout) {
    extern __shared__ double s_w[];  // [S] split weights of this token
    const int64_t t = blockIdx.x;
    const int64_t c0 = (int64_t)blockIdx.y * kMergeCols + 8 * threadIdx.x;
    const bool live = c0 < H;
    // weights in binary64: w_s = exp(lse_s - max lse), summed in split order
    double m = -INFINITY;
    for (int s = 0; s < S; ++s) m = fmax(m, (double)__ldg(lse + (int64_t)s * T + t));
    for (int s = threadIdx.x; s < S; s += blockDim.x) s_w[s] = exp((double)__ldg(lse + (int64_t)s * T + t) - m);
    __syncthreads();
    double wsum = 0.0;
    double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    // splits four at a time: their loads are all in flight before the first is summed
    constexpr int kU = 4;
    const float4* src = reinterpret_cast<const float4*>(O + (int64_t)t * H + c0);
    const int64_t split_stride = T * H / 4;  // float4s between consecutive splits
    int s = 0;
    for (; s + kU <= S; s += kU) {
        float4 a[kU], b[kU];
        if (live) {
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                a[u] = __ldg(src + (s + u) * split_stride);
                b[u] = __ldg(src + (s + u) * split_stride + 1);
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const double wgt = s_w[s + u];
            wsum = wsum + wgt;
            if (live) {
                const float v[8] = {a[u].x, a[u].y, a[u].z, a[u].w, b[u].x, b[u].y, b[u].z, b[u].w};
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = acc[i] + wgt * (double)v[i];  // product, then sum (no FMA)
            }
        }
    }
    for (; s < S; ++s) {
        const double wgt = s_w[s];
        wsum = wsum + wgt;
        if (live) {
            const float4 a = __ldg(src + s * split_stride), b = __ldg(src + s * split_stride + 1);
            const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = acc[i] + wgt * (double)v[i];
        }
    }
    // one rounding to bf16 of the binary64 quotient
    uint32_t x[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint16_t lo, hi;
        asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(lo) : "d"(acc[2 * j] / wsum));
        asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(hi) : "d"(acc[2 * j + 1] / wsum));
        x[j] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    if (live) st_v4(y + t * H + c0, make_uint4(x[0], x[1], x[2], x[3]));
    if (q == nullptr) return;

    // the MXFP8 form of exactly the bf16 values just stored
    uint32_t codes[2];
    const uint32_t scale = qzq::mxfp8_block_x4(x, codes);  // all lanes (full-warp shuffles)
    const int64_t kv = H / 32;
    if (live) {
        st_v2(q + t * H + c0, codes[0], codes[1]);
        if ((threadIdx.x & 3) == 0) sf[qzq::sf_offset(t, c0 / 32, kv, layout)] = (uint8_t)scale;
    }
    // padded rows of the swizzled region: padded row p is zeroed by the CTAs
    // of live row (p - T) % T, each over its own scale columns
    if (layout == QZ_SF_SWIZZLED_128x4 && threadIdx.x < kMergeCols / 32) {
        const int64_t k = (int64_t)blockIdx.y * (kMergeCols / 32) + threadIdx.x;
        if (k < kv) {
            const int64_t pad_end = T + qzq::sf_padded_rows(T);
            for (int64_t p = T + t; p < pad_end; p += T) sf[qzq::sf_offset(p, k, kv, layout)] = 0;
        }
    }
}

cudaError_t launch_attention_merge(const float* O, const float* lse, int S, int64_t T, int64_t H, uint16_t* y,
                                   uint8_t* q, uint8_t* sf, int layout, cudaStream_t s) {
    const dim3 grid((unsigned)T, (unsigned)((H + kMergeCols - 1) / kMergeCols));
    attention_merge_kernel<<<grid, kMergeThreads, (size_t)S * sizeof(double), s>>>(O, lse, S, T, H, y, q, sf, layout);
    return cudaGetLastError();
}

}  // namespace qz
