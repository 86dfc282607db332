// qz_split.cu -- gate|up split of folded fused experts (sm_100a).
//
// Model-Optimizer "Fold fused experts' quantizers into their weights
// shard-locally": a fused expert holds its gate and up projections as one
// (2I, H) weight, quantized as one tensor (gate and up share the per-tensor
// amax, so one weight_scale_2); the split cuts the folded payload and its
// scales by rows into gate (rows [0, cut)) and up (rows [cut, 2I)), each in
// storage of its own, cuts a scale in proportion to the rows it covers, and
// refuses a scale block that the cut would divide.
//
// The MXFP8 / NVFP4 scales here have one scale row per weight row, so every
// cut is exact; each part's SF region is written anew in the destination
// layout with its own padding (0x00), so a swizzled source cut inside one of
// its 128-row tiles is re-laid, not refused.  FP8 with FP32 scales of
// 128 x 128 blocks has one scale row per 128 weight rows: a cut that is not
// a multiple of 128 (and not the end) divides a block and the entry is
// refused (QZ_DERR_CUT).  The per-tensor amax goes to both parts; a per-row
// amax is cut with the rows.
//
// One persistent launch over all entries.  Each entry is a short list of
// jobs -- payload copies, scale copies or re-layouts, amax copies -- cut
// into units of a CTA's work: 32 KB of a copy (four 32-byte pieces per
// thread, narrower pieces in rounds of four when the pointers are less
// aligned), or one 128-row block of a scale re-layout (32-bit words).
#include "qz_device.cuh"

namespace qz {

constexpr int kSplitThreads = 256;
constexpr int64_t kCopyUnit = kSplitThreads * 128;  // bytes of a copy unit

enum SplitJobKind { kJobCopy = 0, kJobTiles = 1, kJobGather = 2, kJobAmax = 3 };

struct SplitJob {
    int kind;
    const uint8_t* src;
    uint8_t* dst;
    int64_t bytes;  // copy: bytes
    int64_t first;  // re-layouts: the fused row of the part's row 0
    int64_t rows;   // re-layouts: rows of the part
    int64_t units;
    int64_t kv;     // re-layouts: scale columns
    float* dst2;    // per-tensor amax: the second part's slot
};

struct SplitCall {
    int fmt, amax_kind, src_layout, dst_layout;
};

__device__ __forceinline__ qz_fused_split load_split_entry(const qz_fused_split* t, int i) {
    qz_fused_split e;
    const int64_t* p = reinterpret_cast<const int64_t*>(t + i);
    e.q = reinterpret_cast<const void*>(__ldg(p + 0));
    e.sf = reinterpret_cast<const uint8_t*>(__ldg(p + 1));
    e.amax = reinterpret_cast<const float*>(__ldg(p + 2));
    e.rows = __ldg(p + 3);
    e.cols = __ldg(p + 4);
    e.cut = __ldg(p + 5);
    e.q_out[0] = reinterpret_cast<void*>(__ldg(p + 6));
    e.q_out[1] = reinterpret_cast<void*>(__ldg(p + 7));
    e.sf_out[0] = reinterpret_cast<uint8_t*>(__ldg(p + 8));
    e.sf_out[1] = reinterpret_cast<uint8_t*>(__ldg(p + 9));
    e.amax_out[0] = reinterpret_cast<float*>(__ldg(p + 10));
    e.amax_out[1] = reinterpret_cast<float*>(__ldg(p + 11));
    return e;
}

__device__ __forceinline__ int64_t split_block(int fmt) {
    return fmt == QZ_FMT_MXFP8 ? 32 : (fmt == QZ_FMT_NVFP4 ? 16 : 1);
}

// log2 of the block: scale columns = cols >> split_block_log2(fmt)
__device__ __forceinline__ int split_block_log2(int fmt) { return fmt == QZ_FMT_MXFP8 ? 5 : (fmt == QZ_FMT_NVFP4 ? 4 : 0); }

__device__ __forceinline__ bool per_tensor_amax_job(const qz_fused_split& e, const SplitCall& c) {
    return c.amax_kind == QZ_AMAX_PER_TENSOR && e.amax && e.amax_out[0] && e.amax_out[1];
}

// The QZ_DERR_* bits that make an entry invalid.
__device__ unsigned split_entry_errors(const qz_fused_split& e, const SplitCall& c) {
    unsigned bad = 0;
    if (e.rows < 0 || e.cols <= 0 || e.cols > QZ_MAX_LD || e.cols % split_block(c.fmt) != 0 || e.cut < 0 ||
        e.cut > e.rows)
        return QZ_DERR_SHAPE;
    if (c.fmt == QZ_FMT_FP8_BLOCK128 && e.cut % 128 != 0 && e.cut < e.rows) bad |= QZ_DERR_CUT;
    const int64_t n[2] = {e.cut, e.rows - e.cut};
    const bool swz_src = c.fmt != QZ_FMT_FP8_BLOCK128 && c.src_layout == QZ_SF_SWIZZLED_128x4;
    const bool swz_dst = c.fmt != QZ_FMT_FP8_BLOCK128 && c.dst_layout == QZ_SF_SWIZZLED_128x4;
    const uintptr_t sf_align = c.fmt == QZ_FMT_FP8_BLOCK128 ? 4 : 1;
    if (e.rows > 0) {
        if (!e.sf) bad |= QZ_DERR_NULL;
        if (e.sf && !aligned(e.sf, swz_src ? 16 : sf_align)) bad |= QZ_DERR_ALIGN;
    }
    for (int p = 0; p < 2; ++p) {
        if (n[p] == 0) continue;
        if (!e.sf_out[p] || (e.q_out[p] && !e.q)) bad |= QZ_DERR_NULL;
        if (e.sf_out[p] && !aligned(e.sf_out[p], swz_dst ? 16 : sf_align)) bad |= QZ_DERR_ALIGN;
        if (c.amax_kind == QZ_AMAX_PER_ROW) {
            if (!e.amax || !e.amax_out[p]) bad |= QZ_DERR_NULL;
            else if (!aligned(e.amax, 4) || !aligned(e.amax_out[p], 4)) bad |= QZ_DERR_ALIGN;
        }
    }
    if (c.amax_kind == QZ_AMAX_PER_TENSOR) {
        if (e.rows > 0 && !(e.amax && e.amax_out[0] && e.amax_out[1])) bad |= QZ_DERR_NULL;
        if (per_tensor_amax_job(e, c) &&
            (!aligned(e.amax, 4) || !aligned(e.amax_out[0], 4) || !aligned(e.amax_out[1], 4)))
            bad |= QZ_DERR_ALIGN;
    }
    return bad;
}

// Visit the jobs of a valid entry in a fixed order; f(job) returns true to
// stop the walk.
template <typename F>
__device__ __forceinline__ void for_each_job(const qz_fused_split& e, const SplitCall& c, F f) {
    const int64_t n[2] = {e.cut, e.rows - e.cut};
    const int64_t first[2] = {0, e.cut};
    const int64_t row_bytes = c.fmt == QZ_FMT_NVFP4 ? e.cols >> 1 : e.cols;
    const uint8_t* q = static_cast<const uint8_t*>(e.q);
    SplitJob j;
    for (int p = 0; p < 2; ++p) {
        if (n[p] == 0 || !e.q_out[p]) continue;
        j = {kJobCopy, q + first[p] * row_bytes, static_cast<uint8_t*>(e.q_out[p]), n[p] * row_bytes, 0, 0, 0};
        j.units = (j.bytes + kCopyUnit - 1) / kCopyUnit;
        if (f(j)) return;
    }
    for (int p = 0; p < 2; ++p) {
        if (n[p] == 0) continue;
        if (c.fmt == QZ_FMT_FP8_BLOCK128) {
            // FP32 scales of 128-row blocks, row-major: whole scale rows move
            const int64_t scol_bytes = ((e.cols + 127) / 128) * 4;
            j = {kJobCopy, e.sf + (first[p] / 128) * scol_bytes, e.sf_out[p], ((n[p] + 127) / 128) * scol_bytes, 0, 0,
                 0};
            j.units = (j.bytes + kCopyUnit - 1) / kCopyUnit;
        } else {
            const int64_t kv = e.cols >> split_block_log2(c.fmt);
            if (c.src_layout == QZ_SF_LINEAR && c.dst_layout == QZ_SF_LINEAR) {
                j = {kJobCopy, e.sf + first[p] * kv, e.sf_out[p], n[p] * kv, 0, 0, 0};
                j.units = (j.bytes + kCopyUnit - 1) / kCopyUnit;
            } else if (c.src_layout == QZ_SF_SWIZZLED_128x4 && c.dst_layout == QZ_SF_SWIZZLED_128x4 &&
                       (first[p] & 127) == 0 && (kv & 3) == 0) {
                // the part starts on a tile boundary and has no padded columns:
                // its whole 128-row blocks are the source's tiles unchanged
                const int64_t full = n[p] >> 7, block_bytes = kv * 128;
                if (full > 0) {
                    j = {kJobCopy, e.sf + (first[p] >> 7) * block_bytes, e.sf_out[p], full * block_bytes, 0, 0, 0};
                    j.units = (j.bytes + kCopyUnit - 1) / kCopyUnit;
                    if (f(j)) return;
                }
                if ((n[p] & 127) == 0) continue;
                // the last, partial block (its padded rows are written 0x00)
                j = {kJobTiles, e.sf, e.sf_out[p] + full * block_bytes, 0, first[p] + full * 128, n[p] - full * 128, 1,
                     kv, nullptr};
            } else {
                // one unit per 128-row block of the part
                j = {c.dst_layout == QZ_SF_SWIZZLED_128x4 ? kJobTiles : kJobGather, e.sf, e.sf_out[p], 0, first[p],
                     n[p], (n[p] + 127) >> 7, kv, nullptr};
            }
        }
        if (f(j)) return;
    }
    if (c.amax_kind == QZ_AMAX_PER_ROW) {
        for (int p = 0; p < 2; ++p) {
            if (n[p] == 0) continue;
            j = {kJobCopy, reinterpret_cast<const uint8_t*>(e.amax + first[p]),
                 reinterpret_cast<uint8_t*>(e.amax_out[p]), n[p] * 4, 0, 0, 0};
            j.units = (j.bytes + kCopyUnit - 1) / kCopyUnit;
            if (f(j)) return;
        }
    }
    if (per_tensor_amax_job(e, c)) {
        j = {kJobAmax, reinterpret_cast<const uint8_t*>(e.amax), reinterpret_cast<uint8_t*>(e.amax_out[0]), 4, 0, 0, 1, 0,
             e.amax_out[1]};
        f(j);
    }
}

struct SplitUnits {
    const qz_fused_split* table;
    SplitCall call;
    unsigned* d_err;
    __device__ long long operator()(int i) const {
        const qz_fused_split e = load_split_entry(table, i);
        const unsigned bad = split_entry_errors(e, call);
        if (bad && d_err && blockIdx.x == 0) atomicOr(d_err, bad);
        if (bad) return 0;
        long long u = 0;
        for_each_job(e, call, [&](const SplitJob& j) {
            u += j.units;
            return false;
        });
        return u;
    }
};

// ---------------------------------------------------------------------------
// copies: bytes [beg, end) of a job, in pieces of W bytes (W divides the
// alignment of both pointers), PER pieces per thread loaded before any store
// ---------------------------------------------------------------------------

template <int W>
struct Piece;
template <>
struct Piece<32> {
    uint4 a, b;
    __device__ void load(const uint8_t* p) {
        uint32_t w[8];
        ld_stream_32<kL2First>(p, w);
        a = make_uint4(w[0], w[1], w[2], w[3]);
        b = make_uint4(w[4], w[5], w[6], w[7]);
    }
    __device__ void store(uint8_t* p) const { st_v8(p, a, b); }
};
template <>
struct Piece<16> {
    uint4 a;
    __device__ void load(const uint8_t* p) { a = __ldg(reinterpret_cast<const uint4*>(p)); }
    __device__ void store(uint8_t* p) const { st_v4(p, a); }
};
template <>
struct Piece<8> {
    uint2 a;
    __device__ void load(const uint8_t* p) { a = __ldg(reinterpret_cast<const uint2*>(p)); }
    __device__ void store(uint8_t* p) const { *reinterpret_cast<uint2*>(p) = a; }
};
template <>
struct Piece<4> {
    uint32_t a;
    __device__ void load(const uint8_t* p) { a = __ldg(reinterpret_cast<const uint32_t*>(p)); }
    __device__ void store(uint8_t* p) const { *reinterpret_cast<uint32_t*>(p) = a; }
};
template <int W>
__device__ __forceinline__ void copy_pieces(const uint8_t* src, uint8_t* dst, int64_t beg, int64_t end) {
    constexpr int kTotal = (int)(kCopyUnit / W / kSplitThreads);  // pieces per thread
    constexpr int kRound = kTotal < 4 ? kTotal : 4;                 // loaded before they are stored
#pragma unroll
    for (int r = 0; r < kTotal; r += kRound) {
        Piece<W> v[kRound];
#pragma unroll
        for (int i = 0; i < kRound; ++i) {
            const int64_t o = beg + ((int64_t)(r + i) * kSplitThreads + threadIdx.x) * W;
            if (o + W <= end) v[i].load(src + o);
        }
#pragma unroll
        for (int i = 0; i < kRound; ++i) {
            const int64_t o = beg + ((int64_t)(r + i) * kSplitThreads + threadIdx.x) * W;
            if (o + W <= end) v[i].store(dst + o);
        }
    }
    // the last unit's tail, shorter than one piece
    const int64_t tail = beg + ((end - beg) / W) * W;
    for (int64_t o = tail + threadIdx.x; o < end; o += kSplitThreads) dst[o] = __ldg(src + o);
}

__device__ __forceinline__ void copy_unit(const SplitJob& j, int64_t u) {
    const int64_t beg = u * kCopyUnit;
    const int64_t end = min(j.bytes, beg + kCopyUnit);
    const uintptr_t mis = reinterpret_cast<uintptr_t>(j.src) | reinterpret_cast<uintptr_t>(j.dst);
    if ((mis & 31) == 0) copy_pieces<32>(j.src, j.dst, beg, end);
    else if ((mis & 15) == 0) copy_pieces<16>(j.src, j.dst, beg, end);
    else if ((mis & 7) == 0) copy_pieces<8>(j.src, j.dst, beg, end);
    else if ((mis & 3) == 0) copy_pieces<4>(j.src, j.dst, beg, end);
    else
        for (int64_t o = beg + threadIdx.x; o < end; o += kSplitThreads) j.dst[o] = __ldg(j.src + o);
}

// ---------------------------------------------------------------------------
// scale re-layouts (MXFP8 / NVFP4 scales, one byte per (row, k))
// ---------------------------------------------------------------------------

// Scale bytes (row rs, columns k0..k0+3) of the source region as one word,
// columns at or past kv as 0x00.  k0 is a multiple of 4.
__device__ __forceinline__ uint32_t sf_word(const uint8_t* sf, int layout, int64_t rs, int64_t k0, int64_t kv) {
    if (layout == QZ_SF_SWIZZLED_128x4) {
        uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(sf + swz_offset(rs, k0, kv)));
        const int64_t live = kv - k0;
        if (live < 4) w &= (1u << (8 * live)) - 1u;
        return w;
    }
    const uint8_t* p = sf + rs * kv + k0;
    if (kv - k0 >= 4 && aligned(p, 4)) return __ldg(reinterpret_cast<const uint32_t*>(p));
    uint32_t w = 0;
    for (int i = 0; i < 4 && k0 + i < kv; ++i) w |= (uint32_t)__ldg(p + i) << (8 * i);
    return w;
}

// Row block u (128 rows) of a swizzled destination region: thread t writes
// word t % 128 -- the four scale columns of row (t % 128) / 4 + 32 (t % 4) of
// the block -- of every other column tile, starting at tile t / 128.
__device__ __forceinline__ void tiles_unit(const SplitJob& j, int src_layout, int64_t u) {
    const int w = threadIdx.x & 127;
    const int64_t r = u * 128 + (w >> 2) + 32 * (w & 3);
    const int64_t nct = (j.kv + 3) >> 2;
    const bool live = r < j.rows;
    uint8_t* dst = j.dst + u * nct * 512 + 4 * w;
#pragma unroll 4
    for (int64_t ct = threadIdx.x >> 7; ct < nct; ct += 2) {
        const uint32_t v = live ? sf_word(j.src, src_layout, j.first + r, ct * 4, j.kv) : 0u;
        *reinterpret_cast<uint32_t*>(dst + ct * 512) = v;
    }
}

// Row block u (128 rows) of a linear destination region from a swizzled
// source: two threads per row, each writing every other group of four scale
// columns.
__device__ __forceinline__ void gather_unit(const SplitJob& j, int64_t u) {
    const int64_t r = u * 128 + (threadIdx.x >> 1);
    if (r >= j.rows) return;
    uint8_t* row = j.dst + r * j.kv;
    for (int64_t k0 = 4 * (threadIdx.x & 1); k0 < j.kv; k0 += 8) {
        const uint32_t w = sf_word(j.src, QZ_SF_SWIZZLED_128x4, j.first + r, k0, j.kv);
        if (j.kv - k0 >= 4 && aligned(row + k0, 4)) {
            *reinterpret_cast<uint32_t*>(row + k0) = w;
        } else {
            for (int i = 0; i < 4 && k0 + i < j.kv; ++i) row[k0 + i] = (uint8_t)(w >> (8 * i));
        }
    }
}

__global__ void __launch_bounds__(kSplitThreads, 3) split_fused_kernel(const qz_fused_split* __restrict__ table, int n,
                                                                    SplitCall call, unsigned* d_err) {
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    const int total = block_prefix(n, s_prefix, s_scan, SplitUnits{table, call, d_err}, d_err);
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        const int ex = find_owner(s_prefix, n, u);
        const qz_fused_split e = load_split_entry(table, ex);
        int64_t local = u - s_prefix[ex];
        SplitJob job{};
        job.kind = -1;
        for_each_job(e, call, [&](const SplitJob& j) {
            if (local < j.units) {
                job = j;
                return true;
            }
            local -= j.units;
            return false;
        });
        switch (job.kind) {
            case kJobCopy: copy_unit(job, local); break;
            case kJobTiles: tiles_unit(job, call.src_layout, local); break;
            case kJobGather: gather_unit(job, local); break;
            case kJobAmax:
                if (threadIdx.x == 0) {
                    const float a = __ldg(reinterpret_cast<const float*>(job.src));
                    *reinterpret_cast<float*>(job.dst) = a;
                    *job.dst2 = a;
                }
                break;
            default: break;
        }
    }
}

cudaError_t launch_split_fused(const qz_fused_split* table, int n, int fmt, int amax_kind, int src_layout,
                               int dst_layout, int grid, cudaStream_t s, unsigned* d_err) {
    const SplitCall call{fmt, amax_kind, src_layout, dst_layout};
    split_fused_kernel<<<grid, kSplitThreads, (size_t)(n + 1) * sizeof(int), s>>>(table, n, call, d_err);
    return cudaGetLastError();
}

int split_blocks_per_sm(int n) {
    int b = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, split_fused_kernel, kSplitThreads, (size_t)(n + 1) * sizeof(int));
    return b > 0 ? b : 1;
}

}  // namespace qz
