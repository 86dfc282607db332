// qz_dequant.cu -- grouped dequantization of MXFP8 / NVFP4 tensors to bf16 (sm_100a).
//
// The inverse map of the grouped quantizers, for reference paths and error
// checks (TransformerEngine PR #3800, Changes: the regression tests compare
// dequantized values; TensorRT-LLM "MXFP8 carrier and quantize folds",
// commit 1: the dequant reference path needs the high-precision tensor).
// An element decodes to the exact product of its code's value and its block
// scale's value (and, for NVFP4, the FP32 decode scale g = RN(A / 2688) of the
// tensor or row), rounded once to bf16 (round to nearest, ties to even).
//
// One persistent launch walks all experts' 128 x 128 tiles like the quantize
// kernels: lane l of warp w owns one scale block per pass (MXFP8: 32
// elements, NVFP4: 16) of rows w + 8 * (lane / LPR) + 64 p (MXFP8) or
// + 32 p (NVFP4) of the tile.  The next tile's payload and scale loads are
// issued before the current tile is decoded; the bf16 output leaves as
// 32-byte stores (16-byte ones when the rows are only 16-byte aligned).
// NVFP4 decodes through a per-block table of the bf16 results of its eight
// e2m1 magnitudes (below), four codes per byte permute, and runs four CTAs
// per SM where MXFP8 runs three.
// NVFP4 decodes through a per-block table of its eight magnitudes (below),
// which leaves it bound by load latency rather than by arithmetic, so it runs
// four CTAs per SM where MXFP8 runs three.
#include <cuda_fp16.h>

#include "qz_device.cuh"

namespace qz {

constexpr int kDqThreads = 256;

template <int FMT>
struct DqGeo {
    static constexpr int kBlock = FMT == QZ_FMT_MXFP8 ? 32 : 16;  // elements per scale block
    static constexpr int kLpr = kTileCols / kBlock;                // lanes per tile row: 4 / 8
    static constexpr int kRpp = 8 * (32 / kLpr);                   // tile rows per pass (8 warps): 64 / 32
    static constexpr int kPasses = kTileRows / kRpp;               // passes per tile: 2 / 4
    static constexpr int kQBytes = FMT == QZ_FMT_MXFP8 ? 32 : 8;           // payload bytes per block
    static constexpr int kQWords = kQBytes / 4;
};

__device__ __forceinline__ unsigned dq_entry_errors(const qz_dq_expert& e, int fmt, int layout, bool per_row) {
    const int64_t block = (fmt == QZ_FMT_MXFP8) ? 32 : 16;
    unsigned bad = 0;
    if (e.rows < 0 || e.cols <= 0 || (e.cols % block) != 0 || e.ldy < e.cols || e.ldy > QZ_MAX_LD) bad |= QZ_DERR_SHAPE;
    if (e.rows > 0) {
        if (!e.q || !e.sf || !e.y || (fmt == QZ_FMT_NVFP4 && !e.amax)) bad |= QZ_DERR_NULL;
        if (!aligned(e.y, 16) || (e.ldy & 7) != 0) bad |= QZ_DERR_ALIGN;
        if (!aligned(e.q, fmt == QZ_FMT_MXFP8 ? 16 : 8)) bad |= QZ_DERR_ALIGN;
        if (fmt == QZ_FMT_NVFP4 && !aligned(e.amax, 4)) bad |= QZ_DERR_ALIGN;
    }
    (void)layout;
    (void)per_row;
    return bad;
}

__device__ __forceinline__ qz_dq_expert load_dq_entry(const qz_dq_expert* t, int i) {
    qz_dq_expert e;
    const int64_t* p = reinterpret_cast<const int64_t*>(t + i);
    e.q = reinterpret_cast<const void*>(__ldg(p + 0));
    e.sf = reinterpret_cast<const uint8_t*>(__ldg(p + 1));
    e.amax = reinterpret_cast<const float*>(__ldg(p + 2));
    e.rows = __ldg(p + 3);
    e.cols = __ldg(p + 4);
    e.y = reinterpret_cast<void*>(__ldg(p + 5));
    e.ldy = __ldg(p + 6);
    return e;
}

template <int FMT, int LAYOUT>
struct DqTiles {
    const qz_dq_expert* table;
    bool per_row;
    unsigned* d_err;
    __device__ long long operator()(int i) const {
        const qz_dq_expert e = load_dq_entry(table, i);
        const unsigned bad = dq_entry_errors(e, FMT, LAYOUT, per_row);
        if (bad && d_err && blockIdx.x == 0) atomicOr(d_err, bad);
        if (bad || e.rows == 0) return 0;
        return ((e.rows + kTileRows - 1) / kTileRows) * ((e.cols + kTileCols - 1) / kTileCols);
    }
};

// bf16 bits of the exact value hi + lo (hi = RN32 of it, lo the exact
// remainder), rounded to nearest even: rounding hi again is right unless hi
// lies exactly halfway between two bf16 numbers, where lo decides.
__device__ __forceinline__ uint32_t bf16_of_exact(float hi, float lo) {
    const uint32_t u = __float_as_uint(hi);
    if ((u & 0xFFFFu) == 0x8000u && lo != 0.0f) {
        const bool larger = (lo > 0.0f) == (hi > 0.0f);  // the exact magnitude exceeds |hi|
        return (u >> 16) + (larger ? 1u : 0u);
    }
    return (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
}

// Two e4m3 codes (bits 0-15, low byte first) as an f16x2 pair, exactly.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t pair) {
    uint32_t h;
    asm("{\n\t.reg .b16 c;\n\tcvt.u16.u32 c, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}" : "=r"(h) : "r"(pair));
    return h;
}

// f16x2 pair times s in binary32 (exact for the products formed here): the
// two binary32 results, low element first.
__device__ __forceinline__ float2 f16x2_times(uint32_t h, float s) {
    const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&h));
    float2 r;
    asm("{\n\t.reg .b64 a, b;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %4};\n\t"
        "mul.rn.f32x2 a, a, b;\n\tmov.b64 {%0, %1}, a;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(v.x), "f"(v.y), "f"(s));
    return r;
}

// bf16x2 of two binary32 values (round to nearest even), low element first.
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ int64_t dq_sf_index(int layout, int64_t row, int64_t k, int64_t kv) {
    return layout == QZ_SF_SWIZZLED_128x4 ? swz_offset(row, k, kv) : row * kv + k;
}

// One thread's view of one tile: its rows' payload words and scale bytes.
template <int FMT>
struct DqTile {
    uint32_t qw[DqGeo<FMT>::kPasses][DqGeo<FMT>::kQWords];
    uint32_t sc[DqGeo<FMT>::kPasses];
};

struct DqRef {
    const uint8_t* q;   // payload byte of (row of pass 0, the lane's block)
    uint16_t* y;        // output element of the same
    const float* amax;  // amax[0], or the row amax of pass 0 (per row)
    const uint8_t* sf;
    int64_t row0, kv, k, qld, ldy, rows;
    bool col_ok;
    bool y32;           // output rows 32-byte aligned: 32-byte stores
    int expert;
};

template <int FMT>
__device__ __forceinline__ DqRef dq_ref(const qz_dq_expert* table, const int* s_prefix, int tile, int e, int w,
                                        int lane, bool per_row) {
    using G = DqGeo<FMT>;
    while (tile >= s_prefix[e + 1]) ++e;  // tiles increase; s_prefix[n] == total > tile
    const qz_dq_expert E = load_dq_entry(table, e);
    const int local = tile - s_prefix[e];
    const int nct = (int)((E.cols + kTileCols - 1) / kTileCols);
    const int rt = local / nct, ct = local - rt * nct;
    DqRef r;
    r.expert = e;
    r.kv = E.cols / G::kBlock;
    r.k = (int64_t)ct * (kTileCols / G::kBlock) + lane % G::kLpr;
    r.col_ok = r.k < r.kv;
    r.qld = FMT == QZ_FMT_MXFP8 ? E.cols : E.cols >> 1;
    r.ldy = E.ldy;
    r.rows = E.rows;
    r.row0 = (int64_t)rt * kTileRows + w + 8 * (lane / G::kLpr);
    r.q = static_cast<const uint8_t*>(E.q) + r.row0 * r.qld + r.k * G::kQBytes;
    r.y = static_cast<uint16_t*>(E.y) + r.row0 * E.ldy + r.k * G::kBlock;
    r.amax = per_row ? E.amax + r.row0 : E.amax;
    r.sf = E.sf;
    r.y32 = ((reinterpret_cast<uintptr_t>(E.y) & 31) == 0) && ((E.ldy & 15) == 0);
    return r;
}

template <int FMT>
__device__ __forceinline__ bool dq_live(const DqRef& r, int p) {
    return r.col_ok && r.row0 + p * DqGeo<FMT>::kRpp < r.rows;
}

// The scale bytes of a lane's passes are affine in the pass: a tile's rows
// lie in one 128-row group and the lane's first row is in its first
// G::kRpp rows, so in the swizzled layout each pass moves kRpp / 32 4-byte
// slices; in the linear one it moves kRpp rows.
template <int FMT, int LAYOUT>
__device__ __forceinline__ void dq_load(const DqRef& r, DqTile<FMT>& t) {
    using G = DqGeo<FMT>;
    const uint8_t* sfp = r.sf + dq_sf_index(LAYOUT, r.row0, r.k, r.kv);
#pragma unroll
    for (int p = 0; p < G::kPasses; ++p) {
        if (!dq_live<FMT>(r, p)) continue;
        const uint8_t* src = r.q + (int64_t)p * G::kRpp * r.qld;
        if (FMT == QZ_FMT_MXFP8) {
            const uint4 a = ld_stream(src), b = ld_stream(src + 16);
            t.qw[p][0] = a.x; t.qw[p][1] = a.y; t.qw[p][2] = a.z; t.qw[p][3] = a.w;
            t.qw[p][4] = b.x; t.qw[p][5] = b.y; t.qw[p][6] = b.z; t.qw[p][7] = b.w;
        } else {
            const uint2 a = __ldg(reinterpret_cast<const uint2*>(src));
            t.qw[p][0] = a.x;
            t.qw[p][1] = a.y;
        }
        t.sc[p] = __ldg(sfp + (LAYOUT == QZ_SF_SWIZZLED_128x4 ? (G::kRpp / 32) * 4 * p : p * G::kRpp * r.kv));
    }
}

// MXFP8: 8 elements (two payload words) of one block, scale s = 2^(byte-127).
__device__ __forceinline__ uint4 dq_mx8(uint32_t w0, uint32_t w1, float s) {
    // exact products (at least 2^-136, above the binary32 subnormal step), so
    // a single rounding to bf16 is the rounding of the exact value
    uint4 o;
    float2 v;
    v = f16x2_times(e4m3x2_to_f16x2(w0 & 0xFFFFu), s); o.x = bf16x2_rn(v.x, v.y);
    v = f16x2_times(e4m3x2_to_f16x2(w0 >> 16), s);     o.y = bf16x2_rn(v.x, v.y);
    v = f16x2_times(e4m3x2_to_f16x2(w1 & 0xFFFFu), s); o.z = bf16x2_rn(v.x, v.y);
    v = f16x2_times(e4m3x2_to_f16x2(w1 >> 16), s);     o.w = bf16x2_rn(v.x, v.y);
    return o;
}

// Value of a non-negative e4m3 code below 0x7F without a branch: the
// subnormal m * 2^-9 is (1 + m/8) * 2^-6 - 2^-6 (both terms and the
// difference exact).
__device__ __forceinline__ float e4m3_value_nb(uint32_t s) {
    const uint32_t ef = s >> 3, m = s & 7u;
    const float v = __uint_as_float(((ef ? ef + 120u : 121u) << 23) | (m << 20));
    return ef ? v : __fsub_rn(v, 0x1p-6f);
}

// NVFP4 decode table of one block: the bf16 bits of value(m) * value(s) * g
// for the eight e2m1 magnitudes m = 0, 0.5, 1, 1.5, 2, 3, 4, 6 (codes 0-7),
// as byte tables -- lo[k] / hi[k] the low / high byte of entry k, entries
// 0-3 in the first word of each pair, 4-7 in the second -- so that a
// prmt with the magnitude codes as selectors looks up four elements at once.
// value(m) * value(s) is exact in binary32 (at most 6 significant bits); its
// RN32 product with g is rounded to bf16, and an entry whose RN32 product
// lies exactly halfway between two bf16 numbers is rounded from the exact
// product (RN32 product + the remainder the fma gives exactly).
struct NvTable {
    uint32_t lo0, lo1, hi0, hi1;
};

__device__ __forceinline__ NvTable nv_table_exact(float sv, float g) {
    float a[8];
    a[0] = 0.0f;
    a[1] = 0.5f * sv;
    a[2] = sv;
    a[3] = 1.5f * sv;
    a[4] = 2.0f * sv;
    a[5] = 3.0f * sv;
    a[6] = 4.0f * sv;
    a[7] = 6.0f * sv;
    float h[8];
    uint32_t p[4];
    // the low 16 bits of every RN32 product, xor 0x8000: a zero half marks a
    // bf16 midpoint; their minimum (per 16-bit half) finds any
    uint32_t mid = 0xFFFFFFFFu;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        asm("{\n\t.reg .b64 x, y;\n\tmov.b64 x, {%2, %3};\n\tmov.b64 y, {%4, %4};\n\t"
            "mul.rn.f32x2 x, x, y;\n\tmov.b64 {%0, %1}, x;\n\t}"
            : "=f"(h[2 * j]), "=f"(h[2 * j + 1])
            : "f"(a[2 * j]), "f"(a[2 * j + 1]), "f"(g));
        p[j] = bf16x2_rn(h[2 * j], h[2 * j + 1]);
        mid = __vminu2(mid, __byte_perm(__float_as_uint(h[2 * j]), __float_as_uint(h[2 * j + 1]), 0x5410) ^ 0x80008000u);
    }
    if ((mid & 0xFFFFu) == 0u || (mid >> 16) == 0u) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float l0 = __fmaf_rn(a[2 * j], g, -h[2 * j]);
            const float l1 = __fmaf_rn(a[2 * j + 1], g, -h[2 * j + 1]);
            p[j] = bf16_of_exact(h[2 * j], l0) | (bf16_of_exact(h[2 * j + 1], l1) << 16);
        }
    }
    NvTable t;
    t.lo0 = __byte_perm(p[0], p[1], 0x6420);
    t.hi0 = __byte_perm(p[0], p[1], 0x7531);
    t.lo1 = __byte_perm(p[2], p[3], 0x6420);
    t.hi1 = __byte_perm(p[2], p[3], 0x7531);
    return t;
}

// The same table from two products.  The magnitudes are 2^k and 1.5 * 2^k, and
// scaling by a power of two commutes with both roundings while every value
// stays normal and finite: with b1 = bf16(value(s) * g) and b3 =
// bf16(1.5 value(s) * g) (each from its RN32 product, midpoints rounded from
// the exact one as above), entry 2^k (k = -1, 0, 1, 2) is b1 with k added to
// its exponent field and entry 1.5 * 2^k (k = 0, 1, 2) is b3 with k added.
// The exponent field e1 of b1 in [3, 251] keeps every entry and every RN32
// product normal and finite (b3's field is e1 or e1 + 1); outside it the
// entries are built one by one.
__device__ __forceinline__ NvTable nv_table(float sv, float g) {
    const float a3 = 1.5f * sv;  // exact
    const float p1 = __fmul_rn(sv, g), p3 = __fmul_rn(a3, g);
    uint32_t b = bf16x2_rn(p1, p3);  // b1 low, b3 high
    if (((__float_as_uint(p1) & 0xFFFFu) == 0x8000u) || ((__float_as_uint(p3) & 0xFFFFu) == 0x8000u))
        b = bf16_of_exact(p1, __fmaf_rn(sv, g, -p1)) | (bf16_of_exact(p3, __fmaf_rn(a3, g, -p3)) << 16);
    const uint32_t e1 = (b >> 7) & 0xFFu;
    if (e1 - 3u > 248u) return nv_table_exact(sv, g);
    const uint32_t p0 = ((b & 0xFFFFu) - 0x80u) << 16;  // magnitudes 0 (zero) and 0.5
    const uint32_t p2 = b + 0x00800080u;                 // magnitudes 2 and 3 (b: 1 and 1.5)
    const uint32_t p4 = b + 0x01000100u;                 // magnitudes 4 and 6
    NvTable t;
    t.lo0 = __byte_perm(p0, b, 0x6420);
    t.hi0 = __byte_perm(p0, b, 0x7531);
    t.lo1 = __byte_perm(p2, p4, 0x6420);
    t.hi1 = __byte_perm(p2, p4, 0x7531);
    return t;
}

// NVFP4: the 8 elements of one payload word (element i in nibble i) through
// the block's table.  Four codes at a time: their magnitudes (the low three
// bits of each nibble) select the low and the high bytes; the high byte takes
// the sign bit of its code; the two byte words interleave into bf16 pairs.
// bf16(-v) is bf16(v) with the sign bit set (round to nearest is symmetric),
// so a negative code decodes to its magnitude's entry with the sign set.
__device__ __forceinline__ uint32_t nv_hi_signed(uint32_t hi, uint32_t codes4) {
    // prmt in sign-replicate mode: a nibble with bit 3 set (a negative code)
    // gives the replicated top bit of 0x7F, 0x00; a positive one gives 0x7F.
    // Adding one per byte (no carries) leaves the top bit set exactly for the
    // positive codes.
    uint32_t t;
    asm("prmt.b32 %0, %1, %1, %2;" : "=r"(t) : "r"(0x7F7F7F7Fu), "r"(codes4));
    t += 0x01010101u;
    return hi | (~t & 0x80808080u);
}

__device__ __forceinline__ uint4 dq_nv8(uint32_t word, const NvTable& T) {
    const uint32_t m = word & 0x77777777u;
    const uint32_t lo_a = __byte_perm(T.lo0, T.lo1, m), lo_b = __byte_perm(T.lo0, T.lo1, m >> 16);
    const uint32_t hi_a = nv_hi_signed(__byte_perm(T.hi0, T.hi1, m), word);
    const uint32_t hi_b = nv_hi_signed(__byte_perm(T.hi0, T.hi1, m >> 16), word >> 16);
    uint4 o;
    o.x = __byte_perm(lo_a, hi_a, 0x5140);
    o.y = __byte_perm(lo_a, hi_a, 0x7362);
    o.z = __byte_perm(lo_b, hi_b, 0x5140);
    o.w = __byte_perm(lo_b, hi_b, 0x7362);
    return o;
}

template <int FMT, int LAYOUT>
__global__ void __launch_bounds__(kDqThreads, FMT == QZ_FMT_NVFP4 ? 4 : 3)
    dequant_kernel(const qz_dq_expert* __restrict__ table, int n, bool per_row, unsigned* d_err) {
    using G = DqGeo<FMT>;
    extern __shared__ int s_prefix[];
    __shared__ long long s_scan[33];
    const int total = block_prefix(n, s_prefix, s_scan, DqTiles<FMT, LAYOUT>{table, per_row, d_err}, d_err);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int tile = blockIdx.x;
    if (tile >= total) return;
    DqRef cur = dq_ref<FMT>(table, s_prefix, tile, 0, w, lane, per_row);
    DqTile<FMT> v;
    dq_load<FMT, LAYOUT>(cur, v);
    for (;;) {
        const int next = tile + gridDim.x;
        const bool more = next < total;
        const DqRef nxt = more ? dq_ref<FMT>(table, s_prefix, next, cur.expert, w, lane, per_row) : cur;
        const DqTile<FMT> t = v;
        if (more) dq_load<FMT, LAYOUT>(nxt, v);  // the next tile's loads fly while this one decodes
        float g = 0.0f;
        if (FMT == QZ_FMT_NVFP4 && !per_row) g = __fdiv_rn(__ldg(cur.amax), 2688.0f);  // the FP32 decode scale
#pragma unroll
        for (int p = 0; p < G::kPasses; ++p) {
            if (!dq_live<FMT>(cur, p)) continue;
            uint16_t* dst = cur.y + (int64_t)p * G::kRpp * cur.ldy;
            if (FMT == QZ_FMT_MXFP8) {
                // 2^(byte - 127); byte 0 is the subnormal 2^-127
                const float s = t.sc[p] ? __uint_as_float(t.sc[p] << 23) : __uint_as_float(0x00400000u);
#pragma unroll
                for (int h = 0; h < 4; h += 2) {
                    const uint4 a = dq_mx8(t.qw[p][2 * h], t.qw[p][2 * h + 1], s);
                    const uint4 b = dq_mx8(t.qw[p][2 * h + 2], t.qw[p][2 * h + 3], s);
                    if (cur.y32) {
                        st_v8(dst + 8 * h, a, b);
                    } else {
                        st_v4(dst + 8 * h, a);
                        st_v4(dst + 8 * h + 8, b);
                    }
                }
            } else {
                if (per_row) g = __fdiv_rn(__ldg(cur.amax + (int64_t)p * G::kRpp), 2688.0f);
                const NvTable T = nv_table(e4m3_value_nb(t.sc[p]), g);
                const uint4 a = dq_nv8(t.qw[p][0], T);
                const uint4 b = dq_nv8(t.qw[p][1], T);
                if (cur.y32) {
                    st_v8(dst, a, b);
                } else {
                    st_v4(dst, a);
                    st_v4(dst + 8, b);
                }
            }
        }
        if (!more) break;
        tile = next;
        cur = nxt;
    }
}

cudaError_t launch_dequant(const qz_dq_expert* table, int n, int fmt, bool per_row, int layout, int grid,
                           cudaStream_t s, unsigned* d_err) {
    const size_t smem = (size_t)(n + 1) * sizeof(int);
    if (fmt == QZ_FMT_MXFP8) {
        if (layout == QZ_SF_SWIZZLED_128x4)
            dequant_kernel<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4><<<grid, kDqThreads, smem, s>>>(table, n, per_row, d_err);
        else
            dequant_kernel<QZ_FMT_MXFP8, QZ_SF_LINEAR><<<grid, kDqThreads, smem, s>>>(table, n, per_row, d_err);
    } else {
        if (layout == QZ_SF_SWIZZLED_128x4)
            dequant_kernel<QZ_FMT_NVFP4, QZ_SF_SWIZZLED_128x4><<<grid, kDqThreads, smem, s>>>(table, n, per_row, d_err);
        else
            dequant_kernel<QZ_FMT_NVFP4, QZ_SF_LINEAR><<<grid, kDqThreads, smem, s>>>(table, n, per_row, d_err);
    }
    return cudaGetLastError();
}

int dequant_blocks_per_sm(int n, int fmt) {
    int b = 1;
    if (fmt == QZ_FMT_NVFP4)
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, dequant_kernel<QZ_FMT_NVFP4, QZ_SF_SWIZZLED_128x4>, kDqThreads,
                                                      (size_t)(n + 1) * sizeof(int));
    else
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, dequant_kernel<QZ_FMT_MXFP8, QZ_SF_SWIZZLED_128x4>, kDqThreads,
                                                      (size_t)(n + 1) * sizeof(int));
    return b > 0 ? b : 1;
}

}  // namespace qz
