// qz_device.cuh -- device helpers of the grouped quantization kernels (sm_100a).
//
// Everything here is register/shared-memory arithmetic shared by the kernels
// in this directory: 128-bit streaming loads, bf16 field access, the exact
// E8M0 exponent, the NVFP4 two-level scale, hardware e4m3/e2m1 conversion,
// the swizzled 128x4 offset and the expert-table walk.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qz.h"

namespace qz {

constexpr int kThreads = 256;     // threads of every grouped CTA
constexpr int kTileRows = 128;    // rows of a tile (one swizzled row block)
constexpr int kTileCols = 128;    // bf16 columns of a tile: 16 chunks of 8 elements

// ---------------------------------------------------------------------------
// memory access
// ---------------------------------------------------------------------------

// 16-byte load that bypasses L1 allocation: every input byte is read once.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_v2(void* p, uint32_t a, uint32_t b) {
    asm volatile("st.global.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(a), "r"(b) : "memory");
}

__device__ __forceinline__ void st_u32(void* p, uint32_t a) {
    asm volatile("st.global.u32 [%0], %1;" ::"l"(p), "r"(a) : "memory");
}

// L2 eviction priority of a load: default, keep (the data is read again
// soon), or drop first (last use).
enum L2Hint { kL2Normal = 0, kL2Last = 1, kL2First = 2 };

#define QZ_LD32(HINTQ)                                                                                         \
    asm volatile("ld.global.nc.L1::no_allocate" HINTQ ".v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"               \
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7]) \
                 : "l"(p))
#define QZ_LD16(HINTQ, OFF, A, B, C, D)                                                                        \
    asm volatile("ld.global.nc" HINTQ ".v4.u32 {%0,%1,%2,%3}, [%4];"                                          \
                 : "=r"(w[A]), "=r"(w[B]), "=r"(w[C]), "=r"(w[D])                                               \
                 : "l"(static_cast<const char*>(p) + (OFF)))

// 32-byte load (the address must be 32-byte aligned).
template <int HINT = kL2Normal>
__device__ __forceinline__ void ld_stream_32(const void* p, uint32_t (&w)[8]) {
    if (HINT == kL2Last) QZ_LD32(".L2::evict_last");
    else if (HINT == kL2First) QZ_LD32(".L2::evict_first");
    else QZ_LD32("");
}

// 32 bytes from a 16-byte aligned address as two 16-byte loads that allocate
// in L1 (the second finds the sectors the first brought in).  The L2
// eviction qualifiers exist only for 256-bit loads, so the hint is dropped.
template <int HINT = kL2Normal>
__device__ __forceinline__ void ld_pair_16(const void* p, uint32_t (&w)[8]) {
    QZ_LD16("", 0, 0, 1, 2, 3);
    QZ_LD16("", 16, 4, 5, 6, 7);
}
#undef QZ_LD32
#undef QZ_LD16

// 32-byte store (the address must be 32-byte aligned).
__device__ __forceinline__ void st_v8(void* p, uint4 a, uint4 b) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(a.x), "r"(a.y), "r"(a.z),
                 "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
                 : "memory");
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// ---------------------------------------------------------------------------
// bf16 fields
// ---------------------------------------------------------------------------

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Packed bf16 maximum of magnitudes (PTX max.xorsign.abs.bf16x2): each half
// holds the larger |x| of the two inputs' halves; its sign bit is the xor of
// theirs and is dropped by the callers.  Subnormal bf16 values are ordered
// exactly (there is no flush for bf16).
__device__ __forceinline__ uint32_t max_abs_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// bf16 magnitude bits of the larger half of a packed magnitude pair (for
// non-negative IEEE values the integer order of the bit patterns is the
// numeric order).
__device__ __forceinline__ uint32_t larger_half(uint32_t m) {
    const uint32_t a = m & 0x7FFF7FFFu;
    return max(a & 0xFFFFu, a >> 16);
}

// Largest |x| of the bf16 pairs in w[0..N) (N a power of two), as bf16
// magnitude bits: a tree of packed magnitude maxima.
template <int N>
__device__ __forceinline__ uint32_t absmax_words(const uint32_t* w) {
    static_assert(N >= 1 && (N & (N - 1)) == 0, "N must be a power of two");
    uint32_t m[N];
#pragma unroll
    for (int i = 0; i < N; ++i) m[i] = w[i];
#pragma unroll
    for (int s = 1; s < N; s <<= 1) {
#pragma unroll
        for (int i = 0; i + s < N; i += 2 * s) m[i] = max_abs_bf16x2(m[i], m[i + s]);
    }
    return larger_half(m[0]);
}

// Largest |x| of the 8 bf16 in v, as bf16 magnitude bits.
__device__ __forceinline__ uint32_t absmax_bits(uint4 v) {
    return larger_half(max_abs_bf16x2(max_abs_bf16x2(v.x, v.y), max_abs_bf16x2(v.z, v.w)));
}

__device__ __forceinline__ float bits_to_float_bf16(uint32_t m16) { return __uint_as_float(m16 << 16); }

// ---------------------------------------------------------------------------
// MXFP8 scale
// ---------------------------------------------------------------------------

// E8M0 byte for a block whose largest magnitude has bf16 bits m16: the
// smallest e with amax <= 448 * 2^e, as e + 127, clamped at 0.  With
// amax = (1 + f/128) * 2^(E-127) and 448 = 1.75 * 2^8, e = E - 127 - 8 when
// f <= 96 (significand <= 1.75) and one more otherwise.  Zero and subnormal
// amax (< 2^-126 < 448 * 2^-128) clamp to byte 0.  Exact: no division.
__device__ __forceinline__ uint32_t e8m0_byte(uint32_t m16) {
    const int E = (int)(m16 >> 7);
    if (E == 0) return 0u;
    const int b = E - 8 + (((m16 & 0x7Fu) > 96u) ? 1 : 0);
    return (uint32_t)max(b, 0);
}

// 2^-e for the scale byte (e = byte - 127): binary32 exponent field 254 - byte.
// byte <= 247 for bf16 input, so the result is always a normal number and the
// flush-to-zero rule never applies.
__device__ __forceinline__ float e8m0_reciprocal(uint32_t byte) {
    return __uint_as_float((254u - byte) << 23);
}

// ---------------------------------------------------------------------------
// hardware conversions (PTX ISA: cvt with .satfinite; the first source
// operand lands in the upper half of the packed result)
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// The element products of the format conversions: each bf16 pair of a word
// is widened to two binary32 values and multiplied by s as one packed
// round-to-nearest product (PTX ISA 8.6 mul.rn.f32x2, sm_100), i.e. RN(x * s)
// for each element, exactly as two scalar products.

// Four e4m3 codes of the bf16 pairs in words a, b times s (element 0 lowest).
__device__ __forceinline__ uint32_t e4m3x4_words(uint32_t a, uint32_t b, float s) {
    uint32_t r;
    asm("{\n\t"
        ".reg .b32 l0, h0, l1, h1;\n\t"
        ".reg .b64 p0, p1, ss;\n\t"
        ".reg .b16 c0, c1;\n\t"
        "mov.b64 ss, {%3, %3};\n\t"
        "shl.b32 l0, %1, 16;\n\tand.b32 h0, %1, -65536;\n\tmov.b64 p0, {l0, h0};\n\t"
        "shl.b32 l1, %2, 16;\n\tand.b32 h1, %2, -65536;\n\tmov.b64 p1, {l1, h1};\n\t"
        "mul.rn.f32x2 p0, p0, ss;\n\tmul.rn.f32x2 p1, p1, ss;\n\t"
        "mov.b64 {l0, h0}, p0;\n\tmov.b64 {l1, h1}, p1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 c0, h0, l0;\n\tcvt.rn.satfinite.e4m3x2.f32 c1, h1, l1;\n\t"
        "mov.b32 %0, {c0, c1};\n\t"
        "}"
        : "=r"(r)
        : "r"(a), "r"(b), "f"(s));
    return r;
}

// Eight e4m3 codes of x[i] * s, element 0 in the lowest byte.
__device__ __forceinline__ uint2 e4m3x8_scaled(uint4 v, float s) {
    return make_uint2(e4m3x4_words(v.x, v.y, s), e4m3x4_words(v.z, v.w, s));
}

// Eight e2m1 codes of the bf16 pairs in words a..d times s (element 0 in the
// lowest nibble; cvt.rn.satfinite.e2m1x2 puts its first operand in the upper
// nibble).
__device__ __forceinline__ uint32_t e2m1x8_words(uint32_t a, uint32_t b, uint32_t c, uint32_t d, float s) {
    uint32_t r;
    asm("{\n\t"
        ".reg .b32 l0, h0, l1, h1, l2, h2, l3, h3;\n\t"
        ".reg .b64 p0, p1, p2, p3, ss;\n\t"
        ".reg .b8 q0, q1, q2, q3;\n\t"
        "mov.b64 ss, {%5, %5};\n\t"
        "shl.b32 l0, %1, 16;\n\tand.b32 h0, %1, -65536;\n\tmov.b64 p0, {l0, h0};\n\t"
        "shl.b32 l1, %2, 16;\n\tand.b32 h1, %2, -65536;\n\tmov.b64 p1, {l1, h1};\n\t"
        "shl.b32 l2, %3, 16;\n\tand.b32 h2, %3, -65536;\n\tmov.b64 p2, {l2, h2};\n\t"
        "shl.b32 l3, %4, 16;\n\tand.b32 h3, %4, -65536;\n\tmov.b64 p3, {l3, h3};\n\t"
        "mul.rn.f32x2 p0, p0, ss;\n\tmul.rn.f32x2 p1, p1, ss;\n\t"
        "mul.rn.f32x2 p2, p2, ss;\n\tmul.rn.f32x2 p3, p3, ss;\n\t"
        "mov.b64 {l0, h0}, p0;\n\tmov.b64 {l1, h1}, p1;\n\tmov.b64 {l2, h2}, p2;\n\tmov.b64 {l3, h3}, p3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q0, h0, l0;\n\tcvt.rn.satfinite.e2m1x2.f32 q1, h1, l1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q2, h2, l2;\n\tcvt.rn.satfinite.e2m1x2.f32 q3, h3, l3;\n\t"
        "mov.b32 %0, {q0, q1, q2, q3};\n\t"
        "}"
        : "=r"(r)
        : "r"(a), "r"(b), "r"(c), "r"(d), "f"(s));
    return r;
}

// Eight e2m1 codes of x[i] * s, element 0 in the lowest nibble.
__device__ __forceinline__ uint32_t e2m1x8_scaled(uint4 v, float s) { return e2m1x8_words(v.x, v.y, v.z, v.w, s); }

// e4m3 code (RNE, satfinite) of one non-negative float.
__device__ __forceinline__ uint32_t e4m3_of(float v) { return cvt_e4m3x2(v, 0.0f) & 0xFFu; }

// Value of a non-negative e4m3 code below 0x7F (bias 7, 3 mantissa bits).
__device__ __forceinline__ float e4m3_value(uint32_t s) {
    const uint32_t ef = s >> 3, m = s & 7u;
    if (ef == 0) return (float)m * 0x1p-9f;
    return __uint_as_float(((ef + 120u) << 23) | (m << 20));
}

// ---------------------------------------------------------------------------
// NVFP4 two-level scale
// ---------------------------------------------------------------------------

// Encode scale from the tensor (or row) amax A: S = RN(1 / RN(A / 2688)),
// zero when the decode scale is zero.
__device__ __forceinline__ float nvfp4_encode_scale(float A) {
    const float g = __fdiv_rn(A, 2688.0f);
    return g == 0.0f ? 0.0f : __fdiv_rn(1.0f, g);
}

// RN(b / 6) for a bf16 magnitude b (8 significant bits), by the quotient
// correction of Markstein (IBM J. Res. Dev. 34(1), 1990): q0 = RN(b * RN(1/6)),
// r = b - 6 q0 exactly (one FMA), q = RN(q0 + r * RN(1/6)).  The correction
// is exact unless b/6 lies within a tiny fraction of an ulp of a rounding
// midpoint; b/6 with an 8-bit b is either exact or has the periodic binary
// expansion ...0101..., a third of an ulp or more from any midpoint, so q is
// the correctly rounded quotient for every bf16 b (checked exhaustively
// against IEEE division in the test suite).
__device__ __forceinline__ float div6_rn(float b) {
    const float c = 1.0f / 6.0f;
    const float q0 = __fmul_rn(b, c);
    const float r = __fmaf_rn(-q0, 6.0f, b);
    return __fmaf_rn(r, c, q0);
}

struct Nvfp4Block {
    uint32_t scale;  // e4m3 code of the block scale
    float rcp;       // multiplier applied to each element
};

// RN(1/m) for m = 0..15 (entry 0 unused), filled once per CTA in shared memory.
__device__ __forceinline__ void fill_inv_table(float* inv) {
    if (threadIdx.x < 16) inv[threadIdx.x] = threadIdx.x ? __fdiv_rn(1.0f, (float)threadIdx.x) : 0.0f;
}

// RN(S / value(s)) for a non-zero e4m3 code s < 0x7F, value(s) = m * 2^k.
// RN(S / m) by Markstein's quotient correction (q0 = RN(S * RN(1/m)),
// r = S - m q0 exactly, q = RN(q0 + r * RN(1/m))), exact for every binary32 S
// and m = 1..15 (checked exhaustively over all significands in the test
// suite); the power of two is then applied exactly.  With bf16 data and a
// finite encode scale the quotient is never below 2^-126, where the rounding
// of the two-step form and of a direct division could differ.
__device__ __forceinline__ float div_by_e4m3(float S, uint32_t s, const float* inv) {
    const uint32_t ef = s >> 3, mt = s & 7u;
    const uint32_t m = ef ? 8u + mt : mt;
    const int k = ef ? (int)ef - 10 : -9;  // value(s) = m * 2^k
    const float c = inv[m];
    const float fm = (float)m;
    const float q0 = __fmul_rn(S, c);
    const float r = __fmaf_rn(-q0, fm, S);
    const float q = __fmaf_rn(r, c, q0);
    return __fmul_rn(q, __uint_as_float((uint32_t)(127 - k) << 23));
}

// Block scale and element multiplier for a block of largest magnitude b.
__device__ __forceinline__ Nvfp4Block nvfp4_block(float b, float S, const float* inv) {
    Nvfp4Block r;
    r.scale = (b == 0.0f) ? 0u : e4m3_of(__fmul_rn(div6_rn(b), S));
    r.rcp = 0.0f;
    if (r.scale != 0u) {
        const float q = div_by_e4m3(S, r.scale, inv);
        r.rcp = (q < 0x1p-126f) ? 0.0f : q;  // flush a subnormal reciprocal to zero
    }
    return r;
}

// Element multiplier of e4m3 scale code s: 0 for s = 0, else
// FTZ(RN(S / value(s))).
__device__ __forceinline__ float nvfp4_rcp(float S, uint32_t s, const float* inv) {
    if (s == 0u) return 0.0f;
    const float q = div_by_e4m3(S, s, inv);
    return (q < 0x1p-126f) ? 0.0f : q;
}

// Element multipliers for a whole warp from 16 exact quotients: lane m
// (1..15) holds q_m = RN(S / m) (Markstein's correction, as in div_by_e4m3)
// and lane 0 holds 0; the multiplier of code s = m * 2^k is then q_m * 2^-k
// (exact scaling), read from lane m by a shuffle, and flushed to zero below
// 2^-126 -- the same value as nvfp4_rcp(S, s, inv).  Every lane of the warp
// must call both functions with the same S.
__device__ __forceinline__ float rcp_lane_quotient(float S, const float* inv, int lane) {
    if (lane < 1 || lane > 15) return 0.0f;
    const float c = inv[lane];
    const float q0 = __fmul_rn(S, c);
    const float r = __fmaf_rn(-q0, (float)lane, S);
    return __fmaf_rn(r, c, q0);
}

__device__ __forceinline__ float nvfp4_rcp_warp(float qm, uint32_t s) {
    const uint32_t ef = s >> 3;
    const uint32_t m = ef ? ((s & 7u) | 8u) : s;  // value(s) = m * 2^k, k = max(ef, 1) - 10
    const float q = __shfl_sync(0xFFFFFFFFu, qm, (int)m);
    const float r = __fmul_rn(q, __uint_as_float((137u - max(ef, 1u)) << 23));
    return (r < 0x1p-126f) ? 0.0f : r;
}

// e4m3 codes of RN(RN(b/6) * S) for two block amaxes b0, b1 (code of b0 in
// bits 0-7, of b1 in bits 8-15): the block scales of nvfp4_block, two at a
// time on packed f32 pairs, with RN(b/6) by the quotient correction of
// div6_rn.  b = 0 gives code 0.
__device__ __forceinline__ uint32_t nvfp4_scale_pair(float b0, float b1, float S) {
    uint16_t r;
    asm("{\n\t"
        ".reg .b64 b, c, m6, ss, q, t;\n\t"
        ".reg .f32 lo, hi;\n\t"
        "mov.b64 b, {%1, %2};\n\t"
        "mov.b64 c, {%4, %4};\n\t"
        "mov.b64 m6, {%5, %5};\n\t"
        "mov.b64 ss, {%3, %3};\n\t"
        "mul.rn.f32x2 q, b, c;\n\t"
        "fma.rn.f32x2 t, q, m6, b;\n\t"
        "fma.rn.f32x2 q, t, c, q;\n\t"
        "mul.rn.f32x2 q, q, ss;\n\t"
        "mov.b64 {lo, hi}, q;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 %0, hi, lo;\n\t"
        "}"
        : "=h"(r)
        : "f"(b0), "f"(b1), "f"(S), "f"(1.0f / 6.0f), "f"(-6.0f));
    return r;
}

// ---------------------------------------------------------------------------
// scale-factor layouts
// ---------------------------------------------------------------------------

__host__ __device__ __forceinline__ int64_t pad_to(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// Byte of (row, k) inside a swizzled region with kv scale columns.
__device__ __forceinline__ int64_t swz_offset(int64_t row, int64_t k, int64_t kv) {
    const int64_t col_tiles = (kv + 3) >> 2;
    const int64_t r = row & 127;
    return (((row >> 7) * col_tiles + (k >> 2)) << 9) + ((((r & 31) << 2) + (r >> 5)) << 2) + (k & 3);
}

// Offset inside a 512-byte tile of (row in tile, k in tile).
__device__ __forceinline__ int swz_in_tile(int r, int kc) { return ((((r & 31) << 2) + (r >> 5)) << 2) + kc; }

// ---------------------------------------------------------------------------
// expert table
// ---------------------------------------------------------------------------

__device__ __forceinline__ bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

// Check one table entry; returns the QZ_DERR_* bits that make it invalid.
// fmt: QZ_FMT_MXFP8 / QZ_FMT_NVFP4; needs_amax: the NVFP4 modes.
__device__ __forceinline__ unsigned entry_errors(const qz_expert& e, int fmt, int layout, bool needs_amax) {
    const int64_t block = (fmt == QZ_FMT_MXFP8) ? 32 : 16;
    unsigned bad = 0;
    if (e.rows < 0 || e.cols <= 0 || (e.cols % block) != 0 || e.ld < e.cols || e.ld > QZ_MAX_LD) bad |= QZ_DERR_SHAPE;
    if (e.rows > 0) {
        if (!e.x || !e.q || !e.sf || (needs_amax && !e.amax)) bad |= QZ_DERR_NULL;
        if (!aligned(e.x, 16) || (e.ld & 7) != 0) bad |= QZ_DERR_ALIGN;
        if (!aligned(e.q, fmt == QZ_FMT_MXFP8 ? 16 : 8)) bad |= QZ_DERR_ALIGN;
        if (layout == QZ_SF_SWIZZLED_128x4 && !aligned(e.sf, 16)) bad |= QZ_DERR_ALIGN;
        if (needs_amax && !aligned(e.amax, 4)) bad |= QZ_DERR_ALIGN;
    }
    return bad;
}

__device__ __forceinline__ qz_expert load_entry(const qz_expert* t, int i) {
    qz_expert e;
    const int64_t* p = reinterpret_cast<const int64_t*>(t + i);
    e.x = reinterpret_cast<const void*>(__ldg(p + 0));
    e.rows = __ldg(p + 1);
    e.cols = __ldg(p + 2);
    e.ld = __ldg(p + 3);
    e.q = reinterpret_cast<void*>(__ldg(p + 4));
    e.sf = reinterpret_cast<uint8_t*>(__ldg(p + 5));
    e.amax = reinterpret_cast<float*>(__ldg(p + 6));
    return e;
}

// Exclusive prefix sum over i in [0, n) of count(i) into s_prefix[0..n] (ints);
// every thread gets the total.  A total above INT32_MAX reports
// QZ_DERR_TOO_LARGE and returns 0 (all CTAs agree).  Contains barriers: every
// thread of the block must call it.
template <typename Count>
__device__ int block_prefix(int n, int* s_prefix, long long* s_scratch, Count count, unsigned* d_err) {
    const int nt = blockDim.x;
    const int per = (n + nt - 1) / nt;
    const int beg = min(n, (int)threadIdx.x * per);
    const int end = min(n, beg + per);
    long long local = 0;
    for (int i = beg; i < end; ++i) local += count(i);
    // inclusive scan of `local` within the warp
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        long long y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) s_scratch[warp] = incl;
    __syncthreads();
    if (threadIdx.x == 0) {
        long long run = 0;
        for (int w = 0; w < nt / 32; ++w) {
            long long t = s_scratch[w];
            s_scratch[w] = run;
            run += t;
        }
        s_scratch[32] = run;
    }
    __syncthreads();
    long long total = s_scratch[32];
    long long run = s_scratch[warp] + incl - local;
    if (total <= 0x7FFFFFFFLL) {
        for (int i = beg; i < end; ++i) {
            s_prefix[i] = (int)run;
            run += count(i);
        }
        if (threadIdx.x == 0) s_prefix[n] = (int)total;
    } else if (threadIdx.x == 0 && blockIdx.x == 0 && d_err) {
        atomicOr(d_err, QZ_DERR_TOO_LARGE);
    }
    __syncthreads();
    return total <= 0x7FFFFFFFLL ? (int)total : 0;
}

// floor(a / b) for 0 <= a, 1 <= b: for a < 2^22 a single-precision estimate (exact
// in binary32: the truncated product of a and the rounded-toward-zero
// reciprocal of b is floor(a / b) or one less) and one correction step.
__device__ __forceinline__ int div_nonneg(int a, int b) {
    if (a >= (1 << 22)) return a / b;
    int q = __float2int_rz(__fmul_rz((float)a, __frcp_rz((float)b)));
    if ((q + 1) * b <= a) ++q;
    return q;
}

// The expert owning unit u: the largest e with s_prefix[e] <= u (empty
// experts share their successor's start and are skipped by the search).
__device__ __forceinline__ int find_owner(const int* s_prefix, int n, int u) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_prefix[mid] <= u) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// A strong (L2-coherent) load without ordering of its own.
__device__ __forceinline__ unsigned ld_relaxed_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

}  // namespace qz
