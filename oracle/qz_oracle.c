/*
 * qz_oracle.c -- CPU oracle for grouped block-scaled (MXFP8 / NVFP4)
 * quantization of MoE expert tensors.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, scalar definition that the
 * CUDA library is checked against.  Only the test suite, the smoke check and
 * the CPU-baseline leg of the benchmark may load it.  It shares no code, header,
 * table or constant with the CUDA library, and the library never calls it.
 *
 * Built with -O2 -fno-fast-math -ffp-contract=off: every `float` expression
 * below is one IEEE binary32 operation rounded to nearest-even, every `double`
 * one binary64 operation (x86-64 SSE, no excess precision, no FMA contraction).
 *
 * Sources (web pages, cited by title and section):
 *  [MX]   NVIDIA-NeMo/RL PR #3804 "perf(refit): batch MXFP8 expert
 *         prequantization" -- Summary; Self-review, "Verified clean".
 *  [FOLD] NVIDIA/Model-Optimizer PR #2750 "Fold fused experts' quantizers into
 *         their weights shard-locally" -- review of the weight_scale_2 slicing;
 *         commit notes on NVFP4 zero-block scales and nibble packers.
 *  [LSF]  NVIDIA/TensorRT-LLM PR #17452 "NVFP4 linear-SF AllReduce epilogue" --
 *         commit 1 (linear SF offset), commit 2 (quantize from the bf16 norm),
 *         commit 3 (fp4_quantize parity test).
 *  [SPL]  NVIDIA/TransformerEngine PR #3800 (row-scaled NVFP4 split
 *         quantization) -- Description; Changes.
 *  [CAR]  NVIDIA/TensorRT-LLM PR #17453 "MXFP8 carrier and quantize folds" --
 *         commit 2 (tl.func quantize, FTZ reciprocal), commit 3 (zeroed invented
 *         SF rows), commit 6 (RESIDUAL_RMS_NORM_OUT_QUANT_MXFP8).
 *  Number formats: OCP Microscaling Formats (MX) v1.0 (e4m3, e2m1, E8M0).
 *  Swizzled SF layout: cuBLAS documentation, "1D Block Scaling Factors Layout".
 *
 * Readings where the pages leave a step open (each is listed in the design
 * notes of the repository):
 *  R1 E8M0 exponent: the smallest integer e with amax <= 448 * 2^e, clamped
 *     below at -127 (byte 0x00), which also covers amax == 0.
 *  R2 NVFP4 two-level scale: g = RN32(A / 2688) is the stored FP32 decode
 *     scale, S = RN32(1 / g) the encode scale (0 when g == 0).
 *  R3 NVFP4 block scale: v = RN32(RN32(b / 6) * S), s = e4m3(v).
 *  R4 NVFP4 element: y = RN32(x * rcp), rcp = FTZ(RN32(S / s)), q = e2m1(y).
 *  R5 Nibble order: first element of a pair in the low nibble.
 *  R6 Swizzled 128x4 tile: 512 bytes ordered [row%32][(row/32)%4][k%4];
 *     tiles row-block-major; padding bytes are 0x00.
 *  R7 Signed zero: the sign bit of the scaled element is kept.
 *  R8 RMSNorm over h = bf16(x + r); y = bf16(h * rstd * gamma).
 *  R11 Dequantization: the exact product of code value, block scale value
 *     (and the NVFP4 decode scale g), rounded once to bf16.
 *  R12 Attention decode merge: partial outputs weighted by exp(lse - max lse),
 *     normalised, rounded to bf16 (binary64 inside), then MXFP8 as usual.
 *  R14 Fused gate|up split: rows [0, cut) and [cut, rows), scales cut with
 *     their rows and laid out anew per part; a scale block that covers rows
 *     on both sides of the cut is refused.
 *  R15 AllReduce ahead of the epilogue: the reduced element is the bf16
 *     rounding of a binary32 sum taken in rank order, identical on every rank.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* Plain helpers                                                              */
/* ------------------------------------------------------------------------- */

/* Round a non-negative double to an integer, ties to the even integer. */
static double round_half_even(double v)
{
    double f = floor(v);
    double r = v - f;
    if (r > 0.5) return f + 1.0;
    if (r < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

static float f32_from_bits(uint32_t u)
{
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static uint32_t bits_from_f32(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
float qzo_bf16_value(uint16_t bits)
{
    return f32_from_bits(((uint32_t)bits) << 16);
}

/* Round a double to the nearest bfloat16 (8 significant bits, exponent range
 * of binary32, subnormal step 2^-133), ties to even.  Values beyond the largest
 * finite bfloat16 round to infinity (outside every workload here). */
uint16_t qzo_bf16_from_double(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (a == 0.0) return sign;
    if (isnan(a)) return 0x7FC0u;
    int E;
    frexp(a, &E);          /* a = m * 2^E, m in [0.5, 1)  ->  2^(E-1) <= a */
    int e = E - 1;         /* a in [2^e, 2^(e+1)) */
    if (e < -126) e = -126; /* subnormal range shares the step of 2^-126 */
    double step = ldexp(1.0, e - 7);
    double n = round_half_even(a / step);
    double r = n * step;   /* exact: n <= 256 */
    if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u);
    float rf = (float)r;   /* exact: r has at most 8 significant bits */
    return (uint16_t)(sign | (bits_from_f32(rf) >> 16));
}

/* ------------------------------------------------------------------------- */
/* e4m3 ("fn" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits,     */
/* no infinities, 0x7F/0xFF are NaN, largest finite 448.  (OCP MX v1.0.)       */
/* ------------------------------------------------------------------------- */

double qzo_e4m3_value(uint8_t code)
{
    int s = code >> 7, ef = (code >> 3) & 0xF, m = code & 7;
    double mag;
    if (ef == 0xF && m == 7) return NAN;
    if (ef == 0) mag = ldexp((double)m, -9);               /* m/8 * 2^-6 */
    else mag = ldexp(8.0 + m, ef - 7 - 3);                 /* (1+m/8) * 2^(ef-7) */
    return s ? -mag : mag;
}

/* Round-to-nearest-even with saturation to +-448 (the "satfinite" rule).
 * The sign of the input is always carried to the code, zeros included (R7). */
uint8_t qzo_e4m3_encode(float x)
{
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (isnan(a)) return 0x7F;
    if (a > 448.0) a = 448.0;                /* saturate */
    if (a < ldexp(1.0, -6)) {
        /* subnormal grid: multiples of 2^-9; n == 8 is the smallest normal */
        double n = round_half_even(a / ldexp(1.0, -9));
        return (uint8_t)(sign | (uint8_t)n);
    }
    int E;
    frexp(a, &E);
    int e = E - 1;                            /* a in [2^e, 2^(e+1)), e in [-6, 8] */
    double n = round_half_even(a / ldexp(1.0, e - 3)); /* n in [8, 16] */
    if (n == 16.0) { n = 8.0; e += 1; }
    return (uint8_t)(sign | (uint8_t)(((e + 7) << 3) | ((int)n - 8)));
}

/* ------------------------------------------------------------------------- */
/* e2m1: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit; magnitudes         */
/* 0, 0.5, 1, 1.5, 2, 3, 4, 6.  (OCP MX v1.0.)                                 */
/* ------------------------------------------------------------------------- */

double qzo_e2m1_value(uint8_t code)
{
    int s = (code >> 3) & 1, ef = (code >> 1) & 3, m = code & 1;
    double mag = (ef == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, ef - 1);
    return s ? -mag : mag;
}

/* Round-to-nearest-even with saturation to +-6; sign carried (R7).
 * Returns the 4-bit code in the low nibble. */
uint8_t qzo_e2m1_encode(float x)
{
    uint8_t sign = signbit(x) ? 0x8 : 0x0;
    double a = fabs((double)x);
    if (isnan(a)) a = 6.0;                   /* outside the contract */
    if (a > 6.0) a = 6.0;
    if (a < 1.0) {
        /* subnormal grid: multiples of 0.5; n == 2 is the smallest normal */
        double n = round_half_even(a / 0.5);
        return (uint8_t)(sign | (uint8_t)n);
    }
    int E;
    frexp(a, &E);
    int e = E - 1;                            /* e in {0, 1, 2} */
    double n = round_half_even(a / ldexp(1.0, e - 1)); /* n in [2, 4] */
    if (n == 4.0) { n = 2.0; e += 1; }
    return (uint8_t)(sign | (uint8_t)(((e + 1) << 1) | ((int)n - 2)));
}

/* ------------------------------------------------------------------------- */
/* MXFP8 block scale ([MX] Self-review: shared quantizer with the E8M0        */
/* zero-scale clamp; [CAR] commit 2: flush-to-zero on the reciprocal).        */
/* ------------------------------------------------------------------------- */

/* R1: smallest integer e with amax <= 448 * 2^e, clamped below at -127.
 * The E8M0 byte is e + 127. */
int qzo_mx_scale_exponent(double amax)
{
    if (!(amax > 0.0)) return -127;           /* zero block: clamp */
    int E;
    frexp(amax, &E);
    int e = E - 10;                           /* 448 * 2^(E-10) < 2^(E-1) <= amax */
    while (amax > ldexp(448.0, e)) e += 1;
    if (e < -127) e = -127;
    return e;
}

/* 2^-e as binary32, flushed to zero when it is not a normal number. */
float qzo_mx_reciprocal(int e)
{
    double r = ldexp(1.0, -e);
    if (r < ldexp(1.0, -126)) return 0.0f;
    return (float)r;                          /* exact power of two */
}

/* ------------------------------------------------------------------------- */
/* Scale-factor layouts                                                       */
/* ------------------------------------------------------------------------- */

/* Linear row-major layout ([LSF] commit 1): one byte per (row, k). */
int64_t qzo_sf_offset_linear(int64_t row, int64_t k, int64_t kv)
{
    return row * kv + k;
}

/* Swizzled 128x4 layout (R6).  The region is cut into tiles of 128 rows by
 * 4 scale columns; tiles follow each other row-block-major, each 512 bytes;
 * inside a tile the byte index is ((row%32) * 4 + (row/32)%4) * 4 + k%4. */
int64_t qzo_sf_offset_swizzled(int64_t row, int64_t k, int64_t kv)
{
    int64_t col_tiles = (kv + 3) / 4;
    int64_t tile = (row / 128) * col_tiles + (k / 4);
    int64_t r = row % 128;
    int64_t inner = ((r % 32) * 4 + (r / 32)) * 4 + (k % 4);
    return tile * 512 + inner;
}

/* Bytes of one expert's SF region.  layout 0: linear rows*kv; layout 1:
 * swizzled, rows padded to 128 and scale columns to 4; empty -> 0. */
int64_t qzo_sf_region_bytes(int64_t rows, int64_t kv, int layout)
{
    if (rows <= 0 || kv <= 0) return 0;
    if (layout == 0) return rows * kv;
    return ((rows + 127) / 128) * 128 * ((kv + 3) / 4) * 4;
}

static int64_t sf_offset(int layout, int64_t row, int64_t k, int64_t kv)
{
    return layout == 0 ? qzo_sf_offset_linear(row, k, kv)
                       : qzo_sf_offset_swizzled(row, k, kv);
}

/* The whole region is first written as 0x00 so that the padded rows and
 * column groups of the swizzled layout read as zero ([CAR] commits 3 and 6). */
static void sf_clear(uint8_t *sf, int64_t rows, int64_t kv, int layout)
{
    int64_t n = qzo_sf_region_bytes(rows, kv, layout);
    for (int64_t i = 0; i < n; i++) sf[i] = 0;
}

/* Linear -> swizzled copy of one SF matrix (the receiver-side conversion
 * mentioned in [MX] Summary); padding written as 0x00. */
void qzo_swizzle(const uint8_t *lin, int64_t rows, int64_t kv, uint8_t *swz)
{
    sf_clear(swz, rows, kv, 1);
    for (int64_t r = 0; r < rows; r++)
        for (int64_t k = 0; k < kv; k++)
            swz[qzo_sf_offset_swizzled(r, k, kv)] = lin[qzo_sf_offset_linear(r, k, kv)];
}

void qzo_unswizzle(const uint8_t *swz, int64_t rows, int64_t kv, uint8_t *lin)
{
    for (int64_t r = 0; r < rows; r++)
        for (int64_t k = 0; k < kv; k++)
            lin[qzo_sf_offset_linear(r, k, kv)] = swz[qzo_sf_offset_swizzled(r, k, kv)];
}

/* ------------------------------------------------------------------------- */
/* MXFP8 quantization of one expert matrix.                                   */
/*   x   : bf16 bits, rows x cols, row stride ld elements                      */
/*   q   : e4m3 codes, rows x cols, dense                                      */
/*   sf  : E8M0 bytes, layout 0 (linear) or 1 (swizzled 128x4)                 */
/* Block = 32 consecutive elements of a row ([MX] Summary and Self-review).   */
/* ------------------------------------------------------------------------- */
void qzo_quantize_mxfp8(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                        uint8_t *q, uint8_t *sf, int layout)
{
    int64_t kv = cols / 32;
    sf_clear(sf, rows, kv, layout);
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t k = 0; k < kv; k++) {
            const uint16_t *blk = x + r * ld + k * 32;
            double amax = 0.0;
            for (int i = 0; i < 32; i++) {
                double a = fabs((double)qzo_bf16_value(blk[i]));
                if (a > amax) amax = a;
            }
            int e = qzo_mx_scale_exponent(amax);
            float rcp = qzo_mx_reciprocal(e);
            sf[sf_offset(layout, r, k, kv)] = (uint8_t)(e + 127);
            for (int i = 0; i < 32; i++) {
                float y = qzo_bf16_value(blk[i]) * rcp;   /* binary32 product */
                q[r * cols + k * 32 + i] = qzo_e4m3_encode(y);
            }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* NVFP4 quantization of one expert matrix ([FOLD] weight_scale_2 review;     */
/* [FOLD] zero block-scale commit; [SPL] Description and Changes;             */
/* [LSF] commit 3).                                                           */
/*   mode 0: per-tensor, A given in amax[0]                                    */
/*   mode 1: per-tensor, A = max |x| over the matrix, written to amax[0]       */
/*   mode 2: per-row,    A_r = max |x| over row r, written to amax[r]          */
/*   q   : packed e2m1, rows x cols/2 bytes, dense, low nibble first (R5)      */
/*   sf  : E4M3 bytes, one per 16 elements, layout 0 or 1                      */
/* ------------------------------------------------------------------------- */

/* Encode scale S from the tensor (or row) amax A (R2). */
static float nvfp4_encode_scale(float A)
{
    float g = A / 2688.0f;            /* stored decode scale, 2688 = 448 * 6 */
    if (g == 0.0f) return 0.0f;
    return 1.0f / g;
}

static void nvfp4_row(const uint16_t *xr, int64_t cols, float S,
                      uint8_t *qr, uint8_t *sf, int64_t r, int64_t kv, int layout)
{
    for (int64_t k = 0; k < kv; k++) {
        const uint16_t *blk = xr + k * 16;
        float b = 0.0f;
        for (int i = 0; i < 16; i++) {
            float a = fabsf(qzo_bf16_value(blk[i]));
            if (a > b) b = a;
        }
        uint8_t s = 0;
        if (b != 0.0f) {
            float v = (b / 6.0f) * S;             /* R3: two binary32 roundings */
            s = qzo_e4m3_encode(v);
        }
        float rcp = 0.0f;                          /* zero scale: no division */
        if ((s & 0x7F) != 0) {
            rcp = S / (float)qzo_e4m3_value(s);   /* R4 */
            if (fabsf(rcp) < ldexp(1.0, -126)) rcp = 0.0f;  /* FTZ */
        }
        sf[sf_offset(layout, r, k, kv)] = s;
        for (int i = 0; i < 16; i += 2) {
            float y0 = qzo_bf16_value(blk[i]) * rcp;
            float y1 = qzo_bf16_value(blk[i + 1]) * rcp;
            qr[k * 8 + i / 2] = (uint8_t)(qzo_e2m1_encode(y0) | (qzo_e2m1_encode(y1) << 4));
        }
    }
    (void)cols;
}

void qzo_quantize_nvfp4(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                        uint8_t *q, uint8_t *sf, int layout, int mode, float *amax)
{
    int64_t kv = cols / 16;
    sf_clear(sf, rows, kv, layout);
    if (mode == 0 || mode == 1) {
        float A;
        if (mode == 0) {
            A = amax[0];
        } else {
            A = 0.0f;
            for (int64_t r = 0; r < rows; r++)
                for (int64_t c = 0; c < cols; c++) {
                    float a = fabsf(qzo_bf16_value(x[r * ld + c]));
                    if (a > A) A = a;
                }
            amax[0] = A;
        }
        float S = nvfp4_encode_scale(A);
        for (int64_t r = 0; r < rows; r++)
            nvfp4_row(x + r * ld, cols, S, q + r * (cols / 2), sf, r, kv, layout);
    } else {
        for (int64_t r = 0; r < rows; r++) {
            float A = 0.0f;
            for (int64_t c = 0; c < cols; c++) {
                float a = fabsf(qzo_bf16_value(x[r * ld + c]));
                if (a > A) A = a;
            }
            amax[r] = A;
            nvfp4_row(x + r * ld, cols, nvfp4_encode_scale(A), q + r * (cols / 2), sf, r, kv, layout);
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Residual add + RMSNorm ([LSF] commit 2; [CAR] commit 6).                   */
/*   h[t,i] = bf16(x + r)            (also the updated residual)              */
/*   rstd   = 1 / sqrt(mean_i h^2 + eps)   (binary64)                          */
/*   y[t,i] = bf16(h * rstd * gamma_i)      (R8)                               */
/* ------------------------------------------------------------------------- */
void qzo_residual_rmsnorm(const uint16_t *x, const uint16_t *res, const uint16_t *gamma,
                          float eps, int64_t T, int64_t H, uint16_t *y, uint16_t *h)
{
    for (int64_t t = 0; t < T; t++) {
        double ss = 0.0;
        for (int64_t i = 0; i < H; i++) {
            double s = (double)qzo_bf16_value(x[t * H + i]) + (double)qzo_bf16_value(res[t * H + i]);
            uint16_t hb = qzo_bf16_from_double(s);
            h[t * H + i] = hb;
            double hv = (double)qzo_bf16_value(hb);
            ss += hv * hv;
        }
        double rstd = 1.0 / sqrt(ss / (double)H + (double)eps);
        for (int64_t i = 0; i < H; i++) {
            double hv = (double)qzo_bf16_value(h[t * H + i]);
            double gv = (double)qzo_bf16_value(gamma[i]);
            y[t * H + i] = qzo_bf16_from_double(hv * rstd * gv);
        }
    }
}

/* The fused epilogue: the norm, then the quantizer applied to the very bf16
 * values of y ([LSF] commit 3; [CAR] commit 6: quantizing inside the epilogue
 * equals quantizing norm_out afterwards).  fmt 0: MXFP8; fmt 1: NVFP4 with the
 * per-tensor amax A given in *amax. */
void qzo_rmsnorm_quantize(const uint16_t *x, const uint16_t *res, const uint16_t *gamma,
                          float eps, int64_t T, int64_t H, uint16_t *y, uint16_t *h,
                          int fmt, uint8_t *q, uint8_t *sf, int layout, float *amax)
{
    qzo_residual_rmsnorm(x, res, gamma, eps, T, H, y, h);
    if (fmt == 0) qzo_quantize_mxfp8(y, T, H, H, q, sf, layout);
    else qzo_quantize_nvfp4(y, T, H, H, q, sf, layout, 0, amax);
}

/* ------------------------------------------------------------------------- */
/* The AllReduce that opens the epilogue ([LSF] commit 2 and [CAR] commit 6:  */
/* the tensor-parallel AllReduce hands the epilogue its input x).             */
/*   R15 out[i] = bf16(acc), acc = x_0[i], then acc = RN32(acc + x_r[i]) for  */
/*       r = 1 .. n-1 (binary32, rank order), so that every rank reduces to   */
/*       the same bits; the epilogue above then runs on out as its x.         */
/*   xs : n pointers to bf16 arrays of count elements                         */
/* ------------------------------------------------------------------------- */
void qzo_rank_sum(const uint16_t *const *xs, int n, int64_t count, uint16_t *out)
{
    for (int64_t i = 0; i < count; i++) {
        float acc = qzo_bf16_value(xs[0][i]);
        for (int r = 1; r < n; r++) acc = acc + qzo_bf16_value(xs[r][i]);
        out[i] = qzo_bf16_from_double((double)acc);
    }
}

/* ------------------------------------------------------------------------- */
/* Dequantization: the decoded tensor of a quantized one ([SPL] Changes: the  */
/* regression tests compare dequantized values; [CAR] commit 1: the dequant   */
/* reference path works on the high-precision tensor).                        */
/*   R11 an element's decoded value is the exact product of its code's value  */
/*       and its block scale's value (and, for NVFP4, of the FP32 decode      */
/*       scale g = RN32(A / 2688) of R2), rounded once to bf16 (RNE); the     */
/*       product has at most 4 + 8 (MXFP8) or 2 + 4 + 24 (NVFP4) significant  */
/*       bits, so binary64 holds it exactly.                                  */
/*   y   : bf16 [rows, cols], row stride ldy                                  */
/* ------------------------------------------------------------------------- */

void qzo_dequantize_mxfp8(const uint8_t *q, const uint8_t *sf, int64_t rows, int64_t cols,
                          int layout, uint16_t *y, int64_t ldy)
{
    int64_t kv = cols / 32;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++) {
            int byte = sf[sf_offset(layout, r, c / 32, kv)];
            double v = qzo_e4m3_value(q[r * cols + c]) * ldexp(1.0, byte - 127);
            y[r * ldy + c] = qzo_bf16_from_double(v);
        }
}

/* amax: per-tensor amax[0] (per_row == 0) or per-row amax[r] (per_row != 0). */
void qzo_dequantize_nvfp4(const uint8_t *q, const uint8_t *sf, const float *amax, int per_row,
                          int64_t rows, int64_t cols, int layout, uint16_t *y, int64_t ldy)
{
    int64_t kv = cols / 16;
    for (int64_t r = 0; r < rows; r++) {
        float A = per_row ? amax[r] : amax[0];
        float g = A / 2688.0f;                         /* R2: binary32 decode scale */
        for (int64_t c = 0; c < cols; c++) {
            uint8_t byte = q[r * (cols / 2) + c / 2];
            uint8_t code = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);   /* R5 */
            uint8_t s = sf[sf_offset(layout, r, c / 16, kv)];
            double v = qzo_e2m1_value(code) * qzo_e4m3_value(s) * (double)g;
            y[r * ldy + c] = qzo_bf16_from_double(v);
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Attention decode merge with its MXFP8 form ([CAR] commit 3: the merge      */
/* kernel that finishes flash-decoding writes the attention output and its    */
/* MXFP8 form, and the SF rows swizzling invents past the last live row).     */
/*   R12 S partial outputs O[s, t, :] (binary32) with log-sum-exps lse[s, t]  */
/*       (natural log, binary32) merge as                                     */
/*         y[t, i] = bf16( sum_s w_s O[s, t, i] / sum_s w_s ),                */
/*         w_s = exp(lse[s, t] - max_s lse[s, t])        (binary64 throughout) */
/*       and y is then quantized to MXFP8 as qzo_quantize_mxfp8 does.         */
/*   O: [S, T, H] contiguous; lse: [S, T]; y: [T, H] bf16                     */
/* ------------------------------------------------------------------------- */

void qzo_attention_merge(const float *O, const float *lse, int64_t S, int64_t T, int64_t H, uint16_t *y)
{
    for (int64_t t = 0; t < T; t++) {
        double m = -INFINITY;
        for (int64_t s = 0; s < S; s++)
            if ((double)lse[s * T + t] > m) m = (double)lse[s * T + t];
        double wsum = 0.0;
        for (int64_t s = 0; s < S; s++) wsum += exp((double)lse[s * T + t] - m);
        for (int64_t i = 0; i < H; i++) {
            double acc = 0.0;
            for (int64_t s = 0; s < S; s++)
                acc += exp((double)lse[s * T + t] - m) * (double)O[(s * T + t) * H + i];
            y[t * H + i] = qzo_bf16_from_double(acc / wsum);
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Gate|up split of a folded fused expert ([FOLD] keep-fused fold: the fused  */
/* (2I, H) expert is quantized as one tensor, gate and up sharing one         */
/* per-tensor amax and so one weight_scale_2; the split then cuts the folded  */
/* payload and its scales by weight rows into gate and up, each with its own  */
/* storage, and refuses a scale block that the cut would divide).             */
/*   R14 part 0 = weight rows [0, cut), part 1 = rows [cut, rows).            */
/*       fmt 0 MXFP8 / 1 NVFP4: one scale row per weight row, so every cut    */
/*       is exact; each part's SF region is laid out anew in dst_layout with  */
/*       its own padding (0x00), whatever src_layout was.                     */
/*       fmt 2 FP8 with FP32 scales of 128 x 128 blocks (linear only, scale   */
/*       matrix [ceil(rows/128), ceil(cols/128)]): a scale row covers 128     */
/*       weight rows, so a cut inside a block (cut % 128 != 0, cut < rows) is */
/*       refused.                                                             */
/*       amax_kind 0: none; 1: one per-tensor amax, given to both parts; 2:  */
/*       one amax per row, cut with the rows.                                 */
/*   Returns 0, or -1 for a refused cut (nothing is written then).            */
/* ------------------------------------------------------------------------- */

int qzo_split_fused(int fmt, const uint8_t *q, const uint8_t *sf, const float *amax, int amax_kind,
                    int64_t rows, int64_t cols, int64_t cut, int src_layout, int dst_layout,
                    uint8_t *q0, uint8_t *sf0, float *amax0, uint8_t *q1, uint8_t *sf1, float *amax1)
{
    int64_t row_block = (fmt == 2) ? 128 : 1;       /* weight rows per scale row */
    if (cut < 0 || cut > rows) return -1;
    if (cut % row_block != 0 && cut < rows) return -1;

    int64_t row_bytes = (fmt == 1) ? cols / 2 : cols;
    int64_t first[2] = {0, cut};
    int64_t count[2] = {cut, rows - cut};
    uint8_t *qo[2] = {q0, q1};
    uint8_t *so[2] = {sf0, sf1};
    float *ao[2] = {amax0, amax1};

    for (int p = 0; p < 2; p++) {
        for (int64_t i = 0; i < count[p] * row_bytes; i++) qo[p][i] = q[first[p] * row_bytes + i];

        if (fmt == 2) {
            /* FP32 block scales, row-major: scale rows [first/128, first/128 + ceil(count/128)) */
            int64_t scols = (cols + 127) / 128;
            int64_t srow0 = first[p] / 128;
            int64_t srows = (count[p] + 127) / 128;
            for (int64_t i = 0; i < srows * scols * 4; i++) so[p][i] = sf[srow0 * scols * 4 + i];
        } else {
            int64_t kv = cols / (fmt == 0 ? 32 : 16);
            sf_clear(so[p], count[p], kv, dst_layout);
            for (int64_t r = 0; r < count[p]; r++)
                for (int64_t k = 0; k < kv; k++)
                    so[p][sf_offset(dst_layout, r, k, kv)] = sf[sf_offset(src_layout, first[p] + r, k, kv)];
        }

        if (amax_kind == 1) ao[p][0] = amax[0];
        if (amax_kind == 2)
            for (int64_t r = 0; r < count[p]; r++) ao[p][r] = amax[first[p] + r];
    }
    return 0;
}
