/*
 * qz.h -- C ABI of the grouped block-scaled quantization library (libqz.so)
 * for NVIDIA B200 (sm_100a).
 *
 * The library quantizes groups of bf16 matrices ("experts") to
 *   MXFP8: e4m3 payload, one E8M0 scale byte per 32 consecutive row elements;
 *   NVFP4: packed e2m1 payload, one E4M3 scale byte per 16 consecutive row
 *          elements, plus an FP32 second-level amax per tensor or per row;
 * and writes each expert's scale factors (SF) in the linear row-major layout
 * or the swizzled 128x4 layout, each expert into its own independently padded
 * region.  A fused residual-add + RMSNorm entry point writes the bf16 norm and
 * its quantized form from one read; its AllReduce form first sums up to eight
 * tensor-parallel ranks' inputs, read through (peer-mapped) device pointers.
 *
 * Conventions that hold for every entry point:
 *  - Pointers whose name starts with d_, and every pointer inside a table, are
 *    DEVICE pointers.  The caller owns every buffer; the library allocates
 *    nothing.  Its only state is a per-device cache of launch limits and the
 *    static device scratch of qz_quantize_grouped_nvfp4_compute_noalloc (with
 *    that array's device address, looked up once per device).
 *  - `stream` is a cudaStream_t (NULL: the legacy default stream).  Every call
 *    is asynchronous on that stream; inputs must be ready on it.  No call
 *    synchronizes.
 *  - Arguments the host can check are checked before anything is launched; on
 *    error nothing is written and the status says why.  Table entries live in
 *    device memory, so they are checked by the kernel: an invalid entry is
 *    skipped (none of its bytes are written) and, when opts->d_err is given,
 *    the reason bits below are OR-ed into *opts->d_err.
 *  - Only the bytes named by the table (payload rows, the expert's own SF
 *    region, its amax slot(s)) are written: re-quantizing one expert is a call
 *    with a one-entry table and touches no other expert's storage.
 *  - Element encodings: RNE with saturation (satfinite); the sign of a zero or
 *    of a value that rounds to zero is kept; an all-zero block gets scale byte
 *    0x00.  Non-finite inputs are outside the contract.
 *
 * Citations (web pages, by title and section):
 *  [MX]   NVIDIA-NeMo/RL PR #3804 "perf(refit): batch MXFP8 expert
 *         prequantization" -- Summary, Why, Self-review.
 *  [FOLD] NVIDIA/Model-Optimizer PR #2750 "Fold fused experts' quantizers into
 *         their weights shard-locally" -- weight_scale_2 review; zero-block notes.
 *  [LSF]  NVIDIA/TensorRT-LLM PR #17452 "NVFP4 linear-SF AllReduce epilogue" --
 *         commits 1-3.
 *  [SPL]  NVIDIA/TransformerEngine PR #3800 (row-scaled NVFP4 split
 *         quantization) -- Description, Changes.
 *  [CAR]  NVIDIA/TensorRT-LLM PR #17453 "MXFP8 carrier and quantize folds" --
 *         commits 2, 3, 5, 6.
 */
#ifndef QZ_H
#define QZ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum qz_status {
    QZ_OK = 0,
    QZ_ERR_INVALID_ARG = 1, /* bad count, null pointer, unknown enum, bad size */
    QZ_ERR_ALIGNMENT = 2,   /* a host-visible pointer or stride is misaligned */
    QZ_ERR_UNSUPPORTED = 3, /* a shape/format/layout combination the kernels do not cover */
    QZ_ERR_CUDA = 4         /* the CUDA runtime reported an error at launch */
} qz_status;

typedef enum qz_sf_layout {
    QZ_SF_LINEAR = 0,        /* byte (row, k) at row * kv + k              ([LSF] commit 1) */
    QZ_SF_SWIZZLED_128x4 = 1 /* 128-row x 4-column tiles of 512 bytes, row-block-major;
                                inside a tile byte ((row%32)*4 + (row%128)/32)*4 + k%4;
                                rows padded to 128 and k to 4 with 0x00 ([CAR] commits 3, 6;
                                cuBLAS "1D Block Scaling Factors Layout") */
} qz_sf_layout;

typedef enum qz_format {
    QZ_FMT_MXFP8 = 0,
    QZ_FMT_NVFP4 = 1,
    QZ_FMT_FP8_BLOCK128 = 2 /* e4m3 payload with FP32 scales of 128 x 128 blocks, row-major
                               [ceil(rows/128), ceil(cols/128)], linear only ([FOLD]: FP8 2-D
                               blockwise experts).  Accepted by qz_sf_bytes and
                               qz_split_fused_experts only; nothing here quantizes to it. */
} qz_format;

/* What a tensor's FP32 amax slot holds (qz_split_fused_experts). */
typedef enum qz_amax_kind {
    QZ_AMAX_NONE = 0,       /* no amax (MXFP8, FP8_BLOCK128) */
    QZ_AMAX_PER_TENSOR = 1, /* one float per tensor (NVFP4 per-tensor scale) */
    QZ_AMAX_PER_ROW = 2     /* one float per row (row-scaled NVFP4) */
} qz_amax_kind;

typedef enum qz_nvfp4_scale_mode {
    QZ_NVFP4_PER_TENSOR_GIVEN = 0,   /* amax[0] is an input (e.g. a calibrated value) */
    QZ_NVFP4_PER_TENSOR_COMPUTE = 1, /* amax[0] = max |x| over the expert, written by the call */
    QZ_NVFP4_PER_ROW = 2             /* amax[r] = max |x| over row r, written by the call ([SPL]) */
} qz_nvfp4_scale_mode;

/* Reason bits OR-ed into *opts->d_err for table entries a kernel skipped. */
#define QZ_DERR_SHAPE 0x1u     /* rows < 0, cols <= 0, cols not a multiple of the block,
                                  ld < cols or ld > QZ_MAX_LD */
#define QZ_DERR_NULL 0x2u      /* x, q, sf (or amax for NVFP4) null on a non-empty entry */
#define QZ_DERR_ALIGN 0x4u     /* x not 16-byte aligned or ld not a multiple of 8; q not
                                  16-byte (MXFP8) / 8-byte (NVFP4) aligned; sf not 16-byte
                                  aligned (swizzled); amax not 4-byte aligned */
#define QZ_DERR_TOO_LARGE 0x8u /* the call's total tile or row count exceeds 2^31 - 1 */
#define QZ_DERR_TIMEOUT 0x10u  /* a bounded wait of the single-launch computed-amax path (quantize
                                  warps waiting for an expert's amax, or the copy, amax and
                                  publishing warps waiting on one another) exceeded
                                  qz_launch_opts.wait_limit_ns; the launch stopped early and some
                                  outputs are unwritten (no such wait is expected to expire) */
#define QZ_DERR_CUT 0x20u      /* qz_split_fused_experts: the cut falls inside a scale block
                                  (FP8_BLOCK128: cut not a multiple of 128 and not the end) */

/* Largest table a grouped call accepts (the kernels keep the table's prefix
 * sums in shared memory). */
#define QZ_MAX_EXPERTS 4096

/* Largest row stride (elements) of a table entry: offsets inside a 128-row
 * tile are 32-bit. */
#define QZ_MAX_LD (1LL << 24)

/* Largest hidden size of qz_rmsnorm_quantize (one row is held in registers). */
#define QZ_MAX_HIDDEN 16384

/* One table entry per expert ([MX] Summary: many same-shape experts per call;
 * [SPL] Description: one concatenated activation split unevenly by expert).
 * The table itself and every pointer in it are device memory.  56 bytes. */
typedef struct qz_expert {
    const void *x; /* bf16 [rows, cols], row stride ld elements.  For a split
                      activation: base + row_offset * ld. */
    int64_t rows;  /* may be 0 (an empty split): nothing is read or written */
    int64_t cols;  /* quantization axis; multiple of 32 (MXFP8) or 16 (NVFP4) */
    int64_t ld;    /* row stride of x in elements, >= cols, <= QZ_MAX_LD, multiple of 8 */
    void *q;       /* payload, row-major and dense (16-byte aligned for MXFP8, 8-byte
                      for NVFP4): MXFP8 e4m3 [rows, cols];
                      NVFP4 e2m1 [rows, cols/2], element 2j in the low nibble
                      of byte j and element 2j+1 in the high nibble */
    uint8_t *sf;   /* this expert's SF region of qz_sf_bytes(rows, cols, fmt, layout) bytes */
    float *amax;   /* NVFP4: per-tensor amax (one float: input in GIVEN mode,
                      output in COMPUTE mode) or per-row amax [rows] (output);
                      MXFP8: unused (may be NULL) */
} qz_expert;

/* One linear -> swizzled conversion ([MX] Summary: the receiver-side MXFP8
 * layout conversion).  Device pointers. */
typedef struct qz_sf_pair {
    const uint8_t *src; /* linear SF [rows, kv], row-major, dense */
    uint8_t *dst;       /* swizzled region of pad(rows,128) * pad(kv,4) bytes, 16-byte aligned */
    int64_t rows;       /* >= 0 */
    int64_t kv;         /* scale columns, >= 1 */
} qz_sf_pair;

/* One expert's quantized tensor to decode (lives in DEVICE memory, 56 bytes). */
typedef struct qz_dq_expert {
    const void *q;      /* MXFP8: e4m3 [rows, cols], 16-byte aligned; NVFP4: packed e2m1
                           [rows, cols/2] (low nibble first), 8-byte aligned; dense rows */
    const uint8_t *sf;  /* this expert's SF region in the layout given to the call */
    const float *amax;  /* NVFP4: amax[0] (per tensor) or amax[rows] (per row), 4-byte
                           aligned; MXFP8: unused (may be NULL) */
    int64_t rows;       /* >= 0 (0: empty, nothing is written) */
    int64_t cols;       /* multiple of 32 (MXFP8) / 16 (NVFP4) */
    void *y;            /* bf16 output [rows, cols], 16-byte aligned, row stride ldy */
    int64_t ldy;        /* >= cols, multiple of 8, <= QZ_MAX_LD */
} qz_dq_expert;

/* One folded fused expert to cut in two (qz_split_fused_experts): part 0 is
 * weight rows [0, cut) (the gate), part 1 rows [cut, rows) (the up
 * projection).  Device memory, 96 bytes. */
typedef struct qz_fused_split {
    const void *q;       /* folded payload [rows, row_bytes], dense; row_bytes = cols (MXFP8,
                            FP8_BLOCK128) or cols / 2 (NVFP4) */
    const uint8_t *sf;   /* folded scales: the SF region of a [rows, cols] tensor in the call's
                            src_layout (16-byte aligned when swizzled); FP8_BLOCK128: FP32
                            [ceil(rows/128), ceil(cols/128)] row-major, 4-byte aligned */
    const float *amax;   /* QZ_AMAX_PER_TENSOR: amax[0]; QZ_AMAX_PER_ROW: amax[rows]; 4-byte
                            aligned; otherwise unused */
    int64_t rows;        /* fused rows (gate + up), >= 0 */
    int64_t cols;        /* multiple of 32 (MXFP8) / 16 (NVFP4), >= 1 (FP8_BLOCK128); <= QZ_MAX_LD */
    int64_t cut;         /* first row of part 1, 0 <= cut <= rows */
    void *q_out[2];      /* payload of each part [n_p, row_bytes], dense, any alignment (wider
                            copies when 32/16/8-byte aligned); NULL: that part's payload is not
                            copied (a caller keeping views into q) */
    uint8_t *sf_out[2];  /* scales of each part: qz_sf_bytes(n_p, cols, fmt, dst_layout) bytes,
                            padding written 0x00; 16-byte aligned when swizzled, 4-byte for
                            FP8_BLOCK128 */
    float *amax_out[2];  /* QZ_AMAX_PER_TENSOR: one float each, both receive amax[0];
                            QZ_AMAX_PER_ROW: n_p floats each, the rows' amaxes */
} qz_fused_split;

/* Optional launch controls; pass NULL for the defaults. */
typedef struct qz_launch_opts {
    unsigned int *d_err;    /* device word; kernels OR QZ_DERR_* bits into it (never clear it) */
    int max_ctas;           /* 0: one wave of resident CTAs on every SM; > 0: cap on the grid.
                               The results do not depend on it. */
    void *d_workspace;      /* optional device scratch for QZ_NVFP4_PER_TENSOR_COMPUTE: with
                               at least qz_workspace_bytes(n_experts) bytes (4-byte aligned),
                               the call runs one cooperative launch that reads the input from
                               HBM once (the quantize side re-reads it from L2) instead of an
                               amax pass and a quantize pass over HBM.  The call zeroes it first (in
                               stream order); calls sharing a workspace must not overlap. */
    size_t workspace_bytes; /* size of d_workspace in bytes */
    int64_t elems_hint;     /* qz_quantize_grouped_mxfp8 and the MXFP8 qz_dequantize_grouped: the call's
                               elements (sum of rows * cols over the table), 0 if unknown.  With it, the
                               grid is sized to the work: about one CTA per ten 128 x 128 tiles, in whole
                               waves (1 to 16), which streams large calls faster than one persistent
                               wave, and one CTA per tile below one wave; without it, one wave.  Any
                               value gives the same results. */
    int64_t wait_limit_ns;  /* single-launch computed-amax path (a workspace, or the allocation-free entry
                               point): the limit of each of its bounded waits, in nanoseconds of the
                               GPU's global timer; 0 = the default of 20 ms.  A wait that runs out
                               sets QZ_DERR_TIMEOUT and ends the launch early. */
    unsigned int test_flags; /* 0 in normal use.  QZ_TEST_WITHHOLD_ARRIVALS makes the single-launch
                               computed-amax path withhold the counts that release its quantize
                               warps, so their waits run out: a test of the timeout path that
                               needs no fault. */
    unsigned int launch_flags; /* QZ_OPT_INDEPENDENT: see below; 0 otherwise. */
} qz_launch_opts;

/* qz_launch_opts.test_flags bits. */
#define QZ_TEST_WITHHOLD_ARRIVALS 0x1u

/* qz_launch_opts.launch_flags bits.
 * The MXFP8 and NVFP4 tile kernels (qz_quantize_grouped_mxfp8; NVFP4 in the
 * GIVEN and PER_TENSOR_COMPUTE-without-workspace modes) are launched with
 * programmatic stream serialization: each lets the next such launch on the
 * stream begin while its own last CTAs still run.  By default a launch then
 * waits, before it reads anything, until the launch before it has completed
 * and its writes are visible, so stream order holds as for any launch.
 * QZ_OPT_INDEPENDENT declares that this call's table and inputs are written,
 * and its outputs read or written, by no kernel that may still be running on
 * the stream -- e.g. a series of calls on disjoint experts whose weights were
 * written earlier -- and skips that wait: the call's tiles start as soon as
 * the previous call's CTAs free their SMs, which recovers, on one stream, the
 * ramp and tail of each short call.  A wrong declaration is a data race. */
#define QZ_OPT_INDEPENDENT 0x1u

/* Bytes of device scratch qz_quantize_grouped_nvfp4 uses for
 * QZ_NVFP4_PER_TENSOR_COMPUTE when given a workspace; 0 for n_experts outside
 * [1, QZ_MAX_EXPERTS]. */
size_t qz_workspace_bytes(int n_experts);

/* Bytes of one expert's SF region: rows * (cols/block) for the linear layout,
 * pad(rows,128) * pad(cols/block,4) for the swizzled one, 0 when rows == 0.
 * fmt selects the block (32 for MXFP8, 16 for NVFP4); QZ_FMT_FP8_BLOCK128
 * (linear only) gives 4 * ceil(rows/128) * ceil(cols/128).  Returns 0 for
 * arguments that describe no valid region (negative sizes, cols not a
 * multiple of the block, unknown enums). */
size_t qz_sf_bytes(int64_t rows, int64_t cols, int fmt, int layout);

/* MXFP8 quantization of every expert in d_table, in one persistent launch
 * ([MX] Summary, Why, Self-review; [CAR] commits 2, 3).  Per 32-element block
 * B of a row: e = the smallest integer with max|B| <= 448 * 2^e, clamped below
 * at -127 (zero blocks: -127); scale byte = e + 127; payload = e4m3(x * 2^-e).
 * Errors: QZ_ERR_INVALID_ARG for n_experts < 0 or > QZ_MAX_EXPERTS, a NULL
 * table with n_experts > 0, or an unknown layout; QZ_ERR_CUDA if the launch
 * fails.  n_experts == 0 launches nothing and returns QZ_OK. */
qz_status qz_quantize_grouped_mxfp8(const qz_expert *d_table, int n_experts, int layout,
                                    void *stream, const qz_launch_opts *opts);

/* NVFP4 quantization of every expert in d_table ([FOLD] weight_scale_2 review
 * and zero-block notes; [SPL] Description, Changes; [LSF] commit 3).
 * With A the tensor (or row) amax: g = RN32(A / 2688) is the FP32 decode
 * scale, S = RN32(1 / g) (0 if g == 0) the encode scale; per 16-element block
 * with amax b: scale s = e4m3(RN32(RN32(b / 6) * S)) (0 if b == 0); payload
 * q = e2m1(RN32(x * r)), r = FTZ(RN32(S / s)) (0 if s == 0).
 * PER_TENSOR_COMPUTE without a workspace runs a clear, an amax pass and the
 * quantize pass (three launches in stream order, the input read twice from
 * HBM); with opts->d_workspace it runs one cooperative launch (plus a memset
 * of the workspace) in which bulk copies bring every expert from HBM into
 * shared memory for its amax, ahead of quantize warps that re-read the expert
 * from L2 once every CTA's share of its amax is in (bounded waits:
 * wait_limit_ns).
 * PER_ROW reads each row once.
 * Entries may share one amax slot, so that the gate and up halves of a fused
 * expert ([FOLD]: one amax over the fused (2I, H) slice, one weight_scale_2)
 * are quantized straight into their own storage in one call: in GIVEN mode
 * the shared value is read by both, and in COMPUTE mode without a workspace
 * every entry sharing the slot feeds the same maximum before any of them is
 * quantized.  The single-launch COMPUTE path (with opts->d_workspace, and
 * qz_quantize_grouped_nvfp4_compute_noalloc) keeps one amax per entry: there
 * entries must not share a slot.
 * Errors as below, plus QZ_ERR_INVALID_ARG for a workspace smaller than
 * qz_workspace_bytes(n_experts) and QZ_ERR_ALIGNMENT for one not 4-byte
 * aligned.
 * Errors as for qz_quantize_grouped_mxfp8, plus QZ_ERR_INVALID_ARG for an
 * unknown mode. */
qz_status qz_quantize_grouped_nvfp4(const qz_expert *d_table, int n_experts, int mode, int layout,
                                    void *stream, const qz_launch_opts *opts);

/* Fused residual add + RMSNorm + quantize of T rows of H elements ([LSF]
 * commits 2, 3; [CAR] commit 6):
 *   h = bf16(x + residual)            -> d_residual_out (nullable)
 *   y = bf16(h / sqrt(mean(h^2) + eps) * gamma)   -> d_norm_out
 *   q, sf = quantize(y) exactly as the grouped entry points would quantize
 *           d_norm_out (MXFP8, or NVFP4 with the per-tensor amax *d_global_amax)
 * All of x, residual, norm_out, residual_out are bf16 [T, H] row-major, gamma
 * bf16 [H].  The swizzled layout's padded rows (T .. pad(T,128)-1) are written
 * as 0x00 by the kernel itself.
 * Errors: QZ_ERR_INVALID_ARG for T < 0, H <= 0, H > QZ_MAX_HIDDEN, H not a
 * multiple of the block (32 / 16), null required pointers, unknown fmt or
 * layout, NVFP4 without d_global_amax; QZ_ERR_UNSUPPORTED for the swizzled
 * layout with H/block not a multiple of 4 (the padded scale columns would be
 * unreachable, [CAR] commit 6); QZ_ERR_ALIGNMENT for bf16 pointers not 16-byte
 * aligned, q not 8-byte aligned, or sf not 16-byte aligned (swizzled) / 4-byte
 * aligned (linear); QZ_ERR_CUDA on launch failure.  T == 0 launches nothing. */
qz_status qz_rmsnorm_quantize(const void *d_x, const void *d_residual, const void *d_gamma, float eps,
                              int64_t T, int64_t H, void *d_norm_out, void *d_residual_out,
                              int fmt, void *d_q, uint8_t *d_sf, int layout,
                              const float *d_global_amax, void *stream);

/* Largest number of rank inputs, and of destinations, of
 * qz_allreduce_rmsnorm_quantize (one tensor-parallel group of an NVLink node). */
#define QZ_MAX_RANKS 8

/* One destination of the AllReduce epilogue's outputs.  Device pointers: this
 * GPU's memory or a peer GPU's buffer mapped into this process. */
typedef struct qz_norm_dest {
    void *norm_out;     /* bf16 [T, H], 16-byte aligned */
    void *residual_out; /* bf16 [T, H], 16-byte aligned, or NULL (not written) */
    void *q;            /* e4m3 [T, H] (MXFP8) or packed e2m1 [T, H/2] (NVFP4), 8-byte aligned */
    uint8_t *sf;        /* SF region of T rows: qz_sf_bytes(T, H, fmt, layout) bytes, aligned as in
                           qz_rmsnorm_quantize */
} qz_norm_dest;

/* The fused epilogue behind a tensor-parallel AllReduce ([LSF] commits 2, 3 and
 * [CAR] commit 6: the AllReduce that ends an attention or MoE block already
 * holds the sum the norm reads, and emits the quantized norm from the same
 * pass).  For the rows [row_begin, row_end):
 *   x = bf16(sum over ranks of rank_x[r]), summed in binary32 in rank order
 *       0 .. n_ranks-1 (rank 0 exact, one rounding per further rank) and
 *       rounded once to bf16 (nearest-even), so every rank obtains the same bits
 *   then exactly qz_rmsnorm_quantize on x: h = bf16(x + residual), y, q, sf,
 * and every output row is written to each of the n_dests destinations.  One
 * call with rows [0, T) and this GPU's buffers as its single destination is the
 * one-shot form; a call per rank on its own slice with every rank's buffers as
 * destinations is the reduce-scatter + all-gather form.  The slice with
 * row_end == T also zeroes the swizzled layout's invented rows T .. pad(T,128)-1
 * of every destination.
 *   rank_x : HOST array of n_ranks device pointers, each to bf16 [T, H]
 *            (16-byte aligned; this GPU's memory or a peer mapping)
 *   dests  : HOST array of n_dests destinations
 * Both host arrays are read during the call only.  The kernel reads the ranks'
 * inputs with plain loads and writes the destinations with plain stores; it
 * never waits on another GPU.  The caller orders the exchange: every rank's
 * input is complete, and every destination free to be written, before this
 * call starts on the stream (a cross-rank barrier), and no rank overwrites its
 * input or reads a peer-written destination until every rank's call has
 * finished (a second barrier).
 * Errors: as qz_rmsnorm_quantize, plus QZ_ERR_INVALID_ARG for n_ranks or
 * n_dests outside 1 .. QZ_MAX_RANKS, NULL arrays or entries, and a row range
 * outside 0 <= row_begin <= row_end <= T; QZ_ERR_ALIGNMENT for any misaligned
 * entry.  An empty range launches nothing unless it must zero invented rows. */
qz_status qz_allreduce_rmsnorm_quantize(const void *const *rank_x, int n_ranks, const void *d_residual,
                                        const void *d_gamma, float eps, int64_t T, int64_t H,
                                        int64_t row_begin, int64_t row_end,
                                        const qz_norm_dest *dests, int n_dests, int fmt, int layout,
                                        const float *d_global_amax, void *stream);

/* Peer mappings for the AllReduce epilogue on a node: every rank exports a
 * CUDA IPC handle of its own buffer, the handles are exchanged over the
 * process group, and every rank imports its peers' buffers, so that one
 * process holds device pointers to all ranks' inputs and destinations
 * ([LSF] commits 1-2: the epilogue reads every rank's partial and writes the
 * result to every rank).  Host-side calls; no stream work, no allocation. */
typedef struct qz_ipc_handle {
    unsigned char handle[64]; /* cudaIpcMemHandle_t of the device allocation holding the pointer */
    uint64_t offset;          /* pointer - start of that allocation */
    uint64_t alloc_bytes;     /* bytes of that allocation */
    int device;               /* the exporting process's device ordinal */
    int reserved;
} qz_ipc_handle;

/* Fill *out for the device pointer d_ptr of the calling process (an address
 * inside a cudaMalloc allocation, on the current device).
 * Errors: QZ_ERR_INVALID_ARG for NULL arguments; QZ_ERR_CUDA when the runtime
 * or driver refuses (no device, not a device allocation, IPC unsupported). */
qz_status qz_ipc_export(const void *d_ptr, qz_ipc_handle *out);

/* Map a peer process's exported allocation into this process (current device;
 * peer access is enabled as needed) and return the peer's pointer in
 * *d_ptr_out (mapping base + offset).  A handle exported by the calling process
 * itself cannot be imported (CUDA IPC): use the pointer directly.
 * Errors: QZ_ERR_INVALID_ARG for NULL arguments; QZ_ERR_CUDA from the runtime. */
qz_status qz_ipc_import(const qz_ipc_handle *h, void **d_ptr_out);

/* Unmap a pointer returned by qz_ipc_import for the same handle.
 * Errors: QZ_ERR_INVALID_ARG for NULL arguments; QZ_ERR_CUDA from the runtime. */
qz_status qz_ipc_close(void *d_ptr, const qz_ipc_handle *h);

/* Linear -> swizzled 128x4 conversion of n SF matrices in one launch, padding
 * written as 0x00 ([MX] Summary; [CAR] commit 5: swizzled and linear agree).
 * Errors: QZ_ERR_INVALID_ARG for n < 0, n > QZ_MAX_EXPERTS or a NULL table
 * with n > 0; entries with rows < 0, kv < 1, null pointers or a misaligned
 * dst are skipped and reported through opts->d_err. */
qz_status qz_swizzle_scales(const qz_sf_pair *d_table, int n, void *stream, const qz_launch_opts *opts);

/* Decode grouped MXFP8 / NVFP4 tensors back to bf16: the inverse map of the
 * quantizers, for reference paths and error checks (TransformerEngine PR #3800,
 * Changes: regression tests on dequantized values; TensorRT-LLM "MXFP8 carrier
 * and quantize folds", commit 1: the dequant reference path).  Element i of
 * block k decodes to
 *   MXFP8: value(q_i) * 2^(sf_k - 127)
 *   NVFP4: value(q_i) * value(sf_k) * g,  g = RN32(A / 2688)
 * (A = amax[0], or amax[row] when per_row != 0) computed exactly and rounded
 * once to bf16, to nearest with ties to even.  fmt is QZ_FMT_MXFP8 or
 * QZ_FMT_NVFP4, layout the SF layout of every entry.  One persistent launch,
 * asynchronous on the stream, no allocation.
 * Errors: QZ_ERR_INVALID_ARG for n < 0, n > QZ_MAX_EXPERTS, a NULL table with
 * n > 0, an unknown fmt or layout; invalid entries are skipped and reported
 * through opts->d_err (QZ_DERR_SHAPE / NULL / ALIGN with the alignments above). */
qz_status qz_dequantize_grouped(const qz_dq_expert *d_table, int n_experts, int fmt, int per_row, int layout,
                                void *stream, const qz_launch_opts *opts);

/* Column-wise (transposed) grouped quantization: the blocks run down the
 * columns of each expert's x [rows, cols], i.e. x^T is quantized row-wise
 * (TransformerEngine PR #3800, Changes: its fast path is "rowwise-only"; the
 * column-wise form is the weight-gradient GEMM's operand).  Per expert:
 *   q:  MXFP8 e4m3 [cols, rows] (16-byte aligned), NVFP4 packed e2m1
 *       [cols, rows/2] (8-byte aligned), dense rows
 *   sf: the SF region of a [cols, rows] matrix, qz_sf_bytes(cols, rows, fmt,
 *       layout) bytes, padding written as 0x00
 *   amax: NVFP4 only, the tensor amax, given (the row-wise
 *       QZ_NVFP4_PER_TENSOR_COMPUTE call of the same tensor writes it)
 * rows must be a multiple of 32 (MXFP8) / 16 (NVFP4); cols any positive
 * number; x as for the row-wise calls.  Results equal the row-wise call on
 * the transposed tensor byte for byte.  One persistent launch, no allocation.
 * Errors: as qz_quantize_grouped_mxfp8, plus QZ_ERR_INVALID_ARG for an
 * unknown fmt; invalid entries are skipped and reported through opts->d_err. */
qz_status qz_quantize_grouped_colwise(const qz_expert *d_table, int n_experts, int fmt, int layout, void *stream,
                                      const qz_launch_opts *opts);

/* Attention decode merge that also writes its MXFP8 form (TensorRT-LLM "MXFP8
 * carrier and quantize folds", commit 3: the kernel finishing flash-decoding
 * writes the attention output and its MXFP8 form, and zeroes the SF rows the
 * swizzled layout invents past the last live row, so no memset is needed).
 * A producer kernel built on include/qz_quant.cuh.
 *   d_partial: float [S, T, H], the S partial outputs of each token
 *   d_lse:     float [S, T], their natural-log sum-exps
 *   d_out:     bf16 [T, H], y[t] = sum_s w_s O[s, t] / sum_s w_s,
 *              w_s = exp(lse[s, t] - max_s lse[s, t]), rounded to nearest even
 *   d_q, d_sf: e4m3 [T, H] and the SF region (qz_sf_bytes(T, H, QZ_FMT_MXFP8,
 *              layout) bytes) of y quantized exactly as qz_quantize_grouped_mxfp8
 *              would; d_q == NULL skips the MXFP8 form (d_sf is then ignored)
 * The merge accumulates in binary64 and rounds once to bf16.
 * 1 <= S <= QZ_MAX_SPLITS, T >= 0, H a multiple of 32 up to QZ_MAX_HIDDEN.
 * One launch, asynchronous on the stream, no allocation.
 * Errors (before any launch): QZ_ERR_INVALID_ARG for a bad S, T < 0, a bad H,
 * an unknown layout or a NULL pointer that is needed; QZ_ERR_ALIGNMENT for
 * d_partial / d_out not 16-byte aligned, d_q not 8-byte aligned or a
 * swizzled d_sf not 16-byte aligned; QZ_ERR_UNSUPPORTED for a swizzled
 * layout with H / 32 not a multiple of 4 (the kernel writes no padded
 * scale columns). */
#define QZ_MAX_SPLITS 4096
qz_status qz_attention_merge_quantize(const float *d_partial, const float *d_lse, int S, int64_t T, int64_t H,
                                      void *d_out, void *d_q, uint8_t *d_sf, int layout, void *stream);

/* Gate|up split of folded fused experts (Model-Optimizer "Fold fused experts'
 * quantizers into their weights shard-locally": a fused expert's (2I, H)
 * weight is quantized as one tensor, gate and up sharing its per-tensor amax
 * and so one weight_scale_2; the split then cuts the folded payload and its
 * stacked scales by rows into gate and up, each in storage of its own, cuts a
 * scale in proportion to the rows it covers and refuses a block scale that
 * the cut would divide).  Per entry and part p (rows [first_p, first_p + n_p)):
 *   payload: rows copied to q_out[p] (skipped when q_out[p] is NULL);
 *   MXFP8 / NVFP4 scales: one scale row per weight row, so every cut is
 *     exact; the part's SF region is written in dst_layout with its own
 *     padding (0x00) from the source region in src_layout -- a swizzled
 *     source cut inside a 128-row tile is re-laid, not refused;
 *   FP8_BLOCK128 scales: whole scale rows copied; a cut that is not a
 *     multiple of 128 and not the end divides a block: the entry is refused
 *     (skipped, QZ_DERR_CUT);
 *   amax: QZ_AMAX_PER_TENSOR gives amax[0] to both parts (one
 *     weight_scale_2), QZ_AMAX_PER_ROW cuts it with the rows.
 * Results equal quantizing each part's rows on their own (with the shared
 * amax for a per-tensor scale).  One persistent launch, no allocation.
 * Errors (before any launch): QZ_ERR_INVALID_ARG for n < 0 or > QZ_MAX_EXPERTS,
 * a NULL table with n > 0, an unknown fmt, amax_kind or layout, an amax kind
 * the format does not have (MXFP8 and FP8_BLOCK128 take QZ_AMAX_NONE only);
 * QZ_ERR_UNSUPPORTED for FP8_BLOCK128 with a swizzled layout.  Invalid
 * entries are skipped and reported through opts->d_err (QZ_DERR_SHAPE for
 * bad sizes or a cut outside [0, rows], QZ_DERR_NULL, QZ_DERR_ALIGN,
 * QZ_DERR_CUT). */
qz_status qz_split_fused_experts(const qz_fused_split *d_table, int n, int fmt, int amax_kind, int src_layout,
                                 int dst_layout, void *stream, const qz_launch_opts *opts);

/* Largest table of qz_quantize_grouped_nvfp4_compute_noalloc. */
#define QZ_STATIC_WS_MAX_EXPERTS 1024

/* Allocation-free NVFP4 quantization with a computed per-tensor amax: the
 * same single cooperative launch as qz_quantize_grouped_nvfp4 in
 * QZ_NVFP4_PER_TENSOR_COMPUTE mode with opts->d_workspace, but its scratch
 * (an abort word, per-expert unit counters and amax words, about 21 KB)
 * is a device array inside the library, so the caller passes only the table,
 * inputs and outputs.  The source pages have no counterpart of this entry
 * point; it exists for callers that cannot allocate device memory themselves,
 * such as code embedded in a framework that owns every device allocation, or
 * a latency-critical loop in which a cudaMalloc would synchronize the device.
 *  - The array is allocated with the library image: every GPU on which the
 *    library is loaded keeps it until the process exits.  The library calls
 *    no cudaMalloc, cudaFree or other allocating routine here.
 *  - The first call on a device looks up the array's device address (a
 *    one-time set-up per device); make that first call before any stream
 *    capture.
 *  - Every call clears the scratch it needs (a memset in stream order) and
 *    leaves its own contents behind; all calls share the one array, so calls
 *    that may overlap on the GPU (other streams, other host threads) race and
 *    must be serialized by the caller.  A race shows up as QZ_DERR_TIMEOUT in
 *    *opts->d_err or as wrong amax, scale or payload bytes.
 *  - The looked-up address is kept for the life of the process: after
 *    cudaDeviceReset on a device, this entry point must not be called again
 *    on that device (the array may have moved with the reloaded library image).
 *  - n_experts above QZ_STATIC_WS_MAX_EXPERTS returns QZ_ERR_INVALID_ARG
 *    before anything is launched; other errors as qz_quantize_grouped_nvfp4;
 *    opts->d_workspace is ignored. */
qz_status qz_quantize_grouped_nvfp4_compute_noalloc(const qz_expert *d_table, int n_experts, int layout,
                                                    void *stream, const qz_launch_opts *opts);

/* A static, human-readable name for a status code. */
const char *qz_status_string(qz_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
int qz_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QZ_H */
