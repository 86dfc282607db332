// qz_api.cu -- the extern "C" entry points declared in include/qz.h.
//
// Host side only: argument checks that need no device memory, grid sizing
// (one wave of resident CTAs on every SM, cached per device), and the
// launches.  Nothing here allocates, synchronizes or reads device memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstring>
#include <mutex>

#include "../../include/qz.h"

namespace qz {
cudaError_t launch_mxfp8(const qz_expert* table, int n, int layout, int grid, cudaStream_t s, unsigned* d_err,
                         bool independent);
cudaError_t launch_nvfp4_tensor(const qz_expert* table, int n, int layout, bool compute_amax, int grid,
                                cudaStream_t s, unsigned* d_err, bool independent);
cudaError_t launch_nvfp4_rows(const qz_expert* table, int n, int layout, int grid, cudaStream_t s, unsigned* d_err);
cudaError_t launch_swizzle(const qz_sf_pair* table, int n, int grid, cudaStream_t s, unsigned* d_err);
cudaError_t launch_rmsnorm_quant(const uint16_t* x, const uint16_t* r, const uint16_t* g, float eps, int64_t T,
                                 int64_t H, uint16_t* y, uint16_t* h, int fmt, uint8_t* q, uint8_t* sf, int layout,
                                 const float* amax, cudaStream_t s, bool latency_mode);
cudaError_t launch_allreduce_norm_quant(const uint16_t* const* xs, int n_x, const uint16_t* r, const uint16_t* g,
                                        float eps, int64_t T, int64_t H, int64_t row_begin, int64_t row_end,
                                        const qz_norm_dest* dsts, int n_dst, int fmt, int layout, const float* amax,
                                        cudaStream_t s, bool latency_mode);
int grouped_blocks_per_sm(int which, int n);
size_t workspace_bytes(int n);
cudaError_t launch_nvfp4_compute_l2(const qz_expert* table, int n, int layout, int grid, unsigned* ws,
                                    cudaStream_t s, unsigned* d_err, long long wait_ns, unsigned test_flags);
cudaError_t launch_nvfp4_compute_l2_static(const qz_expert* table, int n, int layout, int grid, cudaStream_t s,
                                           unsigned* d_err, long long wait_ns, unsigned test_flags);
int rows_blocks_per_sm(int n);
cudaError_t launch_dequant(const qz_dq_expert* table, int n, int fmt, bool per_row, int layout, int grid,
                           cudaStream_t s, unsigned* d_err);
int dequant_blocks_per_sm(int n, int fmt);
cudaError_t launch_colwise(const qz_expert* table, int n, int fmt, int layout, int grid, cudaStream_t s,
                           unsigned* d_err);
int colwise_blocks_per_sm(int n, int fmt);
cudaError_t launch_split_fused(const qz_fused_split* table, int n, int fmt, int amax_kind, int src_layout,
                               int dst_layout, int grid, cudaStream_t s, unsigned* d_err);
int split_blocks_per_sm(int n);
cudaError_t launch_attention_merge(const float* O, const float* lse, int S, int64_t T, int64_t H, uint16_t* y,
                                   uint8_t* q, uint8_t* sf, int layout, cudaStream_t s);
}  // namespace qz

namespace {

constexpr int kMaxDevices = 64;
constexpr int kKinds = 11;  // mxfp8, nvfp4 tile, swizzle, amax, rows, computed-amax L2 path, dequantize MXFP8,
                            // colwise MXFP8, fused split, dequantize NVFP4, colwise NVFP4

struct DeviceLimits {
    int sms = 0;
    int per_sm[kKinds] = {0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0};
};

std::mutex g_mu;
DeviceLimits g_dev[kMaxDevices];

// One wave of resident CTAs for kernel `kind` on the current device.  The
// occupancy is taken once per device with the largest prefix table, so the
// cached value never over-subscribes a smaller call.
int wave_grid(int kind, const qz_launch_opts* opts) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    int grid;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        DeviceLimits& d = g_dev[dev];
        if (d.sms == 0) {
            int sms = 0;
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            d.sms = sms > 0 ? sms : 1;
        }
        if (d.per_sm[kind] == 0)
            d.per_sm[kind] = (kind == 4)   ? qz::rows_blocks_per_sm(QZ_MAX_EXPERTS)
                             : (kind == 6) ? qz::dequant_blocks_per_sm(QZ_MAX_EXPERTS, QZ_FMT_MXFP8)
                             : (kind == 9) ? qz::dequant_blocks_per_sm(QZ_MAX_EXPERTS, QZ_FMT_NVFP4)
                             : (kind == 7) ? qz::colwise_blocks_per_sm(QZ_MAX_EXPERTS, QZ_FMT_MXFP8)
                             : (kind == 10) ? qz::colwise_blocks_per_sm(QZ_MAX_EXPERTS, QZ_FMT_NVFP4)
                             : (kind == 8) ? qz::split_blocks_per_sm(QZ_MAX_EXPERTS)
                                           : qz::grouped_blocks_per_sm(kind, QZ_MAX_EXPERTS);
        grid = d.sms * d.per_sm[kind];
    }
    if (opts && opts->max_ctas > 0 && opts->max_ctas < grid) grid = opts->max_ctas;
    return grid;
}

// SM count of the current device (cached).
int device_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceLimits& d = g_dev[dev];
    if (d.sms == 0) {
        int sms = 0;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        d.sms = sms > 0 ? sms : 1;
    }
    return d.sms;
}

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

unsigned* err_word(const qz_launch_opts* opts) { return opts ? opts->d_err : nullptr; }
long long wait_limit(const qz_launch_opts* opts) { return opts ? (long long)opts->wait_limit_ns : 0; }
unsigned test_flags(const qz_launch_opts* opts) { return opts ? opts->test_flags : 0u; }
bool independent(const qz_launch_opts* opts) { return opts && (opts->launch_flags & QZ_OPT_INDEPENDENT) != 0u; }

qz_status check_table(const void* table, int n) {
    if (n < 0 || n > QZ_MAX_EXPERTS) return QZ_ERR_INVALID_ARG;
    if (n > 0 && table == nullptr) return QZ_ERR_INVALID_ARG;
    return QZ_OK;
}

bool valid_layout(int layout) { return layout == QZ_SF_LINEAR || layout == QZ_SF_SWIZZLED_128x4; }

qz_status from_cuda(cudaError_t e) { return e == cudaSuccess ? QZ_OK : QZ_ERR_CUDA; }

// Grid of the MXFP8 tile kernels (quantize, dequantize): with an element
// count, about one CTA per kTilesPerCta tiles in whole waves (at most
// kMaxWaves), since the hardware's placement of many short CTAs streams a
// large call faster than one persistent wave (measured: 5.4 -> 6.6 TB/s on
// 128 experts of 3072 x 4096), and a call of fewer tiles than one wave
// launches one CTA per tile; a cap in opts->max_ctas still applies.  The
// NVFP4 kernels measured slower that way and keep one wave.
constexpr int64_t kTilesPerCta = 10;
constexpr int64_t kMaxWaves = 16;

int sized_grid(int kind, const qz_launch_opts* opts) {
    const int wave = wave_grid(kind, nullptr);
    int grid = wave;
    if (opts && opts->elems_hint > 0) {
        const int64_t tiles = (opts->elems_hint + 16383) / 16384;
        int64_t waves = (tiles + kTilesPerCta * wave / 2) / (kTilesPerCta * wave);  // rounded
        waves = waves < 1 ? 1 : (waves > kMaxWaves ? kMaxWaves : waves);
        grid = (int)(wave * waves);
        if (tiles < grid) grid = (int)tiles;  // a small call launches no idle CTAs
    }
    if (opts && opts->max_ctas > 0 && opts->max_ctas < grid) grid = opts->max_ctas;
    return grid;
}

}  // namespace

extern "C" {

size_t qz_sf_bytes(int64_t rows, int64_t cols, int fmt, int layout) {
    if (fmt == QZ_FMT_FP8_BLOCK128) {
        if (layout != QZ_SF_LINEAR || rows <= 0 || cols <= 0) return 0;
        return (size_t)(4 * ((rows + 127) / 128) * ((cols + 127) / 128));
    }
    if (fmt != QZ_FMT_MXFP8 && fmt != QZ_FMT_NVFP4) return 0;
    if (!valid_layout(layout)) return 0;
    const int64_t block = fmt == QZ_FMT_MXFP8 ? 32 : 16;
    if (rows <= 0 || cols <= 0 || cols % block != 0) return 0;
    const int64_t kv = cols / block;
    if (layout == QZ_SF_LINEAR) return (size_t)(rows * kv);
    return (size_t)(((rows + 127) / 128) * 128 * ((kv + 3) / 4) * 4);
}

qz_status qz_quantize_grouped_mxfp8(const qz_expert* d_table, int n_experts, int layout, void* stream,
                                    const qz_launch_opts* opts) {
    qz_status st = check_table(d_table, n_experts);
    if (st != QZ_OK) return st;
    if (!valid_layout(layout)) return QZ_ERR_INVALID_ARG;
    if (n_experts == 0) return QZ_OK;
    return from_cuda(qz::launch_mxfp8(d_table, n_experts, layout, sized_grid(0, opts), (cudaStream_t)stream,
                                      err_word(opts), independent(opts)));
}

qz_status qz_quantize_grouped_nvfp4(const qz_expert* d_table, int n_experts, int mode, int layout, void* stream,
                                    const qz_launch_opts* opts) {
    qz_status st = check_table(d_table, n_experts);
    if (st != QZ_OK) return st;
    if (!valid_layout(layout)) return QZ_ERR_INVALID_ARG;
    if (mode != QZ_NVFP4_PER_TENSOR_GIVEN && mode != QZ_NVFP4_PER_TENSOR_COMPUTE && mode != QZ_NVFP4_PER_ROW)
        return QZ_ERR_INVALID_ARG;
    if (opts && opts->wait_limit_ns < 0) return QZ_ERR_INVALID_ARG;
    if (mode == QZ_NVFP4_PER_TENSOR_COMPUTE && opts && opts->d_workspace) {
        if (n_experts > 0 && opts->workspace_bytes < qz::workspace_bytes(n_experts)) return QZ_ERR_INVALID_ARG;
        if (!aligned(opts->d_workspace, 4)) return QZ_ERR_ALIGNMENT;
    }
    if (n_experts == 0) return QZ_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if (mode == QZ_NVFP4_PER_TENSOR_COMPUTE && opts && opts->d_workspace)
        return from_cuda(qz::launch_nvfp4_compute_l2(d_table, n_experts, layout, wave_grid(5, opts),
                                                     static_cast<unsigned*>(opts->d_workspace), s, err_word(opts),
                                                     wait_limit(opts), test_flags(opts)));
    if (mode == QZ_NVFP4_PER_ROW)
        return from_cuda(qz::launch_nvfp4_rows(d_table, n_experts, layout, wave_grid(4, opts), s, err_word(opts)));
    return from_cuda(qz::launch_nvfp4_tensor(d_table, n_experts, layout, mode == QZ_NVFP4_PER_TENSOR_COMPUTE,
                                             wave_grid(1, opts), s, err_word(opts), independent(opts)));
}

qz_status qz_rmsnorm_quantize(const void* d_x, const void* d_residual, const void* d_gamma, float eps, int64_t T,
                              int64_t H, void* d_norm_out, void* d_residual_out, int fmt, void* d_q, uint8_t* d_sf,
                              int layout, const float* d_global_amax, void* stream) {
    if (fmt != QZ_FMT_MXFP8 && fmt != QZ_FMT_NVFP4) return QZ_ERR_INVALID_ARG;
    if (!valid_layout(layout)) return QZ_ERR_INVALID_ARG;
    const int64_t block = fmt == QZ_FMT_MXFP8 ? 32 : 16;
    if (T < 0 || H <= 0 || H > QZ_MAX_HIDDEN || H % block != 0) return QZ_ERR_INVALID_ARG;
    if (T > 0x7FFFFF00LL) return QZ_ERR_INVALID_ARG;
    if (layout == QZ_SF_SWIZZLED_128x4 && (H / block) % 4 != 0) return QZ_ERR_UNSUPPORTED;
    if (T == 0) return QZ_OK;
    if (!d_x || !d_residual || !d_gamma || !d_norm_out || !d_q || !d_sf) return QZ_ERR_INVALID_ARG;
    if (fmt == QZ_FMT_NVFP4 && !d_global_amax) return QZ_ERR_INVALID_ARG;
    if (!aligned(d_x, 16) || !aligned(d_residual, 16) || !aligned(d_gamma, 16) || !aligned(d_norm_out, 16) ||
        (d_residual_out && !aligned(d_residual_out, 16)))
        return QZ_ERR_ALIGNMENT;
    if (!aligned(d_q, 8) || !aligned(d_sf, layout == QZ_SF_SWIZZLED_128x4 ? 16 : 4)) return QZ_ERR_ALIGNMENT;
    if (d_global_amax && !aligned(d_global_amax, 4)) return QZ_ERR_ALIGNMENT;
    const bool latency_mode = T <= 2 * (int64_t)device_sms();
    return from_cuda(qz::launch_rmsnorm_quant(
        static_cast<const uint16_t*>(d_x), static_cast<const uint16_t*>(d_residual),
        static_cast<const uint16_t*>(d_gamma), eps, T, H, static_cast<uint16_t*>(d_norm_out),
        static_cast<uint16_t*>(d_residual_out), fmt, static_cast<uint8_t*>(d_q), d_sf, layout, d_global_amax,
        (cudaStream_t)stream, latency_mode));
}

qz_status qz_allreduce_rmsnorm_quantize(const void* const* rank_x, int n_ranks, const void* d_residual,
                                        const void* d_gamma, float eps, int64_t T, int64_t H, int64_t row_begin,
                                        int64_t row_end, const qz_norm_dest* dests, int n_dests, int fmt,
                                        int layout, const float* d_global_amax, void* stream) {
    if (fmt != QZ_FMT_MXFP8 && fmt != QZ_FMT_NVFP4) return QZ_ERR_INVALID_ARG;
    if (!valid_layout(layout)) return QZ_ERR_INVALID_ARG;
    if (n_ranks < 1 || n_ranks > QZ_MAX_RANKS || n_dests < 1 || n_dests > QZ_MAX_RANKS) return QZ_ERR_INVALID_ARG;
    if (!rank_x || !dests) return QZ_ERR_INVALID_ARG;
    const int64_t block = fmt == QZ_FMT_MXFP8 ? 32 : 16;
    if (T < 0 || H <= 0 || H > QZ_MAX_HIDDEN || H % block != 0) return QZ_ERR_INVALID_ARG;
    if (T > 0x7FFFFF00LL) return QZ_ERR_INVALID_ARG;
    if (row_begin < 0 || row_begin > row_end || row_end > T) return QZ_ERR_INVALID_ARG;
    if (layout == QZ_SF_SWIZZLED_128x4 && (H / block) % 4 != 0) return QZ_ERR_UNSUPPORTED;
    if (T == 0) return QZ_OK;
    if (!d_residual || !d_gamma || (fmt == QZ_FMT_NVFP4 && !d_global_amax)) return QZ_ERR_INVALID_ARG;
    for (int i = 0; i < n_ranks; ++i)
        if (!rank_x[i]) return QZ_ERR_INVALID_ARG;
    for (int d = 0; d < n_dests; ++d)
        if (!dests[d].norm_out || !dests[d].q || !dests[d].sf) return QZ_ERR_INVALID_ARG;
    if (!aligned(d_residual, 16) || !aligned(d_gamma, 16)) return QZ_ERR_ALIGNMENT;
    if (d_global_amax && !aligned(d_global_amax, 4)) return QZ_ERR_ALIGNMENT;
    for (int i = 0; i < n_ranks; ++i)
        if (!aligned(rank_x[i], 16)) return QZ_ERR_ALIGNMENT;
    for (int d = 0; d < n_dests; ++d) {
        const qz_norm_dest& o = dests[d];
        if (!aligned(o.norm_out, 16) || (o.residual_out && !aligned(o.residual_out, 16)) || !aligned(o.q, 8) ||
            !aligned(o.sf, layout == QZ_SF_SWIZZLED_128x4 ? 16 : 4))
            return QZ_ERR_ALIGNMENT;
    }
    const bool latency_mode = row_end - row_begin <= 2 * (int64_t)device_sms();
    return from_cuda(qz::launch_allreduce_norm_quant(
        reinterpret_cast<const uint16_t* const*>(rank_x), n_ranks, static_cast<const uint16_t*>(d_residual),
        static_cast<const uint16_t*>(d_gamma), eps, T, H, row_begin, row_end, dests, n_dests, fmt, layout,
        d_global_amax, (cudaStream_t)stream, latency_mode));
}

qz_status qz_swizzle_scales(const qz_sf_pair* d_table, int n, void* stream, const qz_launch_opts* opts) {
    qz_status st = check_table(d_table, n);
    if (st != QZ_OK) return st;
    if (n == 0) return QZ_OK;
    return from_cuda(qz::launch_swizzle(d_table, n, wave_grid(2, opts), (cudaStream_t)stream, err_word(opts)));
}

qz_status qz_quantize_grouped_nvfp4_compute_noalloc(const qz_expert* d_table, int n_experts, int layout,
                                                    void* stream, const qz_launch_opts* opts) {
    if (n_experts < 0 || n_experts > QZ_STATIC_WS_MAX_EXPERTS) return QZ_ERR_INVALID_ARG;
    if (n_experts > 0 && d_table == nullptr) return QZ_ERR_INVALID_ARG;
    if (opts && opts->wait_limit_ns < 0) return QZ_ERR_INVALID_ARG;
    if (!valid_layout(layout)) return QZ_ERR_INVALID_ARG;
    if (n_experts == 0) return QZ_OK;
    return from_cuda(qz::launch_nvfp4_compute_l2_static(d_table, n_experts, layout, wave_grid(5, opts),
                                                        (cudaStream_t)stream, err_word(opts), wait_limit(opts),
                                                        test_flags(opts)));
}

qz_status qz_dequantize_grouped(const qz_dq_expert* d_table, int n_experts, int fmt, int per_row, int layout,
                                void* stream, const qz_launch_opts* opts) {
    qz_status st = check_table(d_table, n_experts);
    if (st != QZ_OK) return st;
    if (!valid_layout(layout)) return QZ_ERR_INVALID_ARG;
    if (fmt != QZ_FMT_MXFP8 && fmt != QZ_FMT_NVFP4) return QZ_ERR_INVALID_ARG;
    if (n_experts == 0) return QZ_OK;
    return from_cuda(qz::launch_dequant(d_table, n_experts, fmt, per_row != 0, layout,
                                        fmt == QZ_FMT_MXFP8 ? sized_grid(6, opts) : wave_grid(9, opts),
                                        (cudaStream_t)stream, err_word(opts)));
}

qz_status qz_quantize_grouped_colwise(const qz_expert* d_table, int n_experts, int fmt, int layout, void* stream,
                                      const qz_launch_opts* opts) {
    qz_status st = check_table(d_table, n_experts);
    if (st != QZ_OK) return st;
    if (!valid_layout(layout)) return QZ_ERR_INVALID_ARG;
    if (fmt != QZ_FMT_MXFP8 && fmt != QZ_FMT_NVFP4) return QZ_ERR_INVALID_ARG;
    if (n_experts == 0) return QZ_OK;
    return from_cuda(qz::launch_colwise(d_table, n_experts, fmt, layout,
                                        wave_grid(fmt == QZ_FMT_MXFP8 ? 7 : 10, opts), (cudaStream_t)stream,
                                        err_word(opts)));
}

qz_status qz_attention_merge_quantize(const float* d_partial, const float* d_lse, int S, int64_t T, int64_t H,
                                      void* d_out, void* d_q, uint8_t* d_sf, int layout, void* stream) {
    if (S < 1 || S > QZ_MAX_SPLITS || T < 0 || T > 0x7FFFFFFFLL) return QZ_ERR_INVALID_ARG;
    if (H <= 0 || H % 32 != 0 || H > QZ_MAX_HIDDEN) return QZ_ERR_INVALID_ARG;
    if (!valid_layout(layout)) return QZ_ERR_INVALID_ARG;
    if (d_q && layout == QZ_SF_SWIZZLED_128x4 && (H / 32) % 4 != 0) return QZ_ERR_UNSUPPORTED;
    if (T == 0) return QZ_OK;
    if (!d_partial || !d_lse || !d_out || (d_q && !d_sf)) return QZ_ERR_INVALID_ARG;
    if (!aligned(d_partial, 16) || !aligned(d_out, 16)) return QZ_ERR_ALIGNMENT;
    if (d_q && (!aligned(d_q, 8) || (layout == QZ_SF_SWIZZLED_128x4 && !aligned(d_sf, 16)))) return QZ_ERR_ALIGNMENT;
    return from_cuda(qz::launch_attention_merge(d_partial, d_lse, S, T, H, static_cast<uint16_t*>(d_out),
                                                static_cast<uint8_t*>(d_q), d_sf, layout, (cudaStream_t)stream));
}

qz_status qz_split_fused_experts(const qz_fused_split* d_table, int n, int fmt, int amax_kind, int src_layout,
                                 int dst_layout, void* stream, const qz_launch_opts* opts) {
    qz_status st = check_table(d_table, n);
    if (st != QZ_OK) return st;
    if (fmt != QZ_FMT_MXFP8 && fmt != QZ_FMT_NVFP4 && fmt != QZ_FMT_FP8_BLOCK128) return QZ_ERR_INVALID_ARG;
    if (amax_kind != QZ_AMAX_NONE && amax_kind != QZ_AMAX_PER_TENSOR && amax_kind != QZ_AMAX_PER_ROW)
        return QZ_ERR_INVALID_ARG;
    if (fmt != QZ_FMT_NVFP4 && amax_kind != QZ_AMAX_NONE) return QZ_ERR_INVALID_ARG;
    if (!valid_layout(src_layout) || !valid_layout(dst_layout)) return QZ_ERR_INVALID_ARG;
    if (fmt == QZ_FMT_FP8_BLOCK128 && (src_layout != QZ_SF_LINEAR || dst_layout != QZ_SF_LINEAR))
        return QZ_ERR_UNSUPPORTED;
    if (n == 0) return QZ_OK;
    return from_cuda(qz::launch_split_fused(d_table, n, fmt, amax_kind, src_layout, dst_layout, wave_grid(8, opts),
                                            (cudaStream_t)stream, err_word(opts)));
}

qz_status qz_ipc_export(const void* d_ptr, qz_ipc_handle* out) {
    if (!d_ptr || !out) return QZ_ERR_INVALID_ARG;
    static_assert(sizeof(cudaIpcMemHandle_t) == sizeof(out->handle), "IPC handle size");
    // the allocation's start and size: the driver's address-range query,
    // reached through the runtime so the library needs no link to the driver
    typedef int (*AddressRange)(unsigned long long*, size_t*, unsigned long long);
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult found;
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &fn, 12000, cudaEnableDefault, &found) !=
            cudaSuccess ||
        found != cudaDriverEntryPointSuccess || !fn)
        return QZ_ERR_CUDA;
    unsigned long long base = 0;
    size_t size = 0;
    if (reinterpret_cast<AddressRange>(fn)(&base, &size, (unsigned long long)(uintptr_t)d_ptr) != 0) return QZ_ERR_CUDA;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) return QZ_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QZ_ERR_CUDA;
    memcpy(out->handle, &h, sizeof(h));
    out->offset = (uint64_t)((uintptr_t)d_ptr - base);
    out->alloc_bytes = (uint64_t)size;
    out->device = dev;
    out->reserved = 0;
    return QZ_OK;
}

qz_status qz_ipc_import(const qz_ipc_handle* h, void** d_ptr_out) {
    if (!h || !d_ptr_out) return QZ_ERR_INVALID_ARG;
    cudaIpcMemHandle_t ipc;
    memcpy(&ipc, h->handle, sizeof(ipc));
    void* base = nullptr;
    if (cudaIpcOpenMemHandle(&base, ipc, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return QZ_ERR_CUDA;
    *d_ptr_out = static_cast<char*>(base) + h->offset;
    return QZ_OK;
}

qz_status qz_ipc_close(void* d_ptr, const qz_ipc_handle* h) {
    if (!d_ptr || !h) return QZ_ERR_INVALID_ARG;
    return from_cuda(cudaIpcCloseMemHandle(static_cast<char*>(d_ptr) - h->offset));
}

size_t qz_workspace_bytes(int n_experts) {
    if (n_experts < 1 || n_experts > QZ_MAX_EXPERTS) return 0;
    return qz::workspace_bytes(n_experts);
}

const char* qz_status_string(qz_status status) {
    switch (status) {
        case QZ_OK: return "QZ_OK";
        case QZ_ERR_INVALID_ARG: return "QZ_ERR_INVALID_ARG: invalid argument";
        case QZ_ERR_ALIGNMENT: return "QZ_ERR_ALIGNMENT: misaligned pointer or stride";
        case QZ_ERR_UNSUPPORTED: return "QZ_ERR_UNSUPPORTED: unsupported shape/format/layout combination";
        case QZ_ERR_CUDA: return "QZ_ERR_CUDA: CUDA launch error";
    }
    return "unknown qz_status";
}

int qz_version(void) { return 100; }

}  // extern "C"
