"""Grouped block-scaled (MXFP8 / NVFP4) quantization of MoE expert tensors on
NVIDIA B200 (sm_100a).

The compute path is the C-ABI CUDA library ``libqz.so`` (declared in
``include/qz.h``); :mod:`.binding` marshals arguments to it through ctypes.
There is no CPU or library fallback: every call raises if the library is
missing or reports an error.
"""
from .binding import (  # noqa: F401
    AMAX_NONE, AMAX_PER_ROW, AMAX_PER_TENSOR, DERR_ALIGN, DERR_CUT, DERR_NULL, DERR_SHAPE, DERR_TIMEOUT,
    DERR_TOO_LARGE, EXPORTED, OPT_INDEPENDENT, TEST_WITHHOLD_ARRIVALS,
    FMT_FP8_BLOCK128, FMT_MXFP8, FMT_NVFP4, LIB_PATH, MAX_EXPERTS, MAX_HIDDEN, MAX_RANKS, NVFP4_PER_ROW,
    NVFP4_PER_TENSOR_COMPUTE, NVFP4_PER_TENSOR_GIVEN, QZ_ERR_ALIGNMENT, QZ_ERR_CUDA, QZ_ERR_INVALID_ARG,
    QZ_ERR_UNSUPPORTED, QZ_OK, SF_LINEAR, SF_SWIZZLED, STATIC_WS_MAX_EXPERTS, DqEntry, DqTable, Entry, ExpertTable,
    IpcHandle, NormDest, QzError, SfPairTable, SplitEntry, SplitTable, alloc_outputs, alloc_workspace,
    allreduce_rmsnorm_quantize, attention_merge_quantize,
    dequantize_grouped, ipc_close, ipc_export, ipc_import, load, quantize_experts, quantize_grouped_colwise, quantize_grouped_mxfp8,
    quantize_grouped_nvfp4, quantize_grouped_nvfp4_compute_noalloc, rmsnorm_quantize, sf_bytes,
    split_fused_experts, status_string, swizzle_scales, workspace_bytes,
)

__version__ = "0.1.0"
