"""ctypes binding of libqz.so -- argument marshalling only.

Every byte of quantization work happens in the CUDA kernels behind the C ABI
(include/qz.h).  This module packs expert tables into device memory, passes
pointers, sizes and the current CUDA stream, and turns status codes into
exceptions.  There is no fallback: if libqz.so is missing or a call fails, it
raises.  PyTorch supplies device memory and streams.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass
from typing import Iterable, Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqz.so")

# enums of include/qz.h
QZ_OK, QZ_ERR_INVALID_ARG, QZ_ERR_ALIGNMENT, QZ_ERR_UNSUPPORTED, QZ_ERR_CUDA = range(5)
SF_LINEAR, SF_SWIZZLED = 0, 1
FMT_MXFP8, FMT_NVFP4, FMT_FP8_BLOCK128 = 0, 1, 2
NVFP4_PER_TENSOR_GIVEN, NVFP4_PER_TENSOR_COMPUTE, NVFP4_PER_ROW = 0, 1, 2
AMAX_NONE, AMAX_PER_TENSOR, AMAX_PER_ROW = 0, 1, 2
DERR_SHAPE, DERR_NULL, DERR_ALIGN, DERR_TOO_LARGE = 0x1, 0x2, 0x4, 0x8
DERR_TIMEOUT, DERR_CUT = 0x10, 0x20
TEST_WITHHOLD_ARRIVALS = 0x1
OPT_INDEPENDENT = 0x1
MAX_EXPERTS = 4096
MAX_HIDDEN = 16384
MAX_RANKS = 8

EXPORTED = (
    "qz_sf_bytes",
    "qz_quantize_grouped_mxfp8",
    "qz_quantize_grouped_nvfp4",
    "qz_rmsnorm_quantize",
    "qz_swizzle_scales",
    "qz_status_string",
    "qz_version",
    "qz_workspace_bytes",
    "qz_quantize_grouped_nvfp4_compute_noalloc",
    "qz_dequantize_grouped",
    "qz_attention_merge_quantize",
    "qz_quantize_grouped_colwise",
    "qz_split_fused_experts",
    "qz_allreduce_rmsnorm_quantize",
    "qz_ipc_export",
    "qz_ipc_import",
    "qz_ipc_close",
)
STATIC_WS_MAX_EXPERTS = 1024


class QzError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class _Expert(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("ld", ctypes.c_int64), ("q", ctypes.c_void_p), ("sf", ctypes.c_void_p),
                ("amax", ctypes.c_void_p)]


class _DqExpert(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("sf", ctypes.c_void_p), ("amax", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("y", ctypes.c_void_p),
                ("ldy", ctypes.c_int64)]


class _SfPair(ctypes.Structure):
    _fields_ = [("src", ctypes.c_void_p), ("dst", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("kv", ctypes.c_int64)]


class _FusedSplit(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("sf", ctypes.c_void_p), ("amax", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("cut", ctypes.c_int64),
                ("q_out", ctypes.c_void_p * 2), ("sf_out", ctypes.c_void_p * 2), ("amax_out", ctypes.c_void_p * 2)]


class IpcHandle(ctypes.Structure):
    """struct qz_ipc_handle: a CUDA IPC handle of an allocation and the offset
    of the exported pointer in it."""
    _fields_ = [("handle", ctypes.c_ubyte * 64), ("offset", ctypes.c_uint64), ("alloc_bytes", ctypes.c_uint64),
                ("device", ctypes.c_int), ("reserved", ctypes.c_int)]


class _Opts(ctypes.Structure):
    _fields_ = [("d_err", ctypes.c_void_p), ("max_ctas", ctypes.c_int), ("d_workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t), ("elems_hint", ctypes.c_int64),
                ("wait_limit_ns", ctypes.c_int64), ("test_flags", ctypes.c_uint), ("launch_flags", ctypes.c_uint)]


assert ctypes.sizeof(_Expert) == 56 and ctypes.sizeof(_SfPair) == 32 and ctypes.sizeof(_DqExpert) == 56
assert ctypes.sizeof(_FusedSplit) == 96 and ctypes.sizeof(IpcHandle) == 88

_lock = threading.Lock()
_lib = None


def load(path: str = LIB_PATH):
    """Load libqz.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m nvfp4_quantization_moe_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(path)
        P, I, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        lib.qz_sf_bytes.restype = ctypes.c_size_t
        lib.qz_sf_bytes.argtypes = [i64, i64, I, I]
        lib.qz_quantize_grouped_mxfp8.restype = I
        lib.qz_quantize_grouped_mxfp8.argtypes = [P, I, I, P, P]
        lib.qz_quantize_grouped_nvfp4.restype = I
        lib.qz_quantize_grouped_nvfp4.argtypes = [P, I, I, I, P, P]
        lib.qz_rmsnorm_quantize.restype = I
        lib.qz_rmsnorm_quantize.argtypes = [P, P, P, ctypes.c_float, i64, i64, P, P, I, P, P, I, P, P]
        lib.qz_swizzle_scales.restype = I
        lib.qz_swizzle_scales.argtypes = [P, I, P, P]
        lib.qz_status_string.restype = ctypes.c_char_p
        lib.qz_status_string.argtypes = [I]
        lib.qz_version.restype = I
        lib.qz_version.argtypes = []
        lib.qz_workspace_bytes.restype = ctypes.c_size_t
        lib.qz_workspace_bytes.argtypes = [I]
        lib.qz_quantize_grouped_nvfp4_compute_noalloc.restype = I
        lib.qz_quantize_grouped_nvfp4_compute_noalloc.argtypes = [P, I, I, P, P]
        lib.qz_dequantize_grouped.restype = I
        lib.qz_dequantize_grouped.argtypes = [P, I, I, I, I, P, P]
        lib.qz_quantize_grouped_colwise.restype = I
        lib.qz_quantize_grouped_colwise.argtypes = [P, I, I, I, P, P]
        lib.qz_attention_merge_quantize.restype = I
        lib.qz_attention_merge_quantize.argtypes = [P, P, I, i64, i64, P, P, P, I, P]
        lib.qz_split_fused_experts.restype = I
        lib.qz_split_fused_experts.argtypes = [P, I, I, I, I, I, P, P]
        lib.qz_ipc_export.restype = I
        lib.qz_ipc_export.argtypes = [P, P]
        lib.qz_ipc_import.restype = I
        lib.qz_ipc_import.argtypes = [P, P]
        lib.qz_ipc_close.restype = I
        lib.qz_ipc_close.argtypes = [P, P]
        lib.qz_allreduce_rmsnorm_quantize.restype = I
        lib.qz_allreduce_rmsnorm_quantize.argtypes = [P, I, P, P, ctypes.c_float, i64, i64, i64, i64, P, I, I, I,
                                                      P, P]
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return load().qz_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != QZ_OK:
        raise QzError(status, where)


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream))


def _opts(err: Optional[torch.Tensor], max_ctas: int, workspace: Optional[torch.Tensor] = None, elems_hint: int = 0,
          wait_limit_ns: int = 0, test_flags: int = 0, launch_flags: int = 0):
    if (err is None and not max_ctas and workspace is None and not elems_hint and not wait_limit_ns and not test_flags
            and not launch_flags):
        return None
    if err is not None:
        assert err.dtype in (torch.int32, torch.uint32) and err.is_cuda and err.numel() >= 1
    ws_ptr = workspace.data_ptr() if workspace is not None else 0
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return ctypes.byref(_Opts(ctypes.c_void_p(err.data_ptr() if err is not None else 0), int(max_ctas),
                              ctypes.c_void_p(ws_ptr), ctypes.c_size_t(ws_bytes), ctypes.c_int64(int(elems_hint)),
                              ctypes.c_int64(int(wait_limit_ns)), ctypes.c_uint(int(test_flags)),
                              ctypes.c_uint(int(launch_flags))))


def workspace_bytes(n_experts: int) -> int:
    """Device scratch for the single-launch computed-amax NVFP4 path."""
    return int(load().qz_workspace_bytes(int(n_experts)))


def alloc_workspace(n_experts: int, device=None) -> torch.Tensor:
    return torch.empty(max(workspace_bytes(n_experts), 4), dtype=torch.uint8,
                       device=device if device is not None else "cuda")


def _ptr(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else int(t.data_ptr())


def sf_bytes(rows: int, cols: int, fmt: int, layout: int) -> int:
    return int(load().qz_sf_bytes(int(rows), int(cols), int(fmt), int(layout)))


# ---------------------------------------------------------------------------
# device tables
# ---------------------------------------------------------------------------

@dataclass
class Entry:
    """One expert: a bf16 [rows, cols] view (row stride in elements may exceed
    cols), its payload, SF region and (NVFP4) amax storage."""
    x: torch.Tensor
    q: torch.Tensor
    sf: torch.Tensor
    amax: Optional[torch.Tensor] = None


class ExpertTable:
    """A device-resident array of qz_expert entries.  Keeps references to the
    tensors it points into, so they outlive the table."""

    def __init__(self, entries: Sequence[Entry], device=None):
        self.entries = list(entries)
        n = len(self.entries)
        arr = (_Expert * max(n, 1))()
        for i, e in enumerate(self.entries):
            x = e.x
            assert x.dtype == torch.bfloat16 and x.dim() == 2
            rows, cols = x.shape
            ld = x.stride(0) if rows > 1 else max(cols, x.stride(0))
            assert rows == 0 or x.stride(1) == 1, "rows must be contiguous"
            arr[i] = _Expert(x.data_ptr() if rows else 0, rows, cols, ld, _ptr(e.q) if rows else 0,
                             _ptr(e.sf) if rows else 0, _ptr(e.amax))
        host = torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8)
        dev = device if device is not None else (self.entries[0].x.device if n else torch.device("cuda"))
        self.dev = host.to(dev)
        self.n = n
        self.elems = sum(int(e.x.shape[0]) * int(e.x.shape[1]) for e in self.entries)

    @property
    def ptr(self) -> int:
        return int(self.dev.data_ptr()) if self.n else 0

    @classmethod
    def from_raw(cls, raw: Iterable[tuple], device) -> "ExpertTable":
        """Entries from raw (x_ptr, rows, cols, ld, q_ptr, sf_ptr, amax_ptr) tuples
        (tests use this to build deliberately invalid entries)."""
        self = cls.__new__(cls)
        raw = list(raw)
        arr = (_Expert * max(len(raw), 1))(*[_Expert(*r) for r in raw])
        self.entries = []
        self.n = len(raw)
        self.elems = 0
        self.dev = torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8).to(device)
        return self


@dataclass
class DqEntry:
    """One quantized expert to decode: payload q ([rows, cols] e4m3 or
    [rows, cols/2] packed e2m1), its SF region, its amax (NVFP4) and the bf16
    output y [rows, cols] (row stride may exceed cols)."""
    q: torch.Tensor
    sf: torch.Tensor
    y: torch.Tensor
    amax: Optional[torch.Tensor] = None


class DqTable:
    """A device-resident array of qz_dq_expert entries (keeps its tensors alive)."""

    def __init__(self, entries: Sequence[DqEntry], device=None):
        self.entries = list(entries)
        n = len(self.entries)
        arr = (_DqExpert * max(n, 1))()
        for i, e in enumerate(self.entries):
            y = e.y
            assert y.dtype == torch.bfloat16 and y.dim() == 2
            rows, cols = y.shape
            ldy = y.stride(0) if rows > 1 else max(cols, y.stride(0))
            assert rows == 0 or y.stride(1) == 1, "rows must be contiguous"
            arr[i] = _DqExpert(_ptr(e.q) if rows else 0, _ptr(e.sf) if rows else 0, _ptr(e.amax), rows, cols,
                               y.data_ptr() if rows else 0, ldy)
        host = torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8)
        dev = device if device is not None else (self.entries[0].y.device if n else torch.device("cuda"))
        self.dev = host.to(dev)
        self.n = n
        self.elems = sum(int(e.y.shape[0]) * int(e.y.shape[1]) for e in self.entries)

    @property
    def ptr(self) -> int:
        return int(self.dev.data_ptr()) if self.n else 0

    @classmethod
    def from_raw(cls, raw: Iterable[tuple], device) -> "DqTable":
        """Entries from raw (q_ptr, sf_ptr, amax_ptr, rows, cols, y_ptr, ldy) tuples."""
        self = cls.__new__(cls)
        raw = list(raw)
        arr = (_DqExpert * max(len(raw), 1))(*[_DqExpert(*r) for r in raw])
        self.entries = []
        self.n = len(raw)
        self.elems = 0
        self.dev = torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8).to(device)
        return self


@dataclass
class SplitEntry:
    """One folded fused expert to cut at row ``cut``: its payload q (rows
    [rows, row_bytes]), scales sf, amax, and each part's outputs.  q_out[p] may
    be None (that part's payload is not copied)."""
    q: torch.Tensor
    sf: torch.Tensor
    rows: int
    cols: int
    cut: int
    sf_out: tuple
    q_out: tuple = (None, None)
    amax: Optional[torch.Tensor] = None
    amax_out: tuple = (None, None)


class SplitTable:
    """A device-resident array of qz_fused_split entries (keeps its tensors alive)."""

    def __init__(self, entries: Sequence[SplitEntry], device=None):
        self.entries = list(entries)
        n = len(self.entries)
        arr = (_FusedSplit * max(n, 1))()
        P2 = ctypes.c_void_p * 2
        for i, e in enumerate(self.entries):
            arr[i] = _FusedSplit(_ptr(e.q), _ptr(e.sf), _ptr(e.amax), int(e.rows), int(e.cols), int(e.cut),
                                 P2(*[_ptr(t) for t in e.q_out]), P2(*[_ptr(t) for t in e.sf_out]),
                                 P2(*[_ptr(t) for t in e.amax_out]))
        host = torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8)
        dev = device if device is not None else (self.entries[0].q.device if n else torch.device("cuda"))
        self.dev = host.to(dev)
        self.n = n

    @property
    def ptr(self) -> int:
        return int(self.dev.data_ptr()) if self.n else 0

    @classmethod
    def from_raw(cls, raw: Iterable[tuple], device) -> "SplitTable":
        """Entries from raw (q, sf, amax, rows, cols, cut, (q0, q1), (sf0, sf1), (a0, a1)) tuples of
        integers (tests use this to build deliberately invalid entries)."""
        self = cls.__new__(cls)
        raw = list(raw)
        P2 = ctypes.c_void_p * 2
        arr = (_FusedSplit * max(len(raw), 1))(*[_FusedSplit(*r[:6], P2(*r[6]), P2(*r[7]), P2(*r[8])) for r in raw])
        self.entries = []
        self.n = len(raw)
        self.dev = torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8).to(device)
        return self


class SfPairTable:
    def __init__(self, pairs: Sequence[tuple], device):
        """pairs: (src linear uint8 tensor, dst swizzled uint8 tensor, rows, kv)."""
        self.pairs = list(pairs)
        arr = (_SfPair * max(len(self.pairs), 1))()
        for i, (src, dst, rows, kv) in enumerate(self.pairs):
            arr[i] = _SfPair(_ptr(src), _ptr(dst), int(rows), int(kv))
        self.dev = torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8).to(device)
        self.n = len(self.pairs)


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------

def quantize_grouped_mxfp8(table: ExpertTable, layout: int, stream=None, err=None, max_ctas: int = 0,
                           independent: bool = False):
    """MXFP8 over the table; the table's element count goes along as the
    grid-size hint.  ``independent`` sets QZ_OPT_INDEPENDENT (the call touches
    nothing that work still running on the stream touches)."""
    _check(load().qz_quantize_grouped_mxfp8(ctypes.c_void_p(table.ptr), table.n, int(layout),
                                            _stream_ptr(stream),
                                            _opts(err, max_ctas, elems_hint=getattr(table, "elems", 0),
                                                  launch_flags=OPT_INDEPENDENT if independent else 0)),
           "qz_quantize_grouped_mxfp8")


def quantize_grouped_nvfp4(table: ExpertTable, mode: int, layout: int, stream=None, err=None, max_ctas: int = 0,
                           workspace: Optional[torch.Tensor] = None, wait_limit_ns: int = 0, test_flags: int = 0,
                           independent: bool = False):
    _check(load().qz_quantize_grouped_nvfp4(ctypes.c_void_p(table.ptr), table.n, int(mode), int(layout),
                                            _stream_ptr(stream),
                                            _opts(err, max_ctas, workspace, wait_limit_ns=wait_limit_ns,
                                                  test_flags=test_flags,
                                                  launch_flags=OPT_INDEPENDENT if independent else 0)),
           "qz_quantize_grouped_nvfp4")


def quantize_grouped_nvfp4_compute_noalloc(table: ExpertTable, layout: int, stream=None, err=None, max_ctas: int = 0,
                                           wait_limit_ns: int = 0):
    """NVFP4 with computed per-tensor amax, scratch inside the library (no
    device allocation by anyone; see qz_quantize_grouped_nvfp4_compute_noalloc)."""
    _check(load().qz_quantize_grouped_nvfp4_compute_noalloc(ctypes.c_void_p(table.ptr), table.n, int(layout),
                                                            _stream_ptr(stream),
                                                            _opts(err, max_ctas, wait_limit_ns=wait_limit_ns)),
           "qz_quantize_grouped_nvfp4_compute_noalloc")


def rmsnorm_quantize(x, residual, gamma, eps: float, norm_out, residual_out, fmt: int, q, sf, layout: int,
                     global_amax=None, stream=None):
    T, H = x.shape
    _check(load().qz_rmsnorm_quantize(ctypes.c_void_p(_ptr(x)), ctypes.c_void_p(_ptr(residual)),
                                      ctypes.c_void_p(_ptr(gamma)), ctypes.c_float(eps), int(T), int(H),
                                      ctypes.c_void_p(_ptr(norm_out)), ctypes.c_void_p(_ptr(residual_out)),
                                      int(fmt), ctypes.c_void_p(_ptr(q)), ctypes.c_void_p(_ptr(sf)), int(layout),
                                      ctypes.c_void_p(_ptr(global_amax)), _stream_ptr(stream)),
           "qz_rmsnorm_quantize")


class NormDest(ctypes.Structure):
    """One destination of the AllReduce epilogue (struct qz_norm_dest)."""
    _fields_ = [("norm_out", ctypes.c_void_p), ("residual_out", ctypes.c_void_p), ("q", ctypes.c_void_p),
                ("sf", ctypes.c_void_p)]


def _addr(t) -> int:
    """A tensor's device address, or an address given as an int (a peer mapping)."""
    return int(t) if isinstance(t, int) else _ptr(t)


def allreduce_rmsnorm_quantize(rank_x, residual, gamma, eps: float, dests, fmt: int, layout: int, T: int, H: int,
                               rows=None, global_amax=None, stream=None):
    """AllReduce of the rank inputs + residual add + RMSNorm + quantize
    (qz_allreduce_rmsnorm_quantize).  ``rank_x``: bf16 [T, H] tensors or device
    addresses (peer mappings), summed in this order; ``dests``: tuples
    (norm_out, residual_out or None, q, sf) of tensors or addresses, each
    written with the rows ``rows`` = (row_begin, row_end), default all T.
    Every pointer argument takes a tensor, an int address or None."""
    row_begin, row_end = (0, T) if rows is None else rows
    xs = (ctypes.c_void_p * len(rank_x))(*[_addr(x) for x in rank_x])
    ds = (NormDest * len(dests))(*[NormDest(*[_addr(p) for p in d]) for d in dests])
    _check(load().qz_allreduce_rmsnorm_quantize(
        ctypes.cast(xs, ctypes.c_void_p), len(rank_x), ctypes.c_void_p(_addr(residual)),
        ctypes.c_void_p(_addr(gamma)), ctypes.c_float(eps), int(T), int(H), int(row_begin), int(row_end),
        ctypes.cast(ds, ctypes.c_void_p), len(dests), int(fmt), int(layout), ctypes.c_void_p(_addr(global_amax)),
        _stream_ptr(stream)),
        "qz_allreduce_rmsnorm_quantize")


def ipc_export(ptr: int) -> bytes:
    """qz_ipc_export: the IPC handle (88 bytes) of the device allocation holding ``ptr``."""
    h = IpcHandle()
    _check(load().qz_ipc_export(ctypes.c_void_p(int(ptr)), ctypes.byref(h)), "qz_ipc_export")
    return bytes(h)


def ipc_import(handle: bytes) -> int:
    """qz_ipc_import: map a peer process's exported allocation; returns the
    peer's pointer as an address in this process."""
    h = IpcHandle.from_buffer_copy(handle)
    out = ctypes.c_void_p()
    _check(load().qz_ipc_import(ctypes.byref(h), ctypes.byref(out)), "qz_ipc_import")
    return int(out.value)


def ipc_close(ptr: int, handle: bytes) -> None:
    """qz_ipc_close: unmap a pointer returned by ipc_import for ``handle``."""
    h = IpcHandle.from_buffer_copy(handle)
    _check(load().qz_ipc_close(ctypes.c_void_p(int(ptr)), ctypes.byref(h)), "qz_ipc_close")


def dequantize_grouped(table: DqTable, fmt: int, per_row: bool, layout: int, stream=None, err=None,
                       max_ctas: int = 0):
    _check(load().qz_dequantize_grouped(ctypes.c_void_p(table.ptr), table.n, int(fmt), 1 if per_row else 0,
                                        int(layout), _stream_ptr(stream),
                                        _opts(err, max_ctas, elems_hint=getattr(table, "elems", 0))),
           "qz_dequantize_grouped")


def quantize_grouped_colwise(table: ExpertTable, fmt: int, layout: int, stream=None, err=None, max_ctas: int = 0):
    """Column-wise quantization: each entry's q / sf receive x^T quantized
    row-wise (q [cols, rows] or [cols, rows/2]); NVFP4 uses the given amax."""
    _check(load().qz_quantize_grouped_colwise(ctypes.c_void_p(table.ptr), table.n, int(fmt), int(layout),
                                              _stream_ptr(stream), _opts(err, max_ctas)),
           "qz_quantize_grouped_colwise")


def attention_merge_quantize(partial, lse, out, q=None, sf=None, layout: int = SF_SWIZZLED, stream=None):
    """Merge float partial outputs [S, T, H] by their log-sum-exps [S, T] into
    bf16 out [T, H] and (q given) its MXFP8 form q [T, H] + SF region sf."""
    S, T, H = partial.shape
    _check(load().qz_attention_merge_quantize(ctypes.c_void_p(_ptr(partial)), ctypes.c_void_p(_ptr(lse)), int(S),
                                              int(T), int(H), ctypes.c_void_p(_ptr(out)), ctypes.c_void_p(_ptr(q)),
                                              ctypes.c_void_p(_ptr(sf)), int(layout), _stream_ptr(stream)),
           "qz_attention_merge_quantize")


def split_fused_experts(table: SplitTable, fmt: int, amax_kind: int, src_layout: int, dst_layout: int, stream=None,
                        err=None, max_ctas: int = 0):
    """Cut folded fused experts into gate (rows [0, cut)) and up (rows [cut, rows)):
    payload rows, scales re-laid per part in dst_layout, amax shared or cut."""
    _check(load().qz_split_fused_experts(ctypes.c_void_p(table.ptr), table.n, int(fmt), int(amax_kind),
                                         int(src_layout), int(dst_layout), _stream_ptr(stream), _opts(err, max_ctas)),
           "qz_split_fused_experts")


def swizzle_scales(table: SfPairTable, stream=None, err=None, max_ctas: int = 0):
    _check(load().qz_swizzle_scales(ctypes.c_void_p(int(table.dev.data_ptr()) if table.n else 0), table.n,
                                    _stream_ptr(stream), _opts(err, max_ctas)),
           "qz_swizzle_scales")


# ---------------------------------------------------------------------------
# conveniences that allocate outputs with torch and call the entry points
# ---------------------------------------------------------------------------

def alloc_outputs(xs: Sequence[torch.Tensor], fmt: int, layout: int, mode: int = NVFP4_PER_ROW):
    """Payload, SF and amax buffers for a list of bf16 [rows, cols] experts."""
    entries = []
    for x in xs:
        rows, cols = x.shape
        qcols = cols if fmt == FMT_MXFP8 else cols // 2
        q = torch.empty((rows, qcols), dtype=torch.uint8, device=x.device)
        sf = torch.empty(max(sf_bytes(rows, cols, fmt, layout), 16), dtype=torch.uint8, device=x.device)
        amax = None
        if fmt == FMT_NVFP4:
            amax = torch.zeros(max(rows, 1) if mode == NVFP4_PER_ROW else 1, dtype=torch.float32, device=x.device)
        entries.append(Entry(x, q, sf, amax))
    return entries


def quantize_experts(xs: Sequence[torch.Tensor], fmt: int, layout: int, mode: int = NVFP4_PER_ROW,
                     amax_in: Optional[Sequence[float]] = None, stream=None, workspace: Optional[torch.Tensor] = None):
    """Quantize a list of bf16 experts in one launch; returns the entries with
    q, sf (trimmed to the region size) and amax filled."""
    entries = alloc_outputs(xs, fmt, layout, mode)
    if fmt == FMT_NVFP4 and mode == NVFP4_PER_TENSOR_GIVEN:
        for e, a in zip(entries, amax_in):
            e.amax.fill_(float(a))
    table = ExpertTable(entries)
    if fmt == FMT_MXFP8:
        quantize_grouped_mxfp8(table, layout, stream)
    else:
        quantize_grouped_nvfp4(table, mode, layout, stream, workspace=workspace)
    for e in entries:
        rows, cols = e.x.shape
        e.sf = e.sf[: sf_bytes(rows, cols, fmt, layout)]
    return entries
