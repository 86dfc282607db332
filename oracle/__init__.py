"""CPU oracle for grouped MXFP8 / NVFP4 quantization -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never calls it and
shares no code with it; a product path that reached this module would void the
parity claims it exists to check.

The arithmetic lives in ``qz_oracle.c`` (plain scalar C, one IEEE operation per
expression).  This module only compiles it with gcc, loads it with ctypes and
marshals numpy arrays; it adds no arithmetic of its own except the loop over
experts in the grouped helpers.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qz_oracle.c")
_LIB = os.path.join(_HERE, "libqz_oracle.so")
CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c11", "-fPIC", "-shared"]

_lock = threading.Lock()
_lib = None

MXFP8, NVFP4 = 0, 1
FP8_BLOCK128 = 2            # e4m3 payload with FP32 scales of 128 x 128 blocks (split only)
AMAX_NONE, AMAX_PER_TENSOR, AMAX_PER_ROW = 0, 1, 2
LINEAR, SWIZZLED = 0, 1
NVFP4_PER_TENSOR_GIVEN, NVFP4_PER_TENSOR_COMPUTE, NVFP4_PER_ROW = 0, 1, 2


def compile_library(src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle C source into a shared object (gcc)."""
    cmd = ["gcc", *CFLAGS, "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _stale() -> bool:
    return (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)


def _declare(lib):
    c = ctypes
    P = c.c_void_p
    i64 = c.c_int64
    sig = {
        "qzo_bf16_value": (c.c_float, [c.c_uint16]),
        "qzo_bf16_from_double": (c.c_uint16, [c.c_double]),
        "qzo_e4m3_value": (c.c_double, [c.c_uint8]),
        "qzo_e4m3_encode": (c.c_uint8, [c.c_float]),
        "qzo_e2m1_value": (c.c_double, [c.c_uint8]),
        "qzo_e2m1_encode": (c.c_uint8, [c.c_float]),
        "qzo_mx_scale_exponent": (c.c_int, [c.c_double]),
        "qzo_mx_reciprocal": (c.c_float, [c.c_int]),
        "qzo_sf_offset_linear": (i64, [i64, i64, i64]),
        "qzo_sf_offset_swizzled": (i64, [i64, i64, i64]),
        "qzo_sf_region_bytes": (i64, [i64, i64, c.c_int]),
        "qzo_swizzle": (None, [P, i64, i64, P]),
        "qzo_unswizzle": (None, [P, i64, i64, P]),
        "qzo_quantize_mxfp8": (None, [P, i64, i64, i64, P, P, c.c_int]),
        "qzo_quantize_nvfp4": (None, [P, i64, i64, i64, P, P, c.c_int, c.c_int, P]),
        "qzo_residual_rmsnorm": (None, [P, P, P, c.c_float, i64, i64, P, P]),
        "qzo_rmsnorm_quantize": (None, [P, P, P, c.c_float, i64, i64, P, P, c.c_int, P, P, c.c_int, P]),
        "qzo_rank_sum": (None, [P, c.c_int, i64, P]),
        "qzo_dequantize_mxfp8": (None, [P, P, i64, i64, c.c_int, P, i64]),
        "qzo_dequantize_nvfp4": (None, [P, P, P, c.c_int, i64, i64, c.c_int, P, i64]),
        "qzo_attention_merge": (None, [P, P, i64, i64, i64, P]),
        "qzo_split_fused": (c.c_int, [c.c_int, P, P, P, c.c_int, i64, i64, i64, c.c_int, c.c_int,
                                      P, P, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def load(path: str | None = None):
    """Load (compiling first if needed) the oracle library.

    ``path`` loads another build of the same source (the mutation tests use it).
    """
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            override = os.environ.get("QZ_ORACLE_LIB")   # a mutant build, for the mutation tests
            if override:
                _lib = _declare(ctypes.CDLL(override))
            else:
                if _stale():
                    compile_library()
                _lib = _declare(ctypes.CDLL(_LIB))
    return _lib


def _dirty(n: int) -> np.ndarray:
    """An output buffer pre-filled with 0xA5, so every byte the caller reads
    (padding included) must have been written by the oracle."""
    return np.full(max(int(n), 1), 0xA5, dtype=np.uint8)


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


# --------------------------------------------------------------------------
# numpy-level wrappers (arrays are C-contiguous; bf16 is carried as uint16)
# --------------------------------------------------------------------------

def sf_region_bytes(rows: int, kv: int, layout: int, lib=None) -> int:
    lib = lib or load()
    return int(lib.qzo_sf_region_bytes(rows, kv, layout))


def quantize_mxfp8(x: np.ndarray, layout: int, lib=None):
    """x: uint16 [rows, ld] (bf16 bits; the first ``cols`` columns are used
    when ``x`` is a view with a larger row stride).  Returns (q, sf)."""
    lib = lib or load()
    rows, cols = x.shape
    assert x.dtype == np.uint16 and (rows == 0 or x.strides[1] == 2)
    ld = x.strides[0] // 2 if rows > 0 else cols
    q = np.zeros((rows, cols), dtype=np.uint8)
    sf = _dirty(sf_region_bytes(rows, cols // 32, layout, lib))
    if rows > 0:
        lib.qzo_quantize_mxfp8(ctypes.c_void_p(x.__array_interface__["data"][0]), rows, cols, ld,
                               _ptr(q), _ptr(sf), layout)
    return q, sf[: sf_region_bytes(rows, cols // 32, layout, lib)]


def quantize_nvfp4(x: np.ndarray, layout: int, mode: int, amax_in: float | None = None, lib=None):
    """Returns (q [rows, cols/2] uint8, sf bytes, amax float32 array)."""
    lib = lib or load()
    rows, cols = x.shape
    assert x.dtype == np.uint16 and (rows == 0 or x.strides[1] == 2)
    ld = x.strides[0] // 2 if rows > 0 else cols
    q = np.zeros((rows, cols // 2), dtype=np.uint8)
    n_sf = sf_region_bytes(rows, cols // 16, layout, lib)
    sf = _dirty(n_sf)
    if mode == NVFP4_PER_ROW:
        amax = np.zeros(max(rows, 1), dtype=np.float32)
    else:
        amax = np.zeros(1, dtype=np.float32)
        if mode == NVFP4_PER_TENSOR_GIVEN:
            amax[0] = np.float32(amax_in)
    if rows > 0:
        lib.qzo_quantize_nvfp4(ctypes.c_void_p(x.__array_interface__["data"][0]), rows, cols, ld,
                               _ptr(q), _ptr(sf), layout, mode, _ptr(amax))
    return q, sf[:n_sf], (amax[:rows] if mode == NVFP4_PER_ROW else amax)


def dequantize_mxfp8(q: np.ndarray, sf: np.ndarray, layout: int, lib=None) -> np.ndarray:
    """bf16 bits [rows, cols] of an MXFP8 payload q [rows, cols] and its SF bytes (R11)."""
    lib = lib or load()
    rows, cols = q.shape
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    y = np.zeros((rows, cols), dtype=np.uint16)
    if rows > 0:
        lib.qzo_dequantize_mxfp8(_ptr(q), _ptr(sf), rows, cols, layout, _ptr(y), cols)
    return y


def dequantize_nvfp4(q: np.ndarray, sf: np.ndarray, amax: np.ndarray, per_row: bool, layout: int,
                     lib=None) -> np.ndarray:
    """bf16 bits [rows, cols] of a packed NVFP4 payload q [rows, cols/2], its SF
    bytes and its amax (per tensor [1] or per row [rows]) (R11)."""
    lib = lib or load()
    rows, half = q.shape
    cols = 2 * half
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    amax = np.ascontiguousarray(amax, dtype=np.float32)
    y = np.zeros((rows, cols), dtype=np.uint16)
    if rows > 0:
        lib.qzo_dequantize_nvfp4(_ptr(q), _ptr(sf), _ptr(amax), 1 if per_row else 0, rows, cols, layout, _ptr(y), cols)
    return y


def attention_merge(O: np.ndarray, lse: np.ndarray, lib=None) -> np.ndarray:
    """bf16 bits [T, H] of the merged attention output of partial outputs
    O [S, T, H] (float32) with log-sum-exps lse [S, T] (float32) (R12)."""
    lib = lib or load()
    S, T, H = O.shape
    O = np.ascontiguousarray(O, dtype=np.float32)
    lse = np.ascontiguousarray(lse, dtype=np.float32)
    y = np.zeros((T, H), dtype=np.uint16)
    if T > 0:
        lib.qzo_attention_merge(_ptr(O), _ptr(lse), S, T, H, _ptr(y))
    return y


class CutRefused(ValueError):
    """A gate|up cut that would divide a scale block (R14)."""


def split_region_bytes(fmt: int, rows: int, cols: int, layout: int, lib=None) -> int:
    """Scale bytes of one part of ``rows`` weight rows after the split."""
    lib = lib or load()
    if fmt == FP8_BLOCK128:
        return -(-rows // 128) * -(-cols // 128) * 4 if rows > 0 else 0
    return int(lib.qzo_sf_region_bytes(rows, cols // (32 if fmt == MXFP8 else 16), layout))


def split_fused(fmt: int, q: np.ndarray, sf: np.ndarray, amax, amax_kind: int, cols: int, cut: int,
                src_layout: int, dst_layout: int, lib=None):
    """Cut a folded fused expert (payload q [rows, row_bytes], scales sf in
    src_layout, amax per amax_kind) at weight row ``cut`` (R14).  Returns
    [(q_p, sf_p, amax_p)] for part 0 (rows [0, cut)) and part 1 (rows
    [cut, rows)); raises CutRefused when the cut divides a scale block."""
    lib = lib or load()
    q = np.ascontiguousarray(q, dtype=np.uint8)
    rows = q.shape[0]
    sf = np.ascontiguousarray(sf, dtype=np.uint8).reshape(-1)
    row_bytes = cols // 2 if fmt == NVFP4 else cols
    counts = (cut, rows - cut)
    outs = []
    for n in counts:
        qp = np.full((max(n, 0), row_bytes), 0xA5, dtype=np.uint8)
        sp = _dirty(split_region_bytes(fmt, max(n, 0), cols, dst_layout, lib))
        ap = np.full(max(1 if amax_kind == AMAX_PER_TENSOR else max(n, 0), 1), np.nan, dtype=np.float32)
        outs.append((qp, sp, ap))
    a = np.ascontiguousarray(np.zeros(1, np.float32) if amax is None else amax, dtype=np.float32)
    rc = lib.qzo_split_fused(fmt, _ptr(q) if q.size else None, _ptr(sf), _ptr(a), amax_kind, rows, cols, cut,
                             src_layout, dst_layout,
                             _ptr(outs[0][0]), _ptr(outs[0][1]), _ptr(outs[0][2]),
                             _ptr(outs[1][0]), _ptr(outs[1][1]), _ptr(outs[1][2]))
    if rc != 0:
        raise CutRefused(f"cut {cut} of {rows} rows divides a scale block")
    res = []
    for (qp, sp, ap), n in zip(outs, counts):
        nb = split_region_bytes(fmt, n, cols, dst_layout, lib)
        na = 1 if amax_kind == AMAX_PER_TENSOR else (n if amax_kind == AMAX_PER_ROW else 0)
        res.append((qp, sp[:nb], ap[:na]))
    return res


def quantize_colwise(x: np.ndarray, fmt: int, layout: int, mode: int = NVFP4_PER_TENSOR_GIVEN,
                     amax_in: float | None = None, lib=None):
    """Column-wise quantization of x [rows, cols]: blocks run down the columns,
    i.e. the row-wise quantization of the transpose x^T [cols, rows]
    (payload [cols, rows] or [cols, rows/2], SF of a [cols, rows] matrix).
    Returns (q, sf) for MXFP8, (q, sf, amax) for NVFP4."""
    xt = np.ascontiguousarray(np.asarray(x, dtype=np.uint16).T)
    if fmt == MXFP8:
        return quantize_mxfp8(xt, layout, lib)
    return quantize_nvfp4(xt, layout, mode, amax_in, lib)


def swizzle(lin: np.ndarray, rows: int, kv: int, lib=None) -> np.ndarray:
    lib = lib or load()
    lin = np.ascontiguousarray(lin, dtype=np.uint8)
    out = _dirty(sf_region_bytes(rows, kv, SWIZZLED, lib))
    if rows > 0:
        lib.qzo_swizzle(_ptr(lin), rows, kv, _ptr(out))
    return out[: sf_region_bytes(rows, kv, SWIZZLED, lib)]


def unswizzle(swz: np.ndarray, rows: int, kv: int, lib=None) -> np.ndarray:
    lib = lib or load()
    swz = np.ascontiguousarray(swz, dtype=np.uint8)
    out = np.zeros(max(rows * kv, 1), dtype=np.uint8)
    if rows > 0:
        lib.qzo_unswizzle(_ptr(swz), rows, kv, _ptr(out))
    return out[: rows * kv]


def residual_rmsnorm(x: np.ndarray, r: np.ndarray, gamma: np.ndarray, eps: float, lib=None):
    """Returns (y, h) as uint16 bf16 bits."""
    lib = lib or load()
    T, H = x.shape
    x = np.ascontiguousarray(x)
    r = np.ascontiguousarray(r)
    gamma = np.ascontiguousarray(gamma)
    y = np.zeros((T, H), dtype=np.uint16)
    h = np.zeros((T, H), dtype=np.uint16)
    lib.qzo_residual_rmsnorm(_ptr(x), _ptr(r), _ptr(gamma), ctypes.c_float(eps), T, H, _ptr(y), _ptr(h))
    return y, h


def rmsnorm_quantize(x, r, gamma, eps, fmt, layout, amax_in=None, lib=None):
    """Returns (y, h, q, sf)."""
    lib = lib or load()
    T, H = x.shape
    x = np.ascontiguousarray(x)
    r = np.ascontiguousarray(r)
    gamma = np.ascontiguousarray(gamma)
    y = np.zeros((T, H), dtype=np.uint16)
    h = np.zeros((T, H), dtype=np.uint16)
    blk = 32 if fmt == MXFP8 else 16
    q = np.zeros((T, H if fmt == MXFP8 else H // 2), dtype=np.uint8)
    n_sf = sf_region_bytes(T, H // blk, layout, lib)
    sf = _dirty(n_sf)
    amax = np.array([0.0 if amax_in is None else amax_in], dtype=np.float32)
    lib.qzo_rmsnorm_quantize(_ptr(x), _ptr(r), _ptr(gamma), ctypes.c_float(eps), T, H,
                             _ptr(y), _ptr(h), fmt, _ptr(q), _ptr(sf), layout, _ptr(amax))
    return y, h, q, sf[:n_sf]


def rank_sum(xs, lib=None) -> np.ndarray:
    """The AllReduce of same-shape uint16 (bf16 bits) rank inputs (R15)."""
    lib = lib or load()
    xs = [np.ascontiguousarray(x) for x in xs]
    assert xs and all(x.dtype == np.uint16 and x.shape == xs[0].shape for x in xs)
    out = np.zeros(xs[0].shape, dtype=np.uint16)
    table = (ctypes.c_void_p * len(xs))(*[x.ctypes.data for x in xs])
    lib.qzo_rank_sum(table, len(xs), out.size, _ptr(out))
    return out


def allreduce_rmsnorm_quantize(xs, r, gamma, eps, fmt, layout, amax_in=None, lib=None):
    """The fused epilogue on the AllReduce of the rank inputs ``xs``:
    ``rmsnorm_quantize`` applied to ``rank_sum(xs)``.  Returns (y, h, q, sf)."""
    lib = lib or load()
    return rmsnorm_quantize(rank_sum(xs, lib), r, gamma, eps, fmt, layout, amax_in, lib)


def quantize_grouped(experts, fmt: int, layout: int, mode: int = NVFP4_PER_ROW,
                     amax_in=None, threads: int = 1):
    """Quantize a list of uint16 expert matrices independently.

    ``threads`` > 1 runs experts on a thread pool (ctypes releases the GIL
    during each call).  Returns a list of per-expert result tuples.
    """
    lib = load()

    def one(i):
        x = experts[i]
        if fmt == MXFP8:
            return quantize_mxfp8(x, layout, lib)
        a = None if amax_in is None else amax_in[i]
        return quantize_nvfp4(x, layout, mode, a, lib)

    if threads <= 1:
        return [one(i) for i in range(len(experts))]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(one, range(len(experts))))


def host_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1
