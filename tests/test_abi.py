"""The C-ABI library builds, loads and exports every function include/qz.h
declares; host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import nvfp4_quantization_moe_b200 as qz
from nvfp4_quantization_moe_b200 import build as qzbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qz.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qz_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    qzbuild.build()
    return qz.load()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("qz_quantize_grouped_mxfp8", "qz_quantize_grouped_nvfp4", "qz_rmsnorm_quantize",
              "qz_swizzle_scales", "qz_sf_bytes", "qz_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", qz.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT\s+(qz_[a-z0-9_]+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(lib, n)
    assert set(qz.EXPORTED) <= exported


def test_sf_bytes_matches_oracle_regions(lib):
    import oracle
    for rows in (0, 1, 64, 127, 128, 129, 1536, 3000):
        for cols in (16, 32, 48, 64, 256, 768, 2048, 4096, 7168):
            for fmt, blk in ((qz.FMT_MXFP8, 32), (qz.FMT_NVFP4, 16)):
                for layout in (qz.SF_LINEAR, qz.SF_SWIZZLED):
                    got = qz.sf_bytes(rows, cols, fmt, layout)
                    if cols % blk:
                        assert got == 0
                    else:
                        assert got == oracle.sf_region_bytes(rows, cols // blk, layout)
    assert qz.sf_bytes(4, 64, 7, 0) == 0 and qz.sf_bytes(4, 64, 0, 9) == 0 and qz.sf_bytes(-1, 64, 0, 0) == 0


def test_host_errors_without_gpu(lib):
    P = ctypes.c_void_p
    assert lib.qz_quantize_grouped_mxfp8(None, -1, 0, None, None) == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_quantize_grouped_mxfp8(None, 3, 0, None, None) == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_quantize_grouped_mxfp8(P(0x1000), qz.MAX_EXPERTS + 1, 0, None, None) == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_quantize_grouped_mxfp8(P(0x1000), 2, 5, None, None) == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_quantize_grouped_mxfp8(None, 0, 0, None, None) == qz.QZ_OK
    assert lib.qz_quantize_grouped_nvfp4(P(0x1000), 2, 7, 0, None, None) == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_quantize_grouped_nvfp4(None, 0, 2, 1, None, None) == qz.QZ_OK
    assert lib.qz_swizzle_scales(None, 1, None, None) == qz.QZ_ERR_INVALID_ARG
    # a workspace smaller than qz_workspace_bytes is refused before any launch
    small = qz.binding._Opts(None, 0, P(0x10000), ctypes.c_size_t(16))
    assert lib.qz_quantize_grouped_nvfp4(P(0x1000), 4, 1, 1, None, ctypes.byref(small)) == qz.QZ_ERR_INVALID_ARG
    odd = qz.binding._Opts(None, 0, P(0x10002), ctypes.c_size_t(qz.workspace_bytes(4)))
    assert lib.qz_quantize_grouped_nvfp4(P(0x1000), 4, 1, 1, None, ctypes.byref(odd)) == qz.QZ_ERR_ALIGNMENT
    neg = qz.binding._Opts(None, 0, P(0x10000), ctypes.c_size_t(qz.workspace_bytes(4)), 0, -1, 0)
    assert lib.qz_quantize_grouped_nvfp4(P(0x1000), 4, 1, 1, None, ctypes.byref(neg)) == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_quantize_grouped_nvfp4_compute_noalloc(P(0x1000), 4, 1, None, ctypes.byref(neg)) == \
        qz.QZ_ERR_INVALID_ARG
    h = qz.IpcHandle()
    out = ctypes.c_void_p()
    assert lib.qz_ipc_export(None, ctypes.byref(h)) == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_ipc_export(P(0x1000), None) == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_ipc_import(None, ctypes.byref(out)) == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_ipc_import(ctypes.byref(h), None) == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_ipc_close(None, ctypes.byref(h)) == qz.QZ_ERR_INVALID_ARG
    if not torch.cuda.is_available():
        # no device: the runtime refuses, the call reports it
        assert lib.qz_ipc_export(P(0x1000), ctypes.byref(h)) == qz.QZ_ERR_CUDA
    assert qz.workspace_bytes(0) == 0 and qz.workspace_bytes(qz.MAX_EXPERTS + 1) == 0
    assert qz.workspace_bytes(128) >= 4 * (128 + 1)
    assert lib.qz_swizzle_scales(None, 0, None, None) == qz.QZ_OK
    assert lib.qz_dequantize_grouped(None, -1, 0, 0, 0, None, None) == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_dequantize_grouped(None, 2, 0, 0, 0, None, None) == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_dequantize_grouped(P(0x1000), 2, 5, 0, 0, None, None) == qz.QZ_ERR_INVALID_ARG   # format
    assert lib.qz_dequantize_grouped(P(0x1000), 2, 1, 0, 3, None, None) == qz.QZ_ERR_INVALID_ARG   # layout
    assert lib.qz_dequantize_grouped(None, 0, 1, 1, 1, None, None) == qz.QZ_OK
    assert lib.qz_quantize_grouped_colwise(None, 1, 0, 0, None, None) == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_quantize_grouped_colwise(P(0x1000), 1, 3, 0, None, None) == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_quantize_grouped_colwise(P(0x1000), 1, 0, 4, None, None) == qz.QZ_ERR_INVALID_ARG
    assert lib.qz_quantize_grouped_colwise(None, 0, 1, 1, None, None) == qz.QZ_OK

    def split(n=2, fmt=1, amax=1, src=1, dst=1, table=P(0x1000)):
        return lib.qz_split_fused_experts(table, n, fmt, amax, src, dst, None, None)

    assert split(n=-1) == qz.QZ_ERR_INVALID_ARG
    assert split(table=None) == qz.QZ_ERR_INVALID_ARG
    assert split(fmt=3) == qz.QZ_ERR_INVALID_ARG
    assert split(amax=3) == qz.QZ_ERR_INVALID_ARG
    assert split(fmt=0, amax=1) == qz.QZ_ERR_INVALID_ARG            # MXFP8 has no amax
    assert split(fmt=2, amax=2) == qz.QZ_ERR_INVALID_ARG            # nor FP8 with 128 x 128 block scales
    assert split(src=2) == qz.QZ_ERR_INVALID_ARG
    assert split(fmt=2, amax=0, src=0, dst=1) == qz.QZ_ERR_UNSUPPORTED   # FP32 block scales are linear only
    assert split(n=0, table=None) == qz.QZ_OK
    assert qz.sf_bytes(300, 200, qz.FMT_FP8_BLOCK128, qz.SF_LINEAR) == 4 * 3 * 2
    assert qz.sf_bytes(300, 200, qz.FMT_FP8_BLOCK128, qz.SF_SWIZZLED) == 0
    a16 = P(0x10000)

    def merge(S=4, T=3, H=1024, O=a16, lse=a16, y=a16, q=a16, sf=a16, layout=1):
        return lib.qz_attention_merge_quantize(O, lse, S, T, H, y, q, sf, layout, None)

    assert merge(S=0) == qz.QZ_ERR_INVALID_ARG
    assert merge(S=4097) == qz.QZ_ERR_INVALID_ARG
    assert merge(T=-1) == qz.QZ_ERR_INVALID_ARG
    assert merge(H=1000) == qz.QZ_ERR_INVALID_ARG                 # not a multiple of 32
    assert merge(H=96) == qz.QZ_ERR_UNSUPPORTED                   # swizzled with H / 32 = 3
    assert merge(layout=2) == qz.QZ_ERR_INVALID_ARG
    assert merge(O=None) == qz.QZ_ERR_INVALID_ARG
    assert merge(sf=None) == qz.QZ_ERR_INVALID_ARG                # quantized form without SF storage
    assert merge(y=P(0x10008)) == qz.QZ_ERR_ALIGNMENT
    assert merge(sf=P(0x10004)) == qz.QZ_ERR_ALIGNMENT            # swizzled SF wants 16 bytes
    assert merge(T=0) == qz.QZ_OK
    a = P(0x10000)

    def norm(T=4, H=7168, fmt=0, layout=1, x=a, r=a, g=a, y=a, h=None, q=a, sf=a, amax=None):
        return lib.qz_rmsnorm_quantize(x, r, g, ctypes.c_float(1e-6), T, H, y, h, fmt, q, sf, layout, amax, None)

    assert norm(T=-1) == qz.QZ_ERR_INVALID_ARG
    assert norm(H=0) == qz.QZ_ERR_INVALID_ARG
    assert norm(H=qz.MAX_HIDDEN + 128) == qz.QZ_ERR_INVALID_ARG
    assert norm(H=7168 + 16) == qz.QZ_ERR_INVALID_ARG           # not a multiple of 32 (MXFP8)
    assert norm(H=32 * 6) == qz.QZ_ERR_UNSUPPORTED               # swizzled with kv % 4 != 0
    assert norm(fmt=1, layout=0) == qz.QZ_ERR_INVALID_ARG        # NVFP4 without the global amax
    assert norm(x=None) == qz.QZ_ERR_INVALID_ARG
    assert norm(x=P(0x10002)) == qz.QZ_ERR_ALIGNMENT
    assert norm(sf=P(0x10004)) == qz.QZ_ERR_ALIGNMENT            # swizzled SF wants 16 bytes
    assert norm(fmt=7) == qz.QZ_ERR_INVALID_ARG
    assert norm(T=0) == qz.QZ_OK                                  # nothing to do, nothing launched


def test_allreduce_epilogue_host_checks(lib):
    """Every argument error of qz_allreduce_rmsnorm_quantize is returned before
    any launch (the checks read only the host arrays of addresses)."""
    P = ctypes.c_void_p
    a = 0x10000

    def ar(n=2, nd=1, T=4, H=7168, rows=(0, 4), fmt=0, layout=1, xs=None, ds=None, r=a, g=a, amax=None,
           null_arrays=False):
        xs = [a] * n if xs is None else xs
        ds = [(a, None, a, a)] * nd if ds is None else ds
        xa = (P * max(len(xs), 1))(*xs)
        da = (qz.NormDest * max(len(ds), 1))(*[qz.NormDest(*d) for d in ds])
        return lib.qz_allreduce_rmsnorm_quantize(
            None if null_arrays else ctypes.cast(xa, P), n, P(r), P(g), ctypes.c_float(1e-6), T, H, rows[0], rows[1],
            None if null_arrays else ctypes.cast(da, P), nd, fmt, layout, P(amax) if amax else None, None)

    assert ar(n=0) == qz.QZ_ERR_INVALID_ARG
    assert ar(n=qz.MAX_RANKS + 1) == qz.QZ_ERR_INVALID_ARG
    assert ar(nd=0) == qz.QZ_ERR_INVALID_ARG
    assert ar(nd=qz.MAX_RANKS + 1) == qz.QZ_ERR_INVALID_ARG
    assert ar(null_arrays=True) == qz.QZ_ERR_INVALID_ARG
    assert ar(rows=(-1, 4)) == qz.QZ_ERR_INVALID_ARG
    assert ar(rows=(3, 2)) == qz.QZ_ERR_INVALID_ARG
    assert ar(rows=(0, 5)) == qz.QZ_ERR_INVALID_ARG               # past T
    assert ar(H=7168 + 16) == qz.QZ_ERR_INVALID_ARG               # not a multiple of 32 (MXFP8)
    assert ar(H=qz.MAX_HIDDEN + 128) == qz.QZ_ERR_INVALID_ARG
    assert ar(H=32 * 6) == qz.QZ_ERR_UNSUPPORTED                   # swizzled with kv % 4 != 0
    assert ar(fmt=1, layout=0) == qz.QZ_ERR_INVALID_ARG            # NVFP4 without the global amax
    assert ar(fmt=3) == qz.QZ_ERR_INVALID_ARG
    assert ar(layout=2) == qz.QZ_ERR_INVALID_ARG
    assert ar(xs=[a, None]) == qz.QZ_ERR_INVALID_ARG               # a NULL rank input
    assert ar(ds=[(a, None, None, a)]) == qz.QZ_ERR_INVALID_ARG    # a destination without payload storage
    assert ar(r=None) == qz.QZ_ERR_INVALID_ARG
    assert ar(xs=[a, a + 8]) == qz.QZ_ERR_ALIGNMENT                # rank inputs want 16 bytes
    assert ar(nd=2, ds=[(a, None, a, a), (a, a + 2, a, a)]) == qz.QZ_ERR_ALIGNMENT   # residual_out of dest 1
    assert ar(ds=[(a, None, a, a + 4)]) == qz.QZ_ERR_ALIGNMENT     # swizzled SF wants 16 bytes
    assert ar(ds=[(a, None, a + 4, a)]) == qz.QZ_ERR_ALIGNMENT     # payload wants 8 bytes
    assert ar(T=0, rows=(0, 0)) == qz.QZ_OK                        # nothing to do, nothing launched


def test_status_strings(lib):
    for s in range(5):
        assert qz.status_string(s).startswith("QZ_")
    assert qz.status_string(99) == "unknown qz_status"


def test_product_path_does_not_import_oracle():
    """The binding and the CUDA sources never reach the oracle."""
    pkg = os.path.join(ROOT, "nvfp4_quantization_moe_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text and "qz_oracle" not in text, f


def test_element_hint_reaches_the_launch_options():
    """The binding passes a table's element count as qz_launch_opts.elems_hint
    (the MXFP8 kernels size their grid from it); tables built from raw entries
    carry no hint."""
    xs = [torch.zeros((r, c), dtype=torch.bfloat16) for r, c in ((3, 64), (0, 32), (130, 256))]
    entries = [qz.Entry(x, torch.zeros(max(x.numel(), 1), dtype=torch.uint8), torch.zeros(16, dtype=torch.uint8))
               for x in xs]
    table = qz.ExpertTable(entries, device=torch.device("cpu"))
    assert table.elems == 3 * 64 + 130 * 256
    opts = qz.binding._opts(None, 0, elems_hint=table.elems)
    assert opts._obj.elems_hint == table.elems and opts._obj.max_ctas == 0
    assert qz.binding._opts(None, 0) is None
    raw = qz.ExpertTable.from_raw([(0, 0, 64, 64, 0, 0, 0)], torch.device("cpu"))
    assert raw.elems == 0
    assert ctypes.sizeof(qz.binding._Opts) == 56



def test_binding_structs_match_the_header(tmp_path):
    """Every struct the binding mirrors with ctypes has the header's size and
    field offsets (a probe compiled by gcc against include/qz.h prints them)."""
    b = qz.binding
    mirrors = {"qz_expert": b._Expert, "qz_dq_expert": b._DqExpert, "qz_sf_pair": b._SfPair,
               "qz_fused_split": b._FusedSplit, "qz_launch_opts": b._Opts, "qz_norm_dest": b.NormDest,
               "qz_ipc_handle": b.IpcHandle}
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "qz.h"', "int main(void) {"]
    for cname, cls in mirrors.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in cls._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    limits = {"QZ_MAX_EXPERTS": b.MAX_EXPERTS, "QZ_MAX_HIDDEN": b.MAX_HIDDEN, "QZ_MAX_RANKS": b.MAX_RANKS,
              "QZ_STATIC_WS_MAX_EXPERTS": b.STATIC_WS_MAX_EXPERTS}
    for name in limits:
        lines.append(f'  printf("define {name} %lld\\n", (long long)({name}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "probe.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines():
        cname, field, value = line.split()
        got[(cname, field)] = int(value)
    for name, value in limits.items():
        assert got[("define", name)] == value, f"binding constant of {name}"
    for cname, cls in mirrors.items():
        assert got[(cname, "size")] == ctypes.sizeof(cls), cname
        for fname, _ in cls._fields_:
            assert got[(cname, fname)] == getattr(cls, fname).offset, f"{cname}.{fname}"
