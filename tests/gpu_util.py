"""Helpers for the GPU parity tests: move seeded inputs between host and
device, run the oracle on the host copy, compare bytes with readable reports,
and canary-guard output buffers."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

CANARY = 0xA5
GUARD = 64  # canary bytes before and after every guarded buffer


def have_gpu() -> bool:
    return torch.cuda.is_available()


def host_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16, contiguous."""
    return synth.bf16_bits(t.detach().to("cpu"))


def bf16_ulp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """|a - b| in units of bf16 ulps via the ordered integer map of the bits."""
    def key(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, -(u & 0x7FFF), u & 0x7FFF)
    return np.abs(key(a) - key(b))


def mismatch(a: np.ndarray, b: np.ndarray, what: str, limit: int = 8) -> str:
    a = np.asarray(a).reshape(-1)
    b = np.asarray(b).reshape(-1)
    if a.shape != b.shape:
        return f"{what}: shape {a.shape} vs {b.shape}"
    idx = np.nonzero(a != b)[0]
    if idx.size == 0:
        return ""
    rows = ", ".join(f"[{i}] gpu={int(a[i]):#x} oracle={int(b[i]):#x}" for i in idx[:limit])
    return f"{what}: {idx.size} of {a.size} differ: {rows}"


def assert_bytes_equal(gpu, ref, what: str):
    msg = mismatch(gpu, ref, what)
    assert not msg, msg


class Guarded:
    """A uint8 device buffer of n bytes with canary bytes on both sides."""

    def __init__(self, n: int, device="cuda", fill: int = CANARY):
        self.n = int(n)
        self.raw = torch.full((self.n + 2 * GUARD,), fill, dtype=torch.uint8, device=device)
        self.view = self.raw[GUARD:GUARD + self.n]

    def guards_intact(self) -> bool:
        r = self.raw.cpu().numpy()
        return bool(np.all(r[:GUARD] == CANARY) and np.all(r[GUARD + self.n:] == CANARY))

    def host(self) -> np.ndarray:
        return self.view.cpu().numpy()


def guarded_entries(xs, fmt, layout, mode=oracle.NVFP4_PER_ROW, amax_in=None):
    """Entries whose q / sf / amax buffers are canary-guarded (16-byte aligned)."""
    import nvfp4_quantization_moe_b200 as qz
    out = []
    keep = []
    for i, x in enumerate(xs):
        rows, cols = x.shape
        qbytes = rows * (cols if fmt == qz.FMT_MXFP8 else cols // 2)
        q = Guarded(qbytes)
        sf = Guarded(qz.sf_bytes(rows, cols, fmt, layout))
        amax = None
        amax_t = None
        if fmt == qz.FMT_NVFP4:
            na = max(rows, 1) if mode == qz.NVFP4_PER_ROW else 1
            amax = Guarded(4 * na)
            amax_t = amax.view.view(torch.float32)
            if mode == qz.NVFP4_PER_TENSOR_GIVEN:
                amax_t.fill_(float(amax_in[i]))
        e = qz.Entry(x, q.view.view(rows, -1) if rows else q.view, sf.view, amax_t)
        out.append(e)
        keep.append((q, sf, amax))
    return out, keep


def oracle_threads() -> int:
    return max(1, min(16, oracle.host_threads()))
