"""Host side of the AllReduce epilogue on one node's tensor-parallel group.

TensorRT-LLM "NVFP4 linear-SF AllReduce epilogue" (commit 2) and "MXFP8
carrier and quantize folds" (commit 6): the AllReduce that ends a tensor-
parallel block is followed by residual add + RMSNorm + quantize in the same
pass.  The kernel (``qz_allreduce_rmsnorm_quantize``) reads every rank's input
and writes every destination through plain device pointers and never waits on
another GPU.  This module owns what surrounds it:

* ``rank_rows``: the slice form's partition of the T rows over the ranks;
* ``SymmetricLayout``: where each rank's input and output buffers sit inside
  one allocation that every rank maps (the same offsets on every rank);
* ``AllReduceEpilogue``: one call = a barrier (every rank's input written,
  every destination free), the launch with the group's addresses in rank
  order, and a second barrier (no rank overwrites its input, or reads a
  destination that peers write, before all have finished).

The addresses come from ``PeerBuffers``: every rank exports a CUDA IPC handle
of its own allocation (``qz_ipc_export``), the handles are all-gathered over
the process group, and every rank maps its peers' allocations
(``qz_ipc_import``); a symmetric-memory allocator's per-rank pointers serve as
well.  The barrier can be an NCCL all-reduce of one integer on the launching
stream, or a synchronize plus a process-group barrier; either way the process
group's timeout bounds its waits on the host.

The one-shot form computes all T rows on every rank into its own buffers;
the slice form computes ``rank_rows(T, world, rank)`` and writes them to every
rank's buffers (reduce-scatter and all-gather in one kernel).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch.distributed as dist

from . import binding

_ALIGN = 256


def _up(n: int, a: int = _ALIGN) -> int:
    return (n + a - 1) // a * a


def rank_rows(T: int, world: int, rank: int) -> Tuple[int, int]:
    """Rows [begin, end) that ``rank`` reduces in the slice form: T cut into
    ``world`` consecutive runs whose lengths differ by at most one, the longer
    runs first.  Every row belongs to exactly one rank."""
    if world < 1 or not 0 <= rank < world or T < 0:
        raise ValueError(f"rank_rows: T={T}, world={world}, rank={rank}")
    base, extra = divmod(T, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


class SymmetricLayout:
    """Byte offsets of one rank's buffers inside its allocation, for up to
    ``max_T`` rows of ``H``: x (bf16 [max_T, H]) | norm_out | residual_out
    (bf16) | q (payload) | sf (SF region of max_T rows), each 256-byte aligned.
    A call with T <= max_T uses the first T rows of each (the SF region of T
    rows is a prefix of that of max_T rows in both layouts)."""

    def __init__(self, max_T: int, H: int, fmt: int, sf_layout: int, with_residual_out: bool = True):
        self.max_T, self.H, self.fmt, self.sf_layout = int(max_T), int(H), int(fmt), int(sf_layout)
        bf = self.max_T * self.H * 2
        qbytes = self.max_T * (self.H if fmt == binding.FMT_MXFP8 else self.H // 2)
        sfbytes = binding.sf_bytes(self.max_T, self.H, fmt, sf_layout) if self.max_T else 0
        self.x = 0
        self.y = _up(self.x + bf)
        self.h = _up(self.y + bf) if with_residual_out else None
        self.q = _up((self.h if with_residual_out else self.y) + bf)
        self.sf = _up(self.q + qbytes)
        self.total = _up(self.sf + max(sfbytes, 16))


class AllReduceEpilogue:
    """One tensor-parallel group's AllReduce + residual add + RMSNorm + quantize.

    ``bases``: every rank's allocation address as mapped in this process, in
    rank order (this rank's own at index ``rank``); ``barrier``: a
    stream-ordered barrier of the group; ``launch``: the kernel call
    (``binding.allreduce_rmsnorm_quantize``)."""

    def __init__(self, rank: int, world: int, bases: Sequence[int], layout: SymmetricLayout,
                 barrier: Callable[[], None], slice_form: bool = True,
                 launch: Callable = binding.allreduce_rmsnorm_quantize):
        if not 1 <= world <= binding.MAX_RANKS or len(bases) != world or not 0 <= rank < world:
            raise ValueError(f"AllReduceEpilogue: rank {rank} of {world} with {len(bases)} bases")
        self.rank, self.world = rank, world
        self.bases = [int(b) for b in bases]
        self.layout = layout
        self.barrier = barrier
        self.slice_form = slice_form
        self.launch = launch

    def input_ptr(self, r: int) -> int:
        return self.bases[r] + self.layout.x

    def dest(self, r: int) -> Tuple[int, Optional[int], int, int]:
        b, L = self.bases[r], self.layout
        return (b + L.y, None if L.h is None else b + L.h, b + L.q, b + L.sf)

    def plan(self, T: int):
        """(rank inputs, rows, destinations) of this rank's launch for T rows."""
        if not 0 <= T <= self.layout.max_T:
            raise ValueError(f"T={T} outside 0..{self.layout.max_T}")
        xs: List[int] = [self.input_ptr(r) for r in range(self.world)]
        if self.slice_form:
            return xs, rank_rows(T, self.world, self.rank), [self.dest(r) for r in range(self.world)]
        return xs, (0, T), [self.dest(self.rank)]

    def __call__(self, T: int, residual, gamma, eps: float, global_amax=None, stream=None):
        xs, rows, dests = self.plan(T)
        L = self.layout
        self.barrier()
        self.launch(xs, residual, gamma, eps, dests, L.fmt, L.sf_layout, T, L.H, rows=rows,
                    global_amax=global_amax, stream=stream)
        self.barrier()


class PeerBuffers:
    """Every rank's allocation as mapped in this process, in rank order.

    Each rank exports an IPC handle of ``local_ptr`` (its own buffer), the
    handles are all-gathered over ``group`` (any backend), and every peer's
    allocation is mapped; this rank's own pointer is used as is (CUDA IPC
    does not map a handle into the process that exported it).  ``bases`` is
    the list the epilogue takes; ``close()`` unmaps the peers (call it after
    the last launch that reads or writes them has finished)."""

    def __init__(self, local_ptr: int, group=None, export: Callable = binding.ipc_export,
                 import_: Callable = binding.ipc_import, close: Callable = binding.ipc_close):
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        mine = export(int(local_ptr))
        self.handles: List[bytes] = [b""] * self.world
        dist.all_gather_object(self.handles, mine, group=group)
        self._close = close
        self.bases: List[int] = []
        self._opened: List[Tuple[int, bytes]] = []
        try:
            for r, h in enumerate(self.handles):
                if r == self.rank:
                    self.bases.append(int(local_ptr))
                else:
                    p = import_(h)
                    self._opened.append((p, h))
                    self.bases.append(p)
        except Exception:
            self.close()
            raise

    def close(self):
        while self._opened:
            p, h = self._opened.pop()
            self._close(p, h)

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()
