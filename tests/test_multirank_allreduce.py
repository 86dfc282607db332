"""Host logic of the AllReduce epilogue on CPU: the slice partition, the buffer
layout shared by the ranks, and the call sequence of two gloo ranks (barrier,
launch with the group's addresses in rank order, barrier), with the launch
recorded instead of run.  The kernel itself is checked on the GPU with the
ranks emulated as separate buffers (test_gpu_allreduce.py)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import nvfp4_quantization_moe_b200 as qz
from nvfp4_quantization_moe_b200 import allreduce as ar


def test_rank_rows_cover_every_row_once():
    for world in range(1, 9):
        for T in (0, 1, 7, 8, 9, 127, 128, 300, 4096, 4099):
            spans = [ar.rank_rows(T, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == T
            for (b0, e0), (b1, _) in zip(spans, spans[1:]):
                assert e0 == b1
            lens = [e - b for b, e in spans]
            assert max(lens) - min(lens) <= 1 and lens == sorted(lens, reverse=True)
    for bad in ((5, 0, 0), (5, 2, 2), (5, 2, -1), (-1, 2, 0)):
        with pytest.raises(ValueError):
            ar.rank_rows(*bad)


@pytest.mark.parametrize("fmt,layout", [(qz.FMT_MXFP8, qz.SF_SWIZZLED), (qz.FMT_NVFP4, qz.SF_LINEAR)])
def test_layout_regions_are_aligned_and_disjoint(fmt, layout):
    T, H = 300, 7168
    L = ar.SymmetricLayout(T, H, fmt, layout)
    q = T * (H if fmt == qz.FMT_MXFP8 else H // 2)
    regions = [(L.x, T * H * 2), (L.y, T * H * 2), (L.h, T * H * 2), (L.q, q), (L.sf, qz.sf_bytes(T, H, fmt, layout))]
    for off, n in regions:
        assert off % 256 == 0
    for (a, n), (b, _) in zip(regions, regions[1:]):
        assert a + n <= b
    assert regions[-1][0] + regions[-1][1] <= L.total


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from nvfp4_quantization_moe_b200 import allreduce as ar_
    import nvfp4_quantization_moe_b200 as qz_
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bases = [None] * world
        dist.all_gather_object(bases, (rank + 1) << 32)          # each rank's own mapping of its allocation
        events = []

        def barrier():
            dist.barrier()
            events.append("barrier")

        def launch(xs, residual, gamma, eps, dests, fmt, layout, T, H, rows, global_amax, stream):
            events.append(("launch", list(xs), rows, [tuple(d) for d in dests], fmt, layout, T, H))

        L = ar_.SymmetricLayout(300, 7168, qz_.FMT_MXFP8, qz_.SF_SWIZZLED)
        for slice_form in (True, False):
            ep = ar_.AllReduceEpilogue(rank, world, bases, L, barrier, slice_form, launch=launch)
            ep(300, None, None, 1e-6)
        out[rank] = (bases, L.x, L.y, L.h, L.q, L.sf, events)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_call_sequence():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    rows_seen = []
    for rank in range(world):
        bases, ox, oy, oh, oq, osf, events = out[rank]
        assert bases == [1 << 32, 2 << 32]
        # each call: barrier, launch, barrier
        assert [e if isinstance(e, str) else e[0] for e in events] == ["barrier", "launch", "barrier"] * 2
        sl, one = events[1], events[4]
        xs = [b + ox for b in bases]
        dests = [(b + oy, b + oh, b + oq, b + osf) for b in bases]
        # slice form: all ranks' inputs in rank order, this rank's rows, every rank's destinations
        assert sl[1] == xs and sl[3] == dests and sl[6:] == (300, 7168)
        rows_seen.append(sl[2])
        # one-shot form: the same inputs, all rows, this rank's own buffers only
        assert one[1] == xs and one[2] == (0, 300) and one[3] == [dests[rank]]
    assert rows_seen == [(0, 150), (150, 300)]


def _ipc_worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from nvfp4_quantization_moe_b200 import allreduce as ar_
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = (rank + 1) << 40
        opened, closed = [], []

        def export(ptr):                      # a handle that names its exporter
            return f"h:{ptr}".encode()

        def import_(h):
            ptr = int(h.decode().split(":")[1])
            opened.append(ptr)
            return ptr + 0x10                 # the peer's pointer as mapped here

        def close(p, h):
            closed.append((p, h))

        with ar_.PeerBuffers(local, export=export, import_=import_, close=close) as pb:
            bases = list(pb.bases)
        out[rank] = (bases, opened, closed)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_peer_buffers_exchange_over_gloo():
    """Three gloo ranks: every rank's handle reaches every rank, peers are
    mapped in rank order, a rank's own pointer is not mapped, and every
    mapping is closed again."""
    world = 3
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_ipc_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    locals_ = [(r + 1) << 40 for r in range(world)]
    for rank in range(world):
        bases, opened, closed = out[rank]
        assert bases == [p if r == rank else p + 0x10 for r, p in enumerate(locals_)]
        assert opened == [p for r, p in enumerate(locals_) if r != rank]
        assert sorted(p for p, _ in closed) == sorted(p + 0x10 for p in opened)
