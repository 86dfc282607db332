"""The AllReduce epilogue across processes through CUDA IPC mappings.

Two processes (one rank each) share the single GPU: each allocates its
buffer, the IPC handles are exchanged over a gloo group (PeerBuffers), each
rank writes its partial input, and the slice form runs on both: every rank
reduces half of the rows, reading the other rank's input and writing the
other rank's destination through the mapped pointers.  No kernel waits on
another: two host barriers (synchronize, then the group barrier) order the
phases.  Each rank's buffer must then hold every row: the rank sum's
residual output bit-exact with the oracle, norm_out within 1 bf16 ulp of the
oracle, and the quantized bytes equal to the oracle quantizer applied to the
kernel's own norm_out, padding included."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

qz = pytest.importorskip("nvfp4_quantization_moe_b200")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, fmt, layout, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    from datetime import timedelta
    import synth
    import nvfp4_quantization_moe_b200 as qz_
    from nvfp4_quantization_moe_b200 import allreduce as ar
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        T, H = 200, synth.FUSED_NORM["hidden"]
        L = ar.SymmetricLayout(T, H, fmt, layout)
        buf = torch.full((L.total,), 0x5A, dtype=torch.uint8, device="cuda")
        xs, r, g = synth.rank_partials(world, T, seed=11)
        x_mine = buf[L.x:L.x + T * H * 2].view(torch.bfloat16).view(T, H)
        x_mine.copy_(xs[rank].cuda())
        amax = torch.tensor([6.0], dtype=torch.float32, device="cuda") if fmt == qz_.FMT_NVFP4 else None

        def barrier():
            torch.cuda.synchronize()
            dist.barrier()

        with ar.PeerBuffers(buf.data_ptr()) as pb:
            ep = ar.AllReduceEpilogue(rank, world, pb.bases, L, barrier, slice_form=True)
            ep(T, r.cuda(), g.cuda(), 1e-6, global_amax=amax)
            torch.cuda.synchronize()
            dist.barrier()          # no rank unmaps while a peer may still write
        host = buf.cpu().numpy()
        qb = T * (H if fmt == qz_.FMT_MXFP8 else H // 2)
        out[rank] = (host[L.y:L.y + T * H * 2].copy(), host[L.h:L.h + T * H * 2].copy(), host[L.q:L.q + qb].copy(),
                     host[L.sf:L.sf + qz_.sf_bytes(T, H, fmt, layout)].copy())
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("fmt,layout", [(qz.FMT_MXFP8, qz.SF_SWIZZLED), (qz.FMT_NVFP4, qz.SF_LINEAR)])
def test_slice_form_across_processes(fmt, layout):
    import oracle
    import synth
    from gpu_util import assert_bytes_equal, bf16_ulp_diff
    world, T, H = 2, 200, synth.FUSED_NORM["hidden"]
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, fmt, layout, out), nprocs=world, join=True, start_method="spawn")
    xs, r, g = synth.rank_partials(world, T, seed=11)
    bits = lambda t: synth.bf16_bits(t)  # noqa: E731
    y_ref, h_ref, _, _ = oracle.allreduce_rmsnorm_quantize([bits(x) for x in xs], bits(r), bits(g), 1e-6, fmt, layout,
                                                           6.0 if fmt == qz.FMT_NVFP4 else None)
    for rank in range(world):
        y, h, q, sf = out[rank]
        y = y.view(np.uint16).reshape(T, H)
        assert_bytes_equal(h.view(np.uint16).reshape(-1), h_ref.reshape(-1), f"rank {rank} residual_out")
        assert bf16_ulp_diff(y, y_ref).max() <= 1, f"rank {rank} norm_out"
        if fmt == qz.FMT_MXFP8:
            qo, so = oracle.quantize_mxfp8(y, layout)
        else:
            qo, so, _ = oracle.quantize_nvfp4(y, layout, oracle.NVFP4_PER_TENSOR_GIVEN, 6.0)
        assert_bytes_equal(q, qo.reshape(-1), f"rank {rank} payload")
        assert_bytes_equal(sf, so, f"rank {rank} scales")
    assert np.array_equal(out[0][2], out[1][2]) and np.array_equal(out[0][3], out[1][3])
