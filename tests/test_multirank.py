"""Multi-rank host logic of bench.py on CPU: two gloo ranks, each with its own
seeded workload; the job time is the maximum over ranks and the throughput is
all ranks' bytes over that time.  (The data path has no collective.)"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank draws its own inputs
        seed = 2 + bench.rank_seed_offset(rank) * 1000
        x = synth.expert_stack(1, (8, 64), 0.02, seed=seed)
        sig = float(x.float().abs().sum())
        # per-rank times differ; everyone must see the slowest
        mx = bench.max_over_ranks([10.0 + rank, 5.0 * (world - rank)], torch.device("cpu"))
        gathered = [None] * world
        dist.all_gather_object(gathered, (sig, mx))
        out[rank] = gathered
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_max_time_and_distinct_inputs():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    g0, g1 = out[0], out[1]
    assert g0 == g1
    (s0, mx0), (s1, mx1) = g0
    assert s0 != s1, "ranks must quantize different synthetic data"
    assert mx0 == mx1 == [11.0, 10.0]


def test_aggregate_throughput_formula():
    import bench
    # 2 ranks x 1e9 bytes x 4 steps in 2 ms (max over ranks) -> 4000 GB/s
    assert abs(bench.aggregate_gbs(10 ** 9, 2, 4, 2.0) - 4.0e3) < 1e-9
