"""The multi-rank benchmark aggregation (weak scaling, independent batches, max-over-ranks
device time, bytes summed over ranks) on two gloo ranks on the CPU."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r pretends its step took (r+1) ms and moved (r+1) GB
        ms, gbs = bench.aggregate(float(rank + 1), (rank + 1) * 1e9, torch.device("cpu"))
        mx = bench.reduce_max([float(rank), 10.0 - rank], torch.device("cpu"))
        out[rank] = (ms, gbs, mx)
        bench.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_gloo():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    for rank in range(world):
        ms, gbs, mx = out[rank]
        assert ms == 2.0                                   # slowest rank
        assert abs(gbs - 3e9 / 2e-3 / 1e9) < 1e-6           # 3 GB over 2 ms = 1500 GB/s
        assert mx == [1.0, 10.0]


def test_single_process_aggregation_is_identity():
    import bench
    ms, gbs = bench.aggregate(4.0, 8e9, torch.device("cpu"))
    assert ms == 4.0 and abs(gbs - 2000.0) < 1e-9
