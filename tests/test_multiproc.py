"""Host logic of the multi-process (replica) path of bench.py, run as two
gloo ranks on the CPU: the job time is the slowest rank's, the work the sum
of all ranks', and the ranks start on different views."""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 17.25][rank]
        units = [1_000_000, 3_000_000][rank]
        got = bench.combine_ranks(ms, units, dist, "cpu")
        views = [bench.rank_view(k, rank, 8) for k in range(3)]
        out[rank] = (got, views)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_combine_time_and_work():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(out)
    for rank in range(world):
        (ms, units), views = res[rank]
        assert ms == 17.25 and units == 4_000_000
        assert views == [(k + rank) % 8 for k in range(3)]
    assert res[0][1][0] != res[1][1][0]


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.combine_ranks(3.5, 7, None, "cpu") == (3.5, 7.0)
