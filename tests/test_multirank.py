"""The multi-rank (replica) logic of bench.py on CPU: two gloo ranks.

Each rank runs its own independent batch; the only cross-rank operation is the
max of the step time, and the reported value is all ranks' work over it.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                 # rank 1 is the slower one
        mx = bench.max_over_ranks(ms)
        out[rank] = (mx, bench.weak_scaling_value(1e12, world, 4, mx))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_weak_scaling_value():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    for r in range(world):
        mx, val = out[r]
        assert mx == 15.0                        # both ranks see the slowest rank's time
        assert val == pytest.approx(1e12 * 2 * 4 / 15e-3 / 1e12)


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.band_pairs(2048, 2048) == 2048 * 2049 // 2
    assert bench.band_pairs(2048, 512) == 512 * 513 // 2 + 1536 * 512
    assert bench.band_pairs(5, 1) == 5
