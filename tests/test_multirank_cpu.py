"""The multi-replica bench path on CPU: two gloo ranks agree on the slowest rank's time and the summed entries."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms, entries = bench.reduce_over_ranks(10.0 + 5.0 * rank, 262144, torch.device("cpu"))
    out[rank] = (ms, entries)
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_reduce_time_and_entries():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert dict(out) == {0: (15.0, 2 * 262144), 1: (15.0, 2 * 262144)}


def test_reference_arm_other_ranks_do_nothing():
    import bench

    class A:
        steps, warmup = 1, 0
    assert bench.run_reference(A(), rank=1, world=2) is None
