"""Host logic of the multi-GPU bench path, on CPU with two gloo ranks.

With N > 1 every rank runs its own batch (weak scaling, no collective on the
data path); the only collectives are the barrier and the max-over-ranks
reduction of the timed intervals, and rank 0 reports the job's throughput
as all ranks' units over the slowest rank's time.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench.dist_env()
        assert (w, r, lr) == (world, rank, rank)
        # rank r took 10 + r ms for the device interval and 30 - r ms end to end
        t, e = bench.max_over_ranks([10.0 + rank, 30.0 - rank], world, "cpu")
        dist.barrier()
        # the reference arm runs on rank 0 only; the others return at once
        skipped = bench.main_reference(None) if rank != 0 else None
        out[rank] = (t, e, bench.rank_seed(7, rank), skipped)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_seeds():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    assert res[0][:2] == res[1][:2] == (11.0, 30.0)
    assert res[0][2] != res[1][2]           # each rank draws its own batch
    assert res[1][3] is None


def test_job_throughput_is_all_units_over_slowest_time():
    # 2 ranks x 3 steps x 100 units in 0.5 s (the slowest rank's time)
    assert bench.job_throughput(100, 2, 3, 500.0) == pytest.approx(1200.0)
    assert bench.max_over_ranks([1.5, 2.5], 1, "cpu") == [1.5, 2.5]
