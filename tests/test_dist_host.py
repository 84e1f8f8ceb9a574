"""Host-side multi-rank logic of bench.py on CPU with gloo (world size 2): each rank gets its
own seed (weak scaling, no data exchange) and the timing is the max over ranks."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, lr = bench.dist_env()
        elapsed = 10.0 + 5.0 * rank  # rank 1 is the slow one
        mx = bench.max_over_ranks(elapsed, "cpu")
        bench.barrier()
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(r))
        out[rank] = (r, w, lr, mx, bench.aggregate_us_per_step(mx, 64, w), tuple(seeds))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_sharding():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    for rank in range(world):
        r, w, lr, mx, us, seeds = out[rank]
        assert (r, w, lr) == (rank, world, rank)
        assert mx == 15.0                                  # max over ranks, identical on every rank
        assert us == pytest.approx(15.0 * 1000 / (64 * 2))  # whole-job time per step
        assert len(set(seeds)) == world                   # every rank draws its own batch
