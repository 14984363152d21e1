"""Multi-rank host logic of bench.py on CPU: two gloo ranks, each with its own
timed seconds and token count; the job time is the max over ranks and the
units are summed (replicas of the layer, no collective on the data path)."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w, lr = bench.dist_env()
    assert (r, w, lr) == (rank, world, rank)
    bench.init_dist(world, "gloo")
    secs = [0.25, 0.40][rank]
    units = [128 * 10, 128 * 10][rank]
    t, u = bench.reduce_time_and_units(secs, units, world)
    bench.barrier(world)
    out[rank] = (t, u)
    dist.destroy_process_group()


def test_two_rank_max_time_sum_units():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    for rank in range(world):
        t, u = out[rank]
        assert t == 0.40 and u == 2560.0
    # the bench's value for this job
    assert out[0][1] / out[0][0] == 6400.0


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_time_and_units(0.5, 100, 1) == (0.5, 100)
