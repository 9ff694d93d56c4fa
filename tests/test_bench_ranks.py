"""Host-side multi-rank logic of bench.py on CPU: two gloo ranks (no GPU).

Each rank scans its own seeded batch (replicas, no data-path collective); the
timed region is the slowest rank's, and the whole-job value sums all ranks' work.
"""
import os
import socket

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
    dist.init_process_group("gloo", rank=rank, world_size=world)
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    ms = 10.0 + 5.0 * rank                       # rank 1 is the slower one
    out[rank] = (bench.max_over_ranks(ms, world, "cpu"),
                 bench.sum_over_ranks(1.0, world, "cpu"),
                 bench.rank_seed(20263, rank))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_distinct_seeds():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] == res[1][1] == 2.0
    assert res[0][2] != res[1][2]


def test_single_rank_helpers_are_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.sum_over_ranks(2.0, 1) == 2.0
