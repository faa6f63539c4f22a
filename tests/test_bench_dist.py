"""Multi-rank logic of bench.py on CPU: two gloo ranks, no GPU.

The hot path shards by independent sequences (no data-path collective); the
benchmark's only collectives are the barrier and the max-over-ranks of the
elapsed time.  These run here with the gloo backend, world_size 2.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    bench.init_dist(world, "gloo")
    dev = torch.device("cpu")
    bench.barrier(dev)
    got = bench.reduce_max(10.0 + 3.0 * rank, dev)      # rank 1 is the slow one
    seeds = [bench.rank_seed(1000, r) for r in range(world)]
    q.put((rank, got, bench.dist_env(), seeds[rank], bench.rank_units(5, world)))
    bench.barrier(dev)
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks_max_and_seeds():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, env, seed, units in res:
        assert got == 13.0                      # max over ranks, seen by every rank
        assert env == (rank, world, rank)
        assert units == 10                      # value counts the units of all ranks
    assert res[0][3] != res[1][3]               # independent problems per rank
    assert res[0][3] == 1000                    # rank 0 reproduces the single-GPU run


def test_single_process_reduce_is_identity():
    import bench
    assert bench.reduce_max(4.5, torch.device("cpu")) == 4.5
    assert bench.rank_seed(7, 0) == 7
