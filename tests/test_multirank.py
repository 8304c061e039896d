"""The benchmark's multi-rank plumbing on CPU with gloo (world size 2): each rank draws its own
batch (weak scaling), and timings are reduced with max over ranks, bytes with a sum."""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    try:
        w, r, _ = bench.dist_env()
        assert (w, r) == (world, rank)
        bench.init_dist(world, "gloo")
        times = [10.0 + rank, 3.0 - rank]
        mx = bench.max_over_ranks(times, world, "cpu")
        sm = bench.sum_over_ranks([100.0 * (rank + 1)], world, "cpu")
        seeds = bench.shard_seeds(5, world)
        q.put((rank, mx, sm, seeds))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:          # surface the failure to the parent
        q.put((rank, repr(e), None, None))


def test_two_rank_reductions():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, sm, seeds in res:
        assert mx == [11.0, 3.0], mx
        assert sm == [300.0]
        assert len(set(seeds)) == 2 and seeds[rank] == 5 + 1000 * rank
