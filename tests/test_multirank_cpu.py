"""The N > 1 host path of bench.py on CPU with gloo, world size 2.

The verification step shards over sequences / candidates (independent batch
entries), so ranks share no data-path collective: each rank draws its own
batch from a distinct seed, and the only collectives are the timing barrier
and the max-over-ranks reduction of the step time.
"""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from speculative_verification_cover_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        spec = W.TINY_F32
        seed = bench.shard_seed(spec, rank)
        x = W.make_inputs(spec, "cpu", seed=seed)
        bench.barrier(world)
        # rank r reports a step time of 1 + r ms: the job time is the slowest rank's
        got = bench.max_over_ranks([1.0 + rank, 10.0 * (world - rank)], world)
        q.put((rank, seed, float(x["q"].sum()), got))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_ranks_shard_and_max_reduce():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    (r0, s0, sum0, got0), (r1, s1, sum1, got1) = res
    assert s0 != s1 and sum0 != sum1          # independent batches per rank
    assert got0 == got1 == [2.0, 20.0]        # max over ranks, identical everywhere
