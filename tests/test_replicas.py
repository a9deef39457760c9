"""N > 1 host logic of the replica runs, on CPU with gloo (world size 2):
disjoint head ownership, max-over-ranks timing and the whole-job value."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from clustered_block_sparse_b200 import replicas


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        heads = replicas.rank_heads(rank, 3)
        slowest = replicas.max_over_ranks(10.0 + 5.0 * rank)
        q.put((rank, heads, slowest))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_partition_heads_and_take_the_slowest():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    heads = [h for _, hs, _ in out for h in hs]
    assert heads == list(range(6))  # disjoint and covering
    assert all(s == 15.0 for _, _, s in out)  # every rank sees the slowest
    assert replicas.job_ms_per_layer(15.0, world) == 7.5


def test_single_process_needs_no_group():
    assert replicas.max_over_ranks(3.5) == 3.5
    assert replicas.rank_heads(0, 2) == [0, 1]
    with pytest.raises(ValueError):
        replicas.job_ms_per_layer(1.0, 0)
