"""World-size-2 gloo checks of the multi-rank host logic (CPU only).

Each rank computes its shard of the (b, kv head) units and a fake per-rank
time; the union of the shards must be the whole layer exactly once, the
max-over-ranks reduction must return the slowest rank's time, and every rank
must take the same collective steps.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    from block_sparse_long_sm_b200.shard import max_over_ranks, shard_units
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    mine = shard_units(4, 8, world, rank)
    gathered = [None] * world
    dist.all_gather_object(gathered, mine)
    t = max_over_ranks(10.0 + rank)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, gathered, t))


@pytest.mark.parametrize("world", [2])
def test_two_rank_sharding_and_max_timing(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, gathered, t in results:
        flat = [u for shard in gathered for u in shard]
        assert flat == [(b, g) for b in range(4) for g in range(8)]
        assert t == 10.0 + world - 1
