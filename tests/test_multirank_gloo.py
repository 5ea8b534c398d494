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


def test_kv_head_sub_layers_tile_the_layer():
    # CPU: the ranks' sub-layers cover every kv head once, with their q heads,
    # and address disjoint, adjacent slices of the layer's tensors
    import block_sparse_long_sm_b200 as spa
    from block_sparse_long_sm_b200.shard import rank_sub_layer
    L = 4096
    for hq, hkv, world in ((32, 8, 2), (32, 8, 8), (64, 8, 4), (6, 3, 2)):
        p = spa.make_params(1, hq, hkv, L, mode="sale", sink=128, local=256, tau=0.01,
                            tau_per_head=[0.01 + 0.001 * h for h in range(hq)])
        prev_g, prev_h, prev_q = 0, 0, 0
        for r in range(world):
            sub = rank_sub_layer(p, world, r)
            assert (sub.g0, sub.h0, sub.q_off) == (prev_g, prev_h, prev_q)
            assert sub.params.heads_q == sub.h1 - sub.h0 == (sub.g1 - sub.g0) * (hq // hkv)
            assert sub.params.heads_kv == sub.g1 - sub.g0
            assert sub.params.mode == p.mode and sub.params.tau == p.tau
            assert [sub.params.tau_per_head[i] for i in range(sub.params.heads_q)] == \
                [p.tau_per_head[h] for h in range(sub.h0, sub.h1)]
            assert sub.kv_off == sub.g0 * L * 128 * 2 and sub.lse_off == sub.h0 * L * 4
            prev_g, prev_h, prev_q = sub.g1, sub.h1, sub.h1 * L * 128 * 2
        assert (prev_g, prev_h) == (hkv, hq)
