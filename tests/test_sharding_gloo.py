"""Multi-rank host logic of the data-parallel path, on CPU with gloo (world size 2)."""

import os

import numpy as np
import torch.multiprocessing as mp

from generative_recommender_sequence_b200.sharding import (attention_cost, contiguous_users,
                                                           shard_users)


def test_shard_users_covers_every_user_once_and_balances():
    rng = np.random.default_rng(0)
    L = np.clip(rng.zipf(1.2, size=64), 64, 16384)
    for world in (1, 2, 4, 8):
        parts = shard_users(L, world)
        allu = np.concatenate(parts)
        assert sorted(allu.tolist()) == list(range(len(L)))
        loads = [attention_cost(L[p]).sum() for p in parts]
        # greedy LPT: no rank exceeds the mean by more than the largest single user
        assert max(loads) <= np.mean(loads) + attention_cost(L).max() + 1e-6


def test_contiguous_users_partition():
    for world in (1, 3, 8):
        parts = [contiguous_users(40, r, world) for r in range(world)]
        assert np.array_equal(np.concatenate(parts), np.arange(40))


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from generative_recommender_sequence_b200.sharding import (global_step_time, global_units,
                                                               shard_users)
    L = [100, 5000, 300, 16384, 64, 64, 2048, 900]
    mine = shard_users(L, world)[rank]
    other = shard_users(L, world)
    t = global_step_time(0.5 + rank)               # the slowest rank decides
    u = global_units(float(len(mine)))             # units add up over ranks
    q.put((rank, mine.tolist(), [p.tolist() for p in other], t, u))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_shards_and_reduce_time_and_units():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (r0, mine0, all0, t0, u0), (r1, mine1, all1, t1, u1) = res
    assert all0 == all1                       # every rank computes the same plan
    assert sorted(mine0 + mine1) == list(range(8)) and not set(mine0) & set(mine1)
    assert t0 == t1 == 1.5                    # max over ranks
    assert u0 == u1 == 8.0                    # sum over ranks
