"""KV cache manager (LRU eviction to a pinned host tier, onboarding) on the GPU:
evicted users come back with bit-identical K/V and score like never evicted."""

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_common import assert_bf16_close, dev, magnitudes, storage, to_np

pytestmark = pytest.mark.gpu

H, D = 4, 128


def _kv(rng, n):
    return workloads._as_storage(rng.standard_normal((2, n, H, D)).astype(np.float32), "bf16")


def test_lru_eviction_offload_and_onboard_round_trip():
    import generative_recommender_sequence_b200 as hstu
    from generative_recommender_sequence_b200.kv_cache import KVCacheManager
    rng = np.random.default_rng(21)
    n_pages = 24
    table = hstu.KVTable(n_pages, H, D, max_users=8, max_pages_per_user=32,
                         free_order=rng.permutation(n_pages))
    mgr = KVCacheManager(table)
    sent = {}

    def request(users, n_new):
        kv = _kv(rng, int(sum(n_new)))
        off = workloads.offsets_from_lengths(np.array(n_new))
        mgr.append(users, n_new, storage(kv[0], "bf16"), storage(kv[1], "bf16"), dev(off))
        for b, u in enumerate(users):
            sent.setdefault(u, []).append(kv[:, off[b]:off[b + 1]])

    request([0, 1, 2], [200, 300, 150])          # 7 + 10 + 5 = 22 of 24 pages
    assert mgr.free == 2 and mgr.evicted == []
    request([3], [100])                          # needs 4: evicts user 0 (oldest; ties by id)
    assert mgr.evicted == [0] and 0 in mgr.host
    request([1], [10])                           # user 1 becomes most recent
    request([0], [40])                           # 0 comes back (8 pages with the new 40): evicts 2
    assert mgr.onboarded == [0] and mgr.evicted == [0, 2]
    torch.cuda.synchronize()
    assert table.status() == 0
    # every resident user's cache equals what was sent, bit for bit
    for u in (0, 1):
        lens = torch.empty(1, dtype=torch.int64, device="cuda")
        L = mgr.gpu_len[u]
        k = torch.empty((L, H, D), dtype=torch.bfloat16, device="cuda")
        v = torch.empty_like(k)
        table.lookup(dev(np.array([u], np.int64)), lens, None, k, v, dev(np.array([0, L], np.int64)), L)
        ref = np.concatenate(sent[u], axis=1)
        assert lens.item() == L == ref.shape[1]
        assert np.array_equal(k.cpu().float().numpy(), ref[0]) and np.array_equal(v.cpu().float().numpy(), ref[1])
    # candidates of the onboarded user score as over its full history
    nc = 16
    q, kc, vc = (workloads._as_storage(rng.standard_normal((nc, H, D)).astype(np.float32), "bf16")
                 for _ in range(3))
    pt = rng.normal(0, 0.1, 16).astype(np.float32)
    L = mgr.gpu_len[0]
    out = hstu.attn_cached_fwd(table, dev(np.array([0], np.int64)), storage(q, "bf16"),
                               dev(np.array([0, nc], np.int64)), nc, L, hstu.HSTU_MASK_CANDIDATES,
                               k_cand=storage(kc, "bf16"), v_cand=storage(vc, "bf16"),
                               pos_table=dev(pt), scale=1.0 / (L + nc))
    ref_kv = np.concatenate(sent[0], axis=1)
    ref = oracle.attn_candidates(ref_kv[0], ref_kv[1], np.array([0, L]), q, kc, vc, np.array([0, nc]),
                                 pos_table=pt, scale=1.0 / (L + nc))
    mag = magnitudes(oracle.attn_candidates, ref_kv[0], ref_kv[1], np.array([0, L]), q, kc, vc,
                     np.array([0, nc]), pos_table=pt, scale=1.0 / (L + nc))
    assert_bf16_close(to_np(out), ref, "onboarded user", mag=mag)
    table.close()


def test_multi_layer_eviction_and_onboarding_with_the_cached_block_step():
    """Per-layer caches of the cached block step under a pool that is too small:
    a user evicted from every layer (K/V offloaded to host memory) and brought
    back later gives, bit for bit, the results of the same requests served
    with a pool large enough that nothing is evicted."""
    import generative_recommender_sequence_b200 as hstu
    from generative_recommender_sequence_b200.kv_cache import KVCacheManager
    rng = np.random.default_rng(23)
    DM, L = 512, 2
    bf = lambda a: workloads._as_storage(np.asarray(a, np.float32), "bf16")
    w1 = [storage(bf(rng.normal(0, 0.02, (DM, 4 * DM))), "bf16") for _ in range(L)]
    w2 = [storage(bf(rng.normal(0, 0.02, (DM, DM))), "bf16") for _ in range(L)]
    pt = dev(rng.normal(0, 0.1, 16).astype(np.float32))
    requests = [([0, 1], [100, 150], 0), ([2], [40], 0), ([0], [10], 8)]
    xs = [(bf(rng.standard_normal((sum(n), DM))), bf(rng.standard_normal((len(u) * c, DM))))
          for u, n, c in requests]
    scale = 1.0 / 200

    def serve_all(n_pages):
        tables = [hstu.KVTable(n_pages, H, D, max_users=4, max_pages_per_user=16,
                               free_order=np.random.default_rng(3 + l).permutation(n_pages))
                  for l in range(L)]
        mgr = KVCacheManager(tables)
        outs = []
        for (users, n_new, n_c), (x_new, x_c) in zip(requests, xs):
            mgr.make_room(users, n_new)
            x = storage(np.concatenate([x_new, x_c]), "bf16")
            off = lambda n: dev(workloads.offsets_from_lengths(np.array(n)))
            max_cached = max(mgr.cached_length(u) + n for u, n in zip(users, n_new))
            hstu.block_cached_step(tables, dev(np.array(users, np.int64)), x, off(n_new), max(n_new),
                                   off([n_c] * len(users)) if n_c else None, n_c, max_cached, w1, w2,
                                   pos_table=pt, scale=scale, T_new=int(sum(n_new)))
            mgr.commit(users, n_new)
            outs.append(to_np(x))
        torch.cuda.synchronize()
        for t in tables:
            assert t.status() == 0
            t.close()
        return mgr, outs

    small, got = serve_all(10)
    assert small.evicted == [0, 1] and small.onboarded == [0]
    big, ref = serve_all(64)
    assert big.evicted == []
    for g, r in zip(got, ref):
        assert np.array_equal(g, r)
    assert hstu.last_device_error() == 0
