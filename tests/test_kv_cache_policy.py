"""Host-side LRU victim choice of the KV cache manager (no GPU)."""

import pytest

from generative_recommender_sequence_b200.kv_cache import choose_victims


def test_nothing_evicted_when_the_request_fits():
    assert choose_victims({1: 5, 2: 3}, {1: 4, 2: 4}, [9], need_pages=3, free_pages=3) == []


def test_least_recently_used_first_until_enough():
    last = {10: 7, 11: 2, 12: 5, 13: 1}
    pages = {10: 3, 11: 2, 12: 4, 13: 1}
    # 13 (t=1) then 11 (t=2) then 12 (t=5): 1 + 2 + 4 = 7 >= 8 - 1
    assert choose_victims(last, pages, [10], need_pages=8, free_pages=1) == [13, 11, 12]


def test_request_users_and_empty_users_are_never_victims():
    last = {1: 1, 2: 2, 3: 3}
    pages = {1: 0, 2: 5, 3: 5}
    assert choose_victims(last, pages, [2], need_pages=5, free_pages=1) == [3]


def test_ties_break_by_user_id_and_impossible_requests_raise():
    assert choose_victims({5: 1, 4: 1}, {5: 1, 4: 1}, [], need_pages=1, free_pages=0) == [4]
    with pytest.raises(RuntimeError):
        choose_victims({1: 1}, {1: 2}, [], need_pages=10, free_pages=3)


class _FakeTable:
    """Host stand-in for one layer's table: keeps each user's K/V rows (tagged
    with the layer) and records the calls the manager makes."""

    def __init__(self, layer, n_pages=10, H=1, d=2):
        import torch
        self.layer, self.n_pages, self.H, self.d = layer, n_pages, H, d
        self.page_size, self.dtype = 32, torch.float32
        self.rows = {}
        self.calls = []

    def lookup(self, users, k_out=None, v_out=None, out_offsets=None, max_len=0, stream=None):
        off = out_offsets.tolist()
        for i, u in enumerate(users.tolist()):
            k, v = self.rows[u]
            k_out[off[i]:off[i + 1]] = k
            v_out[off[i]:off[i + 1]] = v
        self.calls.append(("lookup", users.tolist()))

    def release(self, users, stream=None):
        for u in users.tolist():
            self.rows.pop(u, None)
        self.calls.append(("release", users.tolist()))

    def alloc(self, users, n_new, stream=None):
        self.calls.append(("alloc", users.tolist(), n_new.tolist()))

    def append(self, users, k, v, offsets, max_new, stream=None):
        import torch
        off = offsets.tolist()
        for i, u in enumerate(users.tolist()):
            old = self.rows.get(u, (torch.zeros((0, self.H, self.d)),) * 2)
            self.rows[u] = (torch.cat([old[0], k[off[i]:off[i + 1]]]),
                            torch.cat([old[1], v[off[i]:off[i + 1]]]))
        self.calls.append(("append", users.tolist()))


def test_multi_layer_manager_evicts_and_onboards_every_layer_together():
    import torch
    from generative_recommender_sequence_b200.kv_cache import KVCacheManager
    tables = [_FakeTable(l) for l in range(3)]
    mgr = KVCacheManager(tables, device="cpu")

    def serve(users, n_new):
        mgr.make_room(users, n_new)
        # what the cached block step does per layer: alloc + append the new rows
        for t in tables:
            t.alloc(torch.tensor(users), torch.tensor(n_new))
            rows = [torch.full((n, 1, 2), 100.0 * t.layer + u) for u, n in zip(users, n_new)]
            off = torch.tensor([0] + list(torch.tensor(n_new).cumsum(0).tolist()))
            t.append(torch.tensor(users), torch.cat(rows), -torch.cat(rows), off, max(n_new))
        mgr.commit(users, n_new)

    serve([0, 1], [100, 150])        # 4 + 5 of 10 pages
    serve([2], [40])                 # needs 2: evicts user 0 from every layer
    assert mgr.evicted == [0] and 0 in mgr.host and len(mgr.host[0]) == 3
    for l, t in enumerate(tables):
        assert 0 not in t.rows and t.calls[-3] == ("release", [0])
        assert torch.equal(mgr.host[0][l][0], torch.full((100, 1, 2), 100.0 * l))
    serve([0], [10])                 # 0 comes back: every layer gets its own rows again
    assert mgr.onboarded == [0] and mgr.evicted == [0, 1]
    for l, t in enumerate(tables):
        k, v = t.rows[0]
        assert k.shape[0] == 110 and torch.equal(k[:100], torch.full((100, 1, 2), 100.0 * l))
        assert torch.equal(v, -k)
    # every layer saw the same sequence of operations on the same users
    ops = [[c[:2] for c in t.calls] for t in tables]
    assert ops[0] == ops[1] == ops[2]
    # resident: user 0 (110 tokens, 4 pages) and user 2 (40 tokens, 2 pages)
    assert mgr.free == 10 - 4 - 2 and mgr.cached_length(1) == 150 and 1 in mgr.host


def test_multi_layer_manager_needs_equal_pools():
    from generative_recommender_sequence_b200.kv_cache import KVCacheManager
    with pytest.raises(ValueError):
        KVCacheManager([_FakeTable(0, n_pages=10), _FakeTable(1, n_pages=12)], device="cpu")
