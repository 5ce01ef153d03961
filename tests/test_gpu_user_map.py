"""Sparse user-id map on the GPU vs the sequential model: identical slots and
statuses; its slots drive the KV table directly."""

import numpy as np
import pytest
import torch

import workloads
from oracle.user_map import OK, OUT_OF_SLOTS, INVALID_ARG, UserMapOracle
from tests.gpu_common import dev, storage

pytestmark = pytest.mark.gpu


def test_random_lookups_inserts_erases_match_the_model():
    import generative_recommender_sequence_b200 as hstu
    rng = np.random.default_rng(17)
    n_slots = 40
    order = rng.permutation(n_slots)
    m = hstu.UserMap(n_slots, free_order=order)
    ref = UserMapOracle(n_slots, order)
    known = []
    for step in range(150):
        r = rng.random()
        if r < 0.45 or not known:       # fresh sparse ids, some repeated within the call
            ids = rng.integers(0, 2**62, size=int(rng.integers(1, 12)))
            if len(ids) > 2:
                ids[-1] = ids[0]
        elif r < 0.8:                   # mix of known and unknown
            ids = np.concatenate([rng.choice(known, size=3), rng.integers(0, 2**62, size=2)])
        else:
            ids = rng.choice(known, size=int(rng.integers(1, 5)))
        insert = rng.random() < 0.8
        if rng.random() < 0.25:
            m.erase(dev(ids.astype(np.int64)))
            assert m.status() == OK
            ref.erase(ids.tolist())
            continue
        got = m.lookup(dev(ids.astype(np.int64)), insert=insert)
        st = m.status()
        rs, rslots = ref.lookup(ids.tolist(), insert)
        assert st == rs, (step, st, rs)
        assert got.cpu().numpy().tolist() == rslots, step
        known = list(ref.slot)
    # running out of slots leaves the map unchanged
    free = len(ref.stack)
    fresh = rng.integers(2**62, 2**63 - 1, size=free + 1)
    got = m.lookup(dev(fresh.astype(np.int64)), insert=True)
    assert m.status() == OUT_OF_SLOTS == ref.lookup(fresh.tolist(), True)[0]
    assert np.all(got.cpu().numpy() == -1)
    probe = np.array(list(ref.slot)[:5] + [int(fresh[0])], dtype=np.int64)
    assert m.lookup(dev(probe), insert=False).cpu().numpy().tolist() == ref.lookup(probe.tolist(), False)[1]
    # a negative id is rejected
    m.lookup(dev(np.array([5, -3], np.int64)))
    assert m.status() == INVALID_ARG
    m.close()


def test_map_slots_name_kv_table_users():
    import generative_recommender_sequence_b200 as hstu
    rng = np.random.default_rng(18)
    m = hstu.UserMap(8)
    t = hstu.KVTable(64, 4, 128, max_users=8, max_pages_per_user=16)
    ids = dev(np.array([10**15 + 7, 42, 10**18], np.int64))
    slots = m.lookup(ids)
    n = np.array([70, 5, 33])
    kv = workloads._as_storage(rng.standard_normal((2, int(n.sum()), 4, 128)).astype(np.float32), "bf16")
    off = workloads.offsets_from_lengths(n)
    t.alloc(slots, dev(n.astype(np.int64)))
    t.append(slots, storage(kv[0], "bf16"), storage(kv[1], "bf16"), dev(off), int(n.max()))
    lens = torch.empty(3, dtype=torch.int64, device="cuda")
    # the same ids in another order reach the same cached users
    again = m.lookup(dev(np.array([42, 10**18, 10**15 + 7], np.int64)), insert=False)
    t.lookup(again, lens)
    assert t.status() == 0 and m.status() == 0
    assert lens.cpu().numpy().tolist() == [5, 33, 70]
    # evict one id: slot back to the map, pages back to the table
    gone = dev(np.array([42], np.int64))
    t.release(m.lookup(gone, insert=False))
    m.erase(gone)
    assert m.lookup(gone, insert=False).cpu().tolist() == [-1]
    assert t.status() == 0 and m.status() == 0
    t.close()
    m.close()
