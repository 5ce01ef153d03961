"""One-call serving step of the KV table (alloc + append + lookup rows, all or
nothing) against the sequential oracle: page ids, lengths, page tables, pool bytes."""

import numpy as np
import pytest
import torch

import workloads
from oracle.kv import INVALID_ARG, OK, OUT_OF_PAGES, KVTableOracle
from tests.gpu_common import dev, storage
from tests.test_gpu_kv import table_pool

pytestmark = pytest.mark.gpu

H, D, PPU = 4, 128, 64


def _kv(rng, n_tokens):
    x = rng.standard_normal((2, max(int(n_tokens), 1), H, D)).astype(np.float32)
    return workloads._as_storage(x, "bf16")


def _check_everything(t, ref, U):
    """Full lookup (with the K/V gather) and the pool bytes against the oracle."""
    users = np.arange(U)
    rl, rt, rk, rv = ref.lookup(users.tolist(), PPU)
    lens = torch.empty(U, dtype=torch.int64, device="cuda")
    table = torch.empty((U, PPU), dtype=torch.int32, device="cuda")
    out_off = workloads.offsets_from_lengths(rl)
    ko = torch.empty((max(int(out_off[-1]), 1), H, D), dtype=torch.bfloat16, device="cuda")
    vo = torch.empty_like(ko)
    t.lookup(dev(users.astype(np.int64)), lens, table, ko, vo, dev(out_off), int(max(rl.max(), 1)))
    assert t.status() == OK
    assert np.array_equal(lens.cpu().numpy(), rl)
    assert np.array_equal(table.cpu().numpy(), rt)
    T = int(out_off[-1])
    assert np.array_equal(ko[:T].cpu().view(torch.int16).numpy().view(np.uint16), rk)
    assert np.array_equal(vo[:T].cpu().view(torch.int16).numpy().view(np.uint16), rv)
    assert np.array_equal(table_pool(t)[:-1], ref.pool)


def _step(t, users, n, kv, max_new, max_pages=PPU):
    B = len(users)
    lens = torch.full((B,), -7, dtype=torch.int64, device="cuda")
    table = torch.full((B, max_pages), -7, dtype=torch.int32, device="cuda")
    off = workloads.offsets_from_lengths(np.asarray(n, np.int64))
    t.step(dev(np.asarray(users, np.int64)), storage(kv[0], "bf16"), storage(kv[1], "bf16"), dev(off),
           max_new, lens, table)
    return t.status(), lens.cpu().numpy(), table.cpu().numpy(), off


@pytest.mark.parametrize("two_launch", [False, True], ids=["one-launch", "two-launch"])
def test_kv_step_matches_alloc_append_lookup(two_launch):
    """Random steps (empty appends, page-boundary crossings, users that need no
    new page) on one table: every step's lookup rows and the final table equal
    the oracle's alloc, append and lookup in sequence, bit for bit."""
    import generative_recommender_sequence_b200 as hstu
    rng = np.random.default_rng(21 + int(two_launch))
    U = 100 if two_launch else 64
    n_pages = 1800 if two_launch else 700
    order = rng.permutation(n_pages)
    t = hstu.KVTable(n_pages, H, D, max_users=U, max_pages_per_user=PPU, free_order=order)
    ref = KVTableOracle(n_pages, 32, H, D, U, PPU, order)
    for step in range(7):
        if two_launch:
            B = int(rng.integers(65, U + 1))
        else:
            B = U if step == 3 else int(rng.integers(1, 9))   # 64 users: the one-launch limit
        users = rng.permutation(U)[:B]
        n = rng.integers(0, 80, size=B)
        n[rng.random(B) < 0.2] = 0
        kv = _kv(rng, n.sum())
        max_new = int(n.max()) + int(rng.integers(0, 3))      # a loose bound is fine
        status, lens, table, off = _step(t, users, n, kv, max_new)
        rs, _ = ref.alloc(users.tolist(), n.tolist())
        assert rs == OK and status == OK
        assert ref.append(users.tolist(), kv[0][: int(n.sum())], kv[1][: int(n.sum())], off) == OK
        rl, rt, _, _ = ref.lookup(users.tolist(), PPU, gather=False)
        assert np.array_equal(lens, rl)
        assert np.array_equal(table, rt)
    _check_everything(t, ref, U)
    t.close()


@pytest.mark.parametrize("two_launch", [False, True], ids=["one-launch", "two-launch"])
def test_kv_step_errors_change_nothing(two_launch):
    """Duplicate or out-of-range users, a count above max_new, and a page
    shortage each record their status and leave the table exactly as it was;
    the lookup rows show the unchanged table."""
    import generative_recommender_sequence_b200 as hstu
    rng = np.random.default_rng(5)
    U = 90 if two_launch else 10
    B = 70 if two_launch else 6
    n_pages = 260 if two_launch else 24
    order = rng.permutation(n_pages)
    t = hstu.KVTable(n_pages, H, D, max_users=U, max_pages_per_user=PPU, free_order=order)
    ref = KVTableOracle(n_pages, 32, H, D, U, PPU, order)
    users = rng.permutation(U)[:B]
    n = rng.integers(1, 40, size=B)
    kv = _kv(rng, n.sum())
    status, _, _, off = _step(t, users, n, kv, int(n.max()))
    assert status == OK
    assert ref.alloc(users.tolist(), n.tolist())[0] == OK
    assert ref.append(users.tolist(), kv[0][: int(n.sum())], kv[1][: int(n.sum())], off) == OK
    rl, rt, _, _ = ref.lookup(users.tolist(), PPU, gather=False)

    # a user listed twice
    dup = users.copy()
    dup[-1] = dup[0]
    status, lens, table, _ = _step(t, dup, n, kv, int(n.max()))
    assert status == INVALID_ARG
    assert np.array_equal(lens[:-1], rl[:-1]) and np.array_equal(table[:-1], rt[:-1])
    # a count above max_new
    status, lens, table, _ = _step(t, users, n, kv, int(n.max()) - 1)
    assert status == INVALID_ARG
    assert np.array_equal(lens, rl) and np.array_equal(table, rt)
    # an out-of-range user id: its row is empty, the others unchanged
    bad = users.copy()
    bad[1] = U + 3
    status, lens, table, _ = _step(t, bad, n, kv, int(n.max()))
    assert status == INVALID_ARG
    assert lens[1] == 0 and np.all(table[1] == -1)
    keep = np.arange(B) != 1
    assert np.array_equal(lens[keep], rl[keep]) and np.array_equal(table[keep], rt[keep])
    # more pages than the free stack holds
    big = np.full(B, 32 * 5, np.int64)     # at least 5 new pages per user
    kv_big = _kv(rng, big.sum())
    status, lens, table, _ = _step(t, users, big, kv_big, int(big.max()))
    assert status == OUT_OF_PAGES
    assert ref.alloc(users.tolist(), big.tolist())[0] == OUT_OF_PAGES
    assert np.array_equal(lens, rl) and np.array_equal(table, rt)
    _check_everything(t, ref, U)
    # the table still works after the failures
    status, lens, table, off = _step(t, users, n, kv, int(n.max()))
    assert status == OK
    assert ref.alloc(users.tolist(), n.tolist())[0] == OK
    assert ref.append(users.tolist(), kv[0][: int(n.sum())], kv[1][: int(n.sum())], off) == OK
    _check_everything(t, ref, U)
    t.close()


def test_kv_step_graph_replay():
    """A captured step replayed several times: each replay is a fresh step (the
    grid-wide completion counter returns to zero every time)."""
    import generative_recommender_sequence_b200 as hstu
    rng = np.random.default_rng(8)
    U, B, n_pages = 16, 8, 400
    order = rng.permutation(n_pages)
    t = hstu.KVTable(n_pages, H, D, max_users=U, max_pages_per_user=PPU, free_order=order)
    ref = KVTableOracle(n_pages, 32, H, D, U, PPU, order)
    users = rng.permutation(U)[:B]
    n = rng.integers(10, 70, size=B)
    kv = _kv(rng, n.sum())
    off = workloads.offsets_from_lengths(n)
    u_d, off_d = dev(users.astype(np.int64)), dev(off)
    k_d, v_d = storage(kv[0], "bf16"), storage(kv[1], "bf16")
    lens = torch.empty(B, dtype=torch.int64, device="cuda")
    table = torch.empty((B, PPU), dtype=torch.int32, device="cuda")
    t.step(u_d, k_d, v_d, off_d, int(n.max()), lens, table)   # warm-up, outside the graph
    torch.cuda.synchronize()
    assert t.status() == OK
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        t.step(u_d, k_d, v_d, off_d, int(n.max()), lens, table)
    torch.cuda.synchronize()
    for _ in range(4):   # the warm-up call plus four replays: five steps
        g.replay()
        torch.cuda.synchronize()
    assert t.status() == OK
    for _ in range(5):
        assert ref.alloc(users.tolist(), n.tolist())[0] == OK
        assert ref.append(users.tolist(), kv[0][: int(n.sum())], kv[1][: int(n.sum())], off) == OK
    rl, rt, _, _ = ref.lookup(users.tolist(), PPU, gather=False)
    assert np.array_equal(lens.cpu().numpy(), rl)
    assert np.array_equal(table.cpu().numpy(), rt)
    _check_everything(t, ref, U)
    del g
    t.close()
