"""Sequential model of the paged GPU KV data table (test infrastructure only).

Source: "NVIDIA Dynamo-Triton Gets End-to-End HSTU Generative Recommender
Workflow", section "What the workflow combines": the GPU cache is a paged KV
data table with lookup, allocation, append (and eviction); "Déploiement de
recommandeurs génératifs avec NVIDIA Dynamo-Triton et HSTU", section "Comment
cela fonctionne": the HSTU attention kernel reads the cached data directly.

The pages give only the operation names.  The readings taken here:
* a pool of ``n_pages`` pages of ``page_size`` tokens; a page stores, for each
  of K and V and each head, ``page_size`` rows of ``d`` elements:
  ``pool[page, kv, head, slot, :]``;
* free pages form a LIFO stack initialised from ``free_order`` (top = last);
* ``alloc(users, n_new)``: user b needs ``ceil((len_b + n_new_b) / page_size)
  - held_b`` more pages (never negative); users take pages from the top of the
  stack in the order they are listed; if the total exceeds the free count the
  table is left unchanged and OUT_OF_PAGES is reported;
* ``append``: token t of user u goes to page ``pages[u][len_u // page_size]``,
  slot ``len_u % page_size``; then ``len_u`` grows by one;
* ``lookup``: cached length per user, the user's page list padded with -1, and
  optionally a jagged copy of the cached K/V.
* ``release(users)`` (eviction of whole users): every page of each listed user
  goes back on the free stack - users in the order listed, each user's pages
  from its last to its first, so its first page ends on top - and the user's
  length and page list become empty; duplicate or out-of-range users leave the
  table unchanged (INVALID_ARG).  The page bytes stay as they were.
Element values are stored as raw bit patterns (uint16 for bf16, uint32 for
fp32), so comparisons with the GPU pool are byte-exact.
"""

from __future__ import annotations

import numpy as np

OK, INVALID_ARG, OUT_OF_PAGES = 0, 1, 2


def to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """Raw storage bits of float32 arrays whose values are exact in ``dtype``."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x.view(np.uint32).copy()
    u = x.view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("value not representable in bf16")
    return (u >> 16).astype(np.uint16)


class KVTableOracle:
    def __init__(self, n_pages, page_size, H, d, max_users, max_pages_per_user, free_order,
                 dtype="bf16"):
        self.n_pages, self.P, self.H, self.d = int(n_pages), int(page_size), int(H), int(d)
        self.max_users, self.max_ppu = int(max_users), int(max_pages_per_user)
        self.dtype = dtype
        order = np.arange(n_pages) if free_order is None else np.asarray(free_order)
        assert sorted(order.tolist()) == list(range(n_pages)), "free order must be a permutation"
        self.stack = [int(p) for p in order]             # top = last element
        self.pages = [[] for _ in range(self.max_users)]
        self.length = [0] * self.max_users
        bits = np.uint16 if dtype == "bf16" else np.uint32
        self.pool = np.zeros((self.n_pages, 2, self.H, self.P, self.d), dtype=bits)

    @property
    def n_free(self):
        return len(self.stack)

    def _check_users(self, users):
        users = [int(u) for u in users]
        if len(set(users)) != len(users) or any(u < 0 or u >= self.max_users for u in users):
            return None
        return users

    def alloc(self, users, n_new):
        """Returns (status, new page ids concatenated in user order)."""
        users = self._check_users(users)
        if users is None:
            return INVALID_ARG, []
        need = []
        for u, n in zip(users, n_new):
            if n < 0:
                return INVALID_ARG, []
            want = -(-(self.length[u] + int(n)) // self.P)
            nb = max(0, want - len(self.pages[u]))
            if len(self.pages[u]) + nb > self.max_ppu:
                return INVALID_ARG, []
            need.append(nb)
        if sum(need) > len(self.stack):
            return OUT_OF_PAGES, []
        got = []
        for u, nb in zip(users, need):
            for _ in range(nb):
                p = self.stack.pop()
                self.pages[u].append(p)
                got.append(p)
        return OK, got

    def append(self, users, k_new, v_new, new_offsets):
        """Write the new tokens' K/V rows ([T_new, H, d] float arrays) into pages."""
        users = self._check_users(users)
        if users is None:
            return INVALID_ARG
        kb, vb = to_bits(k_new, self.dtype), to_bits(v_new, self.dtype)
        for b, u in enumerate(users):
            s, e = int(new_offsets[b]), int(new_offsets[b + 1])
            if self.length[u] + (e - s) > len(self.pages[u]) * self.P:
                return INVALID_ARG
        for b, u in enumerate(users):
            s, e = int(new_offsets[b]), int(new_offsets[b + 1])
            for t in range(s, e):
                pos = self.length[u]
                page = self.pages[u][pos // self.P]
                slot = pos % self.P
                self.pool[page, 0, :, slot, :] = kb[t]
                self.pool[page, 1, :, slot, :] = vb[t]
                self.length[u] += 1
        return OK

    def release(self, users):
        """Evict whole users: their pages return to the free stack."""
        users = self._check_users(users)
        if users is None:
            return INVALID_ARG
        for u in users:
            for p in reversed(self.pages[u]):
                self.stack.append(p)
            self.pages[u] = []
            self.length[u] = 0
        return OK

    def lookup(self, users, max_pages, gather=True):
        """(cached_len[B], page_table[B, max_pages] with -1 padding, k_bits, v_bits)."""
        users = [int(u) for u in users]
        lens = np.array([self.length[u] for u in users], dtype=np.int64)
        table = np.full((len(users), max_pages), -1, dtype=np.int32)
        for b, u in enumerate(users):
            n = min(len(self.pages[u]), max_pages)
            table[b, :n] = self.pages[u][:n]
        if not gather:
            return lens, table, None, None
        ks, vs = [], []
        for u in users:
            for pos in range(self.length[u]):
                page, slot = self.pages[u][pos // self.P], pos % self.P
                ks.append(self.pool[page, 0, :, slot, :])
                vs.append(self.pool[page, 1, :, slot, :])
        shape = (0, self.H, self.d)
        k = np.stack(ks) if ks else np.zeros(shape, self.pool.dtype)
        v = np.stack(vs) if vs else np.zeros(shape, self.pool.dtype)
        return lens, table, k, v
