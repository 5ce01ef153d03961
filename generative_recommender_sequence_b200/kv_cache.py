"""KV cache manager: the paged GPU table plus a host tier, with LRU eviction.

Source: "NVIDIA Dynamo-Triton Gets End-to-End HSTU Generative Recommender
Workflow", section "What the workflow combines": the KV cache manager uses GPU
memory and host storage; the GPU cache is a paged table with lookup,
allocation, append and eviction, older users being evicted under an LRU-style
policy when space is tight; the exported path has cache-aware operations for
lookup, allocation, onboarding, appending and offloading.

This module is host-side policy only.  Every byte moves through the library's
kernels (hstu_kv_lookup's gather, hstu_kv_release, hstu_kv_alloc,
hstu_kv_append) and through copies ordered on the caller's stream:
  * offload  = gather a user's cached K/V on the device, copy it to pinned host
               memory, release the user's pages;
  * onboard  = copy the host K/V back to the device, alloc pages, append.
The host mirror of every user's cached length is exact because only this
manager changes the table while it is in use.
"""

from __future__ import annotations

from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import torch

from . import KVTable


def choose_victims(last_use: Dict[int, int], gpu_pages: Dict[int, int], protected: Iterable[int],
                   need_pages: int, free_pages: int) -> List[int]:
    """Least recently used users (outside `protected`, holding pages) whose
    release brings the free pages to at least `need_pages`; ties by user id.
    Raises if even releasing all of them is not enough."""
    if free_pages >= need_pages:
        return []
    keep = set(int(u) for u in protected)
    order = sorted((t, u) for u, t in last_use.items() if u not in keep and gpu_pages.get(u, 0) > 0)
    victims, got = [], free_pages
    for _, u in order:
        victims.append(u)
        got += gpu_pages[u]
        if got >= need_pages:
            return victims
    raise RuntimeError(f"KV cache: {need_pages} pages needed, at most {got} can be freed")


class KVCacheManager:
    """LRU eviction to a pinned host tier over one table or over the per-layer
    tables of a multi-layer cache.

    With several tables (one per layer, as hstu_block_cached_step uses them)
    every table holds the same users with the same cached lengths, so a user is
    evicted from, and brought back to, all layers together: its K/V of every
    layer goes to the host tier and its pages of every layer are released.
    All tables must have the same number of pages (their free counts then stay
    equal).

    Single table: ``append`` serves a request end to end (room, onboarding,
    alloc + append).  Several tables: ``make_room`` before the cached block step
    (which allocates and appends the new tokens itself) and ``commit`` after
    it."""

    def __init__(self, tables, offload: bool = True, device: str = "cuda"):
        self.tables: List[KVTable] = list(tables) if isinstance(tables, (list, tuple)) else [tables]
        if not self.tables or len({t.n_pages for t in self.tables}) != 1:
            raise ValueError("one or more tables, all with the same number of pages")
        self.table = self.tables[0]
        self.offload = offload
        self.device = device
        self.P = self.table.page_size
        self.clock = 0
        self.last_use: Dict[int, int] = {}
        self.gpu_len: Dict[int, int] = {}
        # host tier: user -> [(k, v) per layer]
        self.host: Dict[int, List[Tuple[torch.Tensor, torch.Tensor]]] = {}
        self.free = self.table.n_pages
        self.evicted: List[int] = []
        self.onboarded: List[int] = []

    def _pages(self, n: int) -> int:
        return -(-int(n) // self.P)

    def cached_length(self, user: int) -> int:
        if user in self.host:
            return int(self.host[user][0][0].shape[0])
        return self.gpu_len.get(user, 0)

    def _dev_i64(self, vals: Sequence[int]) -> torch.Tensor:
        return torch.tensor([int(v) for v in vals], dtype=torch.int64, device=self.device)

    def _offsets(self, lens: Sequence[int]) -> List[int]:
        out = [0]
        for n in lens:
            out.append(out[-1] + int(n))
        return out

    def _host_buffer(self, like: torch.Tensor) -> torch.Tensor:
        pin = torch.cuda.is_available() and like.is_cuda
        return torch.empty(like.shape, dtype=like.dtype, pin_memory=pin)

    def _offload(self, victims: List[int], stream=None):
        lens = [self.gpu_len.get(u, 0) for u in victims]
        users_t = self._dev_i64(victims)
        if self.offload and sum(lens) > 0:
            off = self._offsets(lens)
            off_t = self._dev_i64(off)
            per_layer = []
            for t in self.tables:
                k = torch.empty((off[-1], t.H, t.d), dtype=t.dtype, device=self.device)
                v = torch.empty_like(k)
                t.lookup(users_t, k_out=k, v_out=v, out_offsets=off_t, max_len=max(lens),
                         stream=stream)
                kh, vh = self._host_buffer(k), self._host_buffer(v)
                kh.copy_(k, non_blocking=True)
                vh.copy_(v, non_blocking=True)
                per_layer.append((kh, vh))
            for i, u in enumerate(victims):
                if lens[i] > 0:
                    self.host[u] = [(kh[off[i]:off[i + 1]], vh[off[i]:off[i + 1]])
                                    for kh, vh in per_layer]
        for t in self.tables:
            t.release(users_t, stream=stream)
        for u, n in zip(victims, lens):
            self.free += self._pages(n)
            self.gpu_len[u] = 0
        self.evicted.extend(victims)

    def _onboard(self, users: List[int], stream=None):
        lens = [int(self.host[u][0][0].shape[0]) for u in users]
        users_t = self._dev_i64(users)
        offs = self._offsets(lens)
        offs_t, lens_t = self._dev_i64(offs), self._dev_i64(lens)
        for layer, t in enumerate(self.tables):
            ks = [self.host[u][layer][0] for u in users]
            vs = [self.host[u][layer][1] for u in users]
            # pinned -> device copies on the stream that wrote the pinned buffers,
            # so they are ordered after the offload's device -> host copies (the
            # host side never reads those buffers)
            k = torch.empty((offs[-1],) + tuple(ks[0].shape[1:]), dtype=ks[0].dtype,
                            device=self.device)
            v = torch.empty_like(k)
            for i in range(len(users)):
                k[offs[i]:offs[i + 1]].copy_(ks[i], non_blocking=True)
                v[offs[i]:offs[i + 1]].copy_(vs[i], non_blocking=True)
            t.alloc(users_t, lens_t, stream=stream)
            t.append(users_t, k, v, offs_t, max(lens), stream=stream)
        for u, n in zip(users, lens):
            del self.host[u]
            self.gpu_len[u] = n
            self.free -= self._pages(n)
        self.onboarded.extend(users)

    def make_room(self, users: Sequence[int], n_new: Sequence[int], stream=None):
        """Before a request: evict least recently used users outside it (all
        layers, offloading their K/V) until the request's new pages fit, and
        bring the request's users back from the host tier (all layers)."""
        users = [int(u) for u in users]
        n_new = [int(n) for n in n_new]
        need = 0
        for u, n in zip(users, n_new):
            now = self.cached_length(u)
            resident = 0 if u in self.host else self._pages(self.gpu_len.get(u, 0))
            need += self._pages(now + n) - resident
        gpu_pages = {u: self._pages(n) for u, n in self.gpu_len.items()}
        victims = choose_victims(self.last_use, gpu_pages, users, need, self.free)
        if victims:
            self._offload(victims, stream)
        back = [u for u in users if u in self.host]
        if back:
            self._onboard(back, stream)

    def commit(self, users: Sequence[int], n_new: Sequence[int]):
        """After the request's new tokens were allocated and appended (in every
        table): record the lengths, free pages and recency."""
        self.clock += 1
        for u, n in zip(users, n_new):
            u, n = int(u), int(n)
            before = self._pages(self.gpu_len.get(u, 0))
            self.gpu_len[u] = self.gpu_len.get(u, 0) + n
            self.free -= self._pages(self.gpu_len[u]) - before
            self.last_use[u] = self.clock

    def append(self, users: Sequence[int], n_new: Sequence[int], k_new: torch.Tensor,
               v_new: torch.Tensor, new_offsets: torch.Tensor, users_dev: Optional[torch.Tensor] = None,
               n_new_dev: Optional[torch.Tensor] = None, stream=None):
        """One request on a single table: make room (evicting least recently used
        users outside the request, offloading them), bring back requested users
        from the host tier, then alloc and append the new tokens.  users / n_new:
        host lists.  All work, copies included, is ordered on `stream` (default:
        the current one)."""
        if len(self.tables) != 1:
            raise ValueError("append serves a single table; use make_room / commit per layer set")
        if stream is not None:
            with torch.cuda.stream(stream):
                return self.append(users, n_new, k_new, v_new, new_offsets, users_dev, n_new_dev)
        users = [int(u) for u in users]
        n_new = [int(n) for n in n_new]
        self.make_room(users, n_new)
        ut = users_dev if users_dev is not None else self._dev_i64(users)
        nt = n_new_dev if n_new_dev is not None else self._dev_i64(n_new)
        self.table.alloc(ut, nt, stream=stream)
        if max(n_new, default=0) > 0:
            self.table.append(ut, k_new, v_new, new_offsets, max(n_new), stream=stream)
        self.commit(users, n_new)
