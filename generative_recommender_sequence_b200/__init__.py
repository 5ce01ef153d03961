"""B200-native HSTU attention hot path (jagged SiLU attention, paged KV table,
cached candidate scoring, HSTU block stack).

Python binding of the C ABI in ``include/hstu.h``: each function checks and
marshals its arguments (device torch tensors, the current CUDA stream) and calls
the CUDA library.  Nothing here computes; nothing falls back to the CPU.
"""

from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import torch

from . import _lib
from ._lib import (HSTU_BF16, HSTU_ERR_INVALID_ARG, HSTU_F32, HSTU_MASK_CANDIDATES,
                   HSTU_MASK_CAUSAL_SUFFIX, HstuError, HstuRab, check, declared_symbols, load)

__all__ = ["attn_fwd", "attn_cached_fwd", "attn_beam_decode", "KVTable", "UserMap", "block_fwd", "block_cached_step",
           "block_cached_workspace_size", "HstuError", "load",
           "declared_symbols", "device_check", "last_device_error",
           "HSTU_MASK_CANDIDATES", "HSTU_MASK_CAUSAL_SUFFIX"]


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA device tensors")
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return HSTU_BF16
    if t.dtype == torch.float32:
        return HSTU_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def _rab(pos_table=None, time_table=None, timestamps=None) -> Optional[HstuRab]:
    if pos_table is None and time_table is None:
        return None
    _need_cuda(pos_table, time_table, timestamps)
    r = HstuRab()
    r.pos_table = _ptr(pos_table)
    r.n_pos_buckets = 0 if pos_table is None else pos_table.numel()
    r.time_table = _ptr(time_table)
    r.n_time_buckets = 0 if time_table is None else time_table.numel()
    r.timestamps = _ptr(timestamps)
    return r


def device_check():
    check("hstu_device_check", load().hstu_device_check())


def last_device_error(stream=None) -> int:
    return load().hstu_last_device_error(_stream(stream))


def wait_timeout_selftest(timeout_us: int = 20000, stream=None) -> None:
    """Run the bounded-wait self test: a GPU wait that nothing completes gives up
    after timeout_us and records HSTU_ERR_TIMEOUT for last_device_error()."""
    check("hstu_wait_timeout_selftest", load().hstu_wait_timeout_selftest(int(timeout_us), _stream(stream)))


def attn_fwd(q, k, v, seq_offsets, max_len: int, pos_table=None, time_table=None, timestamps=None,
             scale: float = 1.0, out=None, stream=None) -> torch.Tensor:
    """Jagged causal HSTU attention; q, k, v: [T, H, d] (bf16 or fp32), seq_offsets int64 [B+1]."""
    _need_cuda(q, k, v, seq_offsets)
    T, H, d = q.shape
    if out is None:
        out = torch.empty((T, H, v.shape[2]), dtype=q.dtype, device=q.device)
    _need_cuda(out)
    rab = _rab(pos_table, time_table, timestamps)
    st = load().hstu_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), seq_offsets.numel() - 1,
                              int(max_len), T, H, d, v.shape[2], _dtype_code(q),
                              ctypes.byref(rab) if rab else None, float(scale), _ptr(out),
                              _stream(stream))
    check("hstu_attn_fwd", st)
    return out


class KVTable:
    """Paged KV data table (pool, free stack, per-user page lists) on the current device."""

    def __init__(self, n_pages: int, H: int, d: int, dtype=torch.bfloat16, max_users: int = 1024,
                 max_pages_per_user: int = 1024, free_order: Optional[Sequence[int]] = None,
                 page_size: int = 32):
        self.lib = load()
        self.n_pages, self.H, self.d, self.page_size = n_pages, H, d, page_size
        self.dtype = dtype
        self.max_users, self.max_ppu = max_users, max_pages_per_user
        handle = ctypes.c_void_p()
        order = None
        if free_order is not None:
            arr = (ctypes.c_int32 * n_pages)(*[int(x) for x in free_order])
            order = ctypes.cast(arr, ctypes.c_void_p)
        st = self.lib.hstu_kv_table_create(n_pages, page_size, H, d, _dtype_code(torch.empty(0, dtype=dtype)),
                                           max_users, max_pages_per_user, order,
                                           ctypes.byref(handle))
        check("hstu_kv_table_create", st)
        self.handle = handle

    def close(self):
        if getattr(self, "handle", None):
            self.lib.hstu_kv_table_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def status(self, stream=None) -> int:
        return self.lib.hstu_kv_table_status(self.handle, _stream(stream))

    def storage(self):
        """Device pointers: (pool, page_lists, lengths, free_stack, free_top)."""
        ptrs = [ctypes.c_void_p() for _ in range(5)]
        check("hstu_kv_table_info", self.lib.hstu_kv_table_info(self.handle, *[ctypes.byref(p) for p in ptrs]))
        return tuple(p.value for p in ptrs)

    def alloc(self, users, n_new, page_ids_out=None, stream=None):
        _need_cuda(users, n_new, page_ids_out)
        cap = 0 if page_ids_out is None else page_ids_out.numel()
        st = self.lib.hstu_kv_alloc(self.handle, _ptr(users), _ptr(n_new), users.numel(),
                                    _ptr(page_ids_out), cap, _stream(stream))
        check("hstu_kv_alloc", st)

    def append(self, users, k_new, v_new, new_offsets, max_new: int, stream=None):
        _need_cuda(users, k_new, v_new, new_offsets)
        st = self.lib.hstu_kv_append(self.handle, _ptr(users), _ptr(k_new), _ptr(v_new),
                                     _ptr(new_offsets), users.numel(), int(max_new), _stream(stream))
        check("hstu_kv_append", st)

    def step(self, users, k_new, v_new, new_offsets, max_new: int, cached_len_out=None,
             page_table_out=None, stream=None):
        """alloc + append + lookup rows of one serving step, all or nothing (hstu_kv_step)."""
        _need_cuda(users, k_new, v_new, new_offsets, cached_len_out, page_table_out)
        max_pages = 0 if page_table_out is None else page_table_out.shape[-1]
        st = self.lib.hstu_kv_step(self.handle, _ptr(users), _ptr(k_new), _ptr(v_new), _ptr(new_offsets),
                                   users.numel(), int(max_new), _ptr(cached_len_out),
                                   _ptr(page_table_out), max_pages, _stream(stream))
        check("hstu_kv_step", st)

    def release(self, users, stream=None):
        """Evict whole users: every page of each listed user returns to the free stack."""
        _need_cuda(users)
        check("hstu_kv_release", self.lib.hstu_kv_release(self.handle, _ptr(users), users.numel(),
                                                          _stream(stream)))

    def lookup(self, users, cached_len_out=None, page_table_out=None, k_out=None, v_out=None,
               out_offsets=None, max_len: int = 0, stream=None):
        _need_cuda(users, cached_len_out, page_table_out, k_out, v_out, out_offsets)
        max_pages = 0 if page_table_out is None else page_table_out.shape[-1]
        st = self.lib.hstu_kv_lookup(self.handle, _ptr(users), users.numel(), _ptr(cached_len_out),
                                     _ptr(page_table_out), max_pages, _ptr(k_out), _ptr(v_out),
                                     _ptr(out_offsets), int(max_len), _stream(stream))
        check("hstu_kv_lookup", st)

    def workspace_size(self, B: int, total_q: int, max_q: int, max_cached: int, mask_mode: int) -> int:
        return self.lib.hstu_attn_cached_workspace_size(self.handle, B, total_q, max_q, max_cached,
                                                        mask_mode)


class UserMap:
    """Sparse int64 user ids -> dense KV-table slots (hstu_user_map_* in include/hstu.h)."""

    def __init__(self, n_slots: int, free_order: Optional[Sequence[int]] = None):
        self.lib = load()
        self.n_slots = n_slots
        handle = ctypes.c_void_p()
        order = None
        if free_order is not None:
            arr = (ctypes.c_int32 * n_slots)(*[int(x) for x in free_order])
            order = ctypes.cast(arr, ctypes.c_void_p)
        check("hstu_user_map_create", self.lib.hstu_user_map_create(n_slots, order, ctypes.byref(handle)))
        self.handle = handle

    def close(self):
        if getattr(self, "handle", None):
            self.lib.hstu_user_map_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def lookup(self, ids, insert: bool = True, out=None, stream=None) -> torch.Tensor:
        _need_cuda(ids, out)
        if out is None:
            out = torch.empty(ids.numel(), dtype=torch.int64, device=ids.device)
        check("hstu_user_map_lookup", self.lib.hstu_user_map_lookup(
            self.handle, _ptr(ids), ids.numel(), 1 if insert else 0, _ptr(out), _stream(stream)))
        return out

    def erase(self, ids, stream=None):
        _need_cuda(ids)
        check("hstu_user_map_erase", self.lib.hstu_user_map_erase(self.handle, _ptr(ids), ids.numel(),
                                                                  _stream(stream)))

    def status(self, stream=None) -> int:
        return self.lib.hstu_user_map_status(self.handle, _stream(stream))


def attn_cached_fwd(table: KVTable, users, q, q_offsets, max_q: int, max_cached: int,
                    mask_mode: int, k_cand=None, v_cand=None, pos_table=None, scale: float = 1.0,
                    out=None, workspace=None, stream=None) -> torch.Tensor:
    """Attention whose history K/V is read from ``table`` page by page (see hstu.h)."""
    _need_cuda(users, q, q_offsets, k_cand, v_cand, pos_table)
    if out is None:
        out = torch.empty_like(q)
    B = users.numel()
    total_q = q.shape[0]
    need = table.workspace_size(B, total_q, max_q, max_cached, mask_mode)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    rab = _rab(pos_table)
    st = table.lib.hstu_attn_cached_fwd(
        table.handle, _ptr(users), B, _ptr(q), _ptr(k_cand), _ptr(v_cand), _ptr(q_offsets),
        total_q, int(max_q), int(max_cached), int(mask_mode), ctypes.byref(rab) if rab else None,
        float(scale), _ptr(out), _ptr(workspace) if need else None,
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream))
    check("hstu_attn_cached_fwd", st)
    return out


def block_workspace_size(T: int, d_model: int, H: int, dh: int) -> int:
    return load().hstu_block_workspace_size(T, d_model, H, dh)


def block_fwd(x, seq_offsets, max_len: int, w_uvqk: Sequence[torch.Tensor],
              w_o: Sequence[torch.Tensor], pos_table=None, time_table=None, timestamps=None,
              scale: float = 1.0, ln_eps: float = 1e-5, H: int = 4, dh: int = 128,
              workspace=None, stream=None) -> torch.Tensor:
    """HSTU block stack, in place on x [T, d_model] bf16."""
    _need_cuda(x, seq_offsets, *w_uvqk, *w_o)
    T, dm = x.shape
    L = len(w_uvqk)
    need = block_workspace_size(T, dm, H, dh)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    w1 = (ctypes.c_void_p * L)(*[w.data_ptr() for w in w_uvqk])
    w2 = (ctypes.c_void_p * L)(*[w.data_ptr() for w in w_o])
    rab = _rab(pos_table, time_table, timestamps)
    st = load().hstu_block_fwd(_ptr(x), _ptr(seq_offsets), seq_offsets.numel() - 1, int(max_len), T,
                               L, dm, H, dh, ctypes.cast(w1, ctypes.c_void_p),
                               ctypes.cast(w2, ctypes.c_void_p), ctypes.byref(rab) if rab else None,
                               float(scale), float(ln_eps), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    check("hstu_block_fwd", st)
    return x


def _tables_array(tables: Sequence["KVTable"]):
    arr = (ctypes.c_void_p * len(tables))(*[t.handle.value for t in tables])
    return arr, ctypes.cast(arr, ctypes.c_void_p)


def block_cached_workspace_size(tables: Sequence["KVTable"], B: int, T_new: int, T_cand: int,
                                max_cand: int, max_cached: int, d_model: int = 512, H: int = 4,
                                dh: int = 128) -> int:
    arr, ptr = _tables_array(tables)
    return load().hstu_block_cached_workspace_size(ptr, len(tables), B, T_new, T_cand, max_cand,
                                                   max_cached, d_model, H, dh)


def block_cached_step(tables: Sequence["KVTable"], users, x, new_offsets, max_new: int,
                      cand_offsets, max_cand: int, max_cached: int, w_uvqk: Sequence[torch.Tensor],
                      w_o: Sequence[torch.Tensor], pos_table=None, scale: float = 1.0,
                      ln_eps: float = 1e-5, H: int = 4, dh: int = 128, T_new: Optional[int] = None,
                      workspace=None, stream=None) -> torch.Tensor:
    """KV-cached block step, in place on x = [new rows; candidate rows] (bf16).

    tables[l] caches layer l's K/V; new_offsets / cand_offsets: [B+1] int64 device
    (either may be None when there are no such rows).  T_new: number of new rows
    (default: all rows when cand_offsets is None, else x rows minus candidates,
    which needs cand_offsets on the host side as well - pass it explicitly)."""
    _need_cuda(users, x, new_offsets, cand_offsets, *w_uvqk, *w_o)
    T, dm = x.shape
    L = len(w_uvqk)
    if len(tables) != L or len(w_o) != L:
        raise ValueError("one table, one w_uvqk and one w_o per layer")
    if T_new is None:
        if cand_offsets is not None:
            raise ValueError("pass T_new when there are candidate rows")
        T_new = T
    T_cand = T - T_new
    B = users.numel()
    need = block_cached_workspace_size(tables, B, T_new, T_cand, max_cand, max_cached, dm, H, dh)
    if need == 0:
        raise HstuError("hstu_block_cached_workspace_size", HSTU_ERR_INVALID_ARG)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    arr, tptr = _tables_array(tables)
    w1 = (ctypes.c_void_p * L)(*[w.data_ptr() for w in w_uvqk])
    w2 = (ctypes.c_void_p * L)(*[w.data_ptr() for w in w_o])
    rab = _rab(pos_table, None, None)
    st = load().hstu_block_cached_step(
        tptr, L, _ptr(users), B, _ptr(x), _ptr(new_offsets), int(T_new), int(max_new),
        _ptr(cand_offsets), int(T_cand), int(max_cand), int(max_cached), dm, H, dh,
        ctypes.cast(w1, ctypes.c_void_p), ctypes.cast(w2, ctypes.c_void_p),
        ctypes.byref(rab) if rab else None, float(scale), float(ln_eps), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    check("hstu_block_cached_step", st)
    return x


def attn_beam_decode(table: KVTable, users, q, beam_offsets, max_beams: int, max_ctx: int, step: int,
                     beam_k, beam_v, beam_parent=None, pos_table=None, scale: float = 1.0, out=None,
                     workspace=None, stream=None) -> torch.Tensor:
    """Beam decode attention at step `step` over the shared context in `table`
    (hstu_attn_beam_decode in include/hstu.h).  beam_k / beam_v: [step+1, T_beam, H, 128]."""
    _need_cuda(users, q, beam_offsets, beam_k, beam_v, beam_parent, out)
    if out is None:
        out = torch.empty_like(q)
    T = q.shape[0]
    B = users.numel()
    need = load().hstu_attn_beam_decode_workspace_size(table.handle, B, T, int(max_beams),
                                                      int(max_ctx), int(step))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    rab = _rab(pos_table, None, None)
    st = load().hstu_attn_beam_decode(
        table.handle, _ptr(users), B, _ptr(q), _ptr(beam_offsets), T, int(max_beams), int(max_ctx),
        int(step), _ptr(beam_k), _ptr(beam_v), _ptr(beam_parent), ctypes.byref(rab) if rab else None,
        float(scale), _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream))
    check("hstu_attn_beam_decode", st)
    return out
