"""ctypes binding of ``libhstu_b200.so`` (the C ABI in ``include/hstu.h``).

Argument marshalling only: every computation runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  There is no
fallback of any kind: if the library is missing or no sm_100 GPU is present the
calls raise.
"""

from __future__ import annotations

import ctypes
import os
import re
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhstu_b200.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "hstu.h")

HSTU_OK, HSTU_ERR_INVALID_ARG, HSTU_ERR_OUT_OF_PAGES, HSTU_ERR_CUDA, HSTU_ERR_UNSUPPORTED, \
    HSTU_ERR_TIMEOUT = range(6)
HSTU_F32, HSTU_BF16 = 0, 1
HSTU_MASK_CANDIDATES, HSTU_MASK_CAUSAL_SUFFIX = 0, 1

STATUS_NAMES = {0: "ok", 1: "invalid argument", 2: "out of KV pages", 3: "CUDA error",
                4: "unsupported configuration", 5: "device wait timed out"}


class HstuError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)} (status {status})")
        self.status = status


class HstuRab(ctypes.Structure):
    _fields_ = [("pos_table", ctypes.c_void_p), ("n_pos_buckets", ctypes.c_int32),
                ("time_table", ctypes.c_void_p), ("n_time_buckets", ctypes.c_int32),
                ("timestamps", ctypes.c_void_p)]


_P, _I32, _I64, _F, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_SIGNATURES = {
    "hstu_version": ([], _I32),
    "hstu_device_check": ([], _I32),
    "hstu_status_string": ([_I32], ctypes.c_char_p),
    "hstu_last_device_error": ([_P], _I32),
    "hstu_attn_fwd": ([_P, _P, _P, _P, _I32, _I32, _I64, _I32, _I32, _I32, _I32, _P, _F, _P, _P], _I32),
    "hstu_kv_table_create": ([_I64, _I32, _I32, _I32, _I32, _I64, _I32, _P, _P], _I32),
    "hstu_kv_table_destroy": ([_P], None),
    "hstu_kv_table_status": ([_P, _P], _I32),
    "hstu_kv_table_info": ([_P, _P, _P, _P, _P, _P], _I32),
    "hstu_kv_alloc": ([_P, _P, _P, _I32, _P, _I32, _P], _I32),
    "hstu_kv_append": ([_P, _P, _P, _P, _P, _I32, _I32, _P], _I32),
    "hstu_kv_release": ([_P, _P, _I32, _P], _I32),
    "hstu_attn_beam_decode": ([_P, _P, _I32, _P, _P, _I64, _I32, _I32, _I32, _P, _P, _P, _P, _F, _P,
                               _P, _SZ, _P], _I32),
    "hstu_attn_beam_decode_workspace_size": ([_P, _I32, _I64, _I32, _I32, _I32], _SZ),
    "hstu_user_map_create": ([_I32, _P, _P], _I32),
    "hstu_user_map_destroy": ([_P], None),
    "hstu_user_map_lookup": ([_P, _P, _I32, _I32, _P, _P], _I32),
    "hstu_user_map_erase": ([_P, _P, _I32, _P], _I32),
    "hstu_user_map_status": ([_P, _P], _I32),
    "hstu_kv_lookup": ([_P, _P, _I32, _P, _P, _I32, _P, _P, _P, _I32, _P], _I32),
    "hstu_kv_step": ([_P, _P, _P, _P, _P, _I32, _I32, _P, _P, _I32, _P], _I32),
    "hstu_wait_timeout_selftest": ([_I32, _P], _I32),
    "hstu_attn_cached_fwd": ([_P, _P, _I32, _P, _P, _P, _P, _I64, _I32, _I32, _I32, _P, _F, _P, _P,
                              _SZ, _P], _I32),
    "hstu_attn_cached_workspace_size": ([_P, _I32, _I64, _I32, _I32, _I32], _SZ),
    "hstu_attn_cached_noalloc_max_scratch": ([], _SZ),
    "hstu_attn_cached_fwd_noalloc": ([_P, _P, _I32, _P, _P, _P, _P, _I64, _I32, _I32, _I32, _P, _F, _P,
                                      _P], _I32),
    "hstu_block_fwd": ([_P, _P, _I32, _I32, _I64, _I32, _I32, _I32, _I32, _P, _P, _P, _F, _F, _P,
                        _SZ, _P], _I32),
    "hstu_block_workspace_size": ([_I64, _I32, _I32, _I32], _SZ),
    "hstu_block_cached_step": ([_P, _I32, _P, _I32, _P, _P, _I64, _I32, _P, _I64, _I32, _I32, _I32,
                                _I32, _I32, _P, _P, _P, _F, _F, _P, _SZ, _P], _I32),
    "hstu_block_cached_workspace_size": ([_P, _I32, _I32, _I64, _I64, _I32, _I32, _I32, _I32, _I32],
                                         _SZ),
}

_lock = threading.Lock()
_lib = None


def declared_symbols() -> list[str]:
    """Every entry point that include/hstu.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^HSTU_API\s+[\w\s\*]+?\b(hstu_\w+)\s*\(", text, flags=re.M)))


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (no GPU needed to load; kernels need an sm_100 device)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m generative_recommender_sequence_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (args, res) in _SIGNATURES.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        _lib = lib
        return lib


def check(fn: str, status: int):
    if status != HSTU_OK:
        raise HstuError(fn, status)
