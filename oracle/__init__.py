"""Plain, slow, fp64 CPU oracle for the HSTU attention hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The
product package never imports it and shares no code with it.

Contents
* ``hstu_oracle.c`` (compiled here with gcc): causal and candidate attention,
  the rab bucket functions, SiLU, bf16 rounding, LayerNorm gate and the block
  stack, all as straight fp64 loop nests (see the header of that file for the
  definitions and their sources).
* ``kv.py``: the paged KV table as a sequential Python model (free stack,
  per-user page lists, byte-exact pool).
* ``brute.py``: an independent numpy restatement used only to cross-check the C
  code on tiny inputs.
* ``cached.py``: the KV-cached multi-layer serving step, defined as the
  uncached block stack over whole sequences (``hstu_block_cached``).

Parity status: every function here is pinned by tests under
``tests/test_oracle_*.py`` (closed forms, reductions to library routines,
invariants, hand tables, brute force).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hstu_oracle.c")
_LIB = os.path.join(_HERE, "libhstu_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (fp64, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
               "-shared", "-pthread", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P, I, L, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_pos_bucket.argtypes = [L, I]
            lib.oracle_pos_bucket.restype = I
            lib.oracle_time_bucket.argtypes = [L, I]
            lib.oracle_time_bucket.restype = I
            lib.oracle_silu.argtypes = [D]
            lib.oracle_silu.restype = D
            lib.oracle_round_bf16.argtypes = [D]
            lib.oracle_round_bf16.restype = D
            lib.oracle_attn_causal.argtypes = [I, I, I, I, P, P, P, P, P, P, P, I, P, I, D, P, L, P, I]
            lib.oracle_attn_causal.restype = I
            lib.oracle_attn_candidates.argtypes = [I, I, I, I, P, P, P, P, P, P, P, P, I, D, P, L, P, I]
            lib.oracle_attn_candidates.restype = I
            lib.oracle_attn_causal_magnitude.argtypes = lib.oracle_attn_causal.argtypes + [I]
            lib.oracle_attn_causal_magnitude.restype = I
            lib.oracle_attn_candidates_magnitude.argtypes = lib.oracle_attn_candidates.argtypes + [I]
            lib.oracle_attn_candidates_magnitude.restype = I
            lib.oracle_layernorm_gate.argtypes = [L, L, P, P, D, I, P, I]
            lib.oracle_layernorm_gate.restype = I
            lib.oracle_hstu_block.argtypes = [L, I, P, I, I, I, I, P, P, P, P, P, I, P, I, D, D, I, I, P, I]
            lib.oracle_hstu_block.restype = I
            _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def _f64(x):
    return None if x is None else np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i64(x):
    return None if x is None else np.ascontiguousarray(np.asarray(x, dtype=np.int64))


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


_MAGNITUDE_KIND = {"silu": 1, "score": 2}


def pos_bucket(delta: int, n_buckets: int) -> int:
    return _load().oracle_pos_bucket(int(delta), int(n_buckets))


def time_bucket(dt: int, n_buckets: int) -> int:
    return _load().oracle_time_bucket(int(dt), int(n_buckets))


def silu(x: float) -> float:
    return _load().oracle_silu(float(x))


def round_bf16(x) -> np.ndarray:
    f = _load().oracle_round_bf16
    a = np.asarray(x, dtype=np.float64)
    return np.vectorize(f, otypes=[np.float64])(a) if a.size else a.copy()


def attn_causal(q, k, v, kv_offsets, q_offsets=None, timestamps=None, pos_table=None,
                time_table=None, scale=1.0, rows=None, threads=None,
                magnitude=None) -> np.ndarray:
    """Causal HSTU attention; the queries of user b are its last nq_b tokens.

    q: [Tq,H,dqk], k: [Tk,H,dqk], v: [Tk,H,dv]; returns fp64 [Tq or len(rows), H, dv].
    magnitude="silu" returns |scale| * sum_j |SiLU(s_j)| |v_j| and magnitude="score"
    |scale| * sum_j |s_j| |v_j| (s_j = q . k_j + rab) instead: the sizes of the
    sum's terms, for rounding-error bounds, not attention results.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    kv_off = _i64(kv_offsets)
    q_off = kv_off if q_offsets is None else _i64(q_offsets)
    B = len(kv_off) - 1
    H, dqk = q.shape[1], q.shape[2]
    dv = v.shape[2]
    ts = _i64(timestamps)
    pt, tt = _f64(pos_table), _f64(time_table)
    rows_a = _i64(rows)
    n_rows = len(rows_a) if rows_a is not None else int(q_off[-1])
    out = np.zeros((n_rows, H, dv), dtype=np.float64)
    args = (B, H, dqk, dv, _p(kv_off), _p(q_off), _p(q), _p(k), _p(v), _p(ts), _p(pt),
            0 if pt is None else len(pt), _p(tt), 0 if tt is None else len(tt), float(scale),
            _p(rows_a), n_rows, _p(out), threads or default_threads())
    if magnitude is None:
        rc = _load().oracle_attn_causal(*args)
    else:
        rc = _load().oracle_attn_causal_magnitude(*args, _MAGNITUDE_KIND[magnitude])
    if rc != 0:
        raise ValueError("oracle_attn_causal: bad arguments")
    return out


def attn_candidates(hist_k, hist_v, hist_offsets, q, k_cand, v_cand, cand_offsets,
                    pos_table=None, scale=1.0, rows=None, threads=None,
                    magnitude=None) -> np.ndarray:
    """Candidates of user b attend to all of b's cached tokens plus themselves.

    magnitude="silu" / "score": term-by-term magnitudes instead (see attn_causal)."""
    hk, hv = _f64(hist_k), _f64(hist_v)
    q, kc, vc = _f64(q), _f64(k_cand), _f64(v_cand)
    ho, co = _i64(hist_offsets), _i64(cand_offsets)
    B = len(co) - 1
    H, dqk, dv = q.shape[1], q.shape[2], vc.shape[2]
    pt = _f64(pos_table)
    rows_a = _i64(rows)
    n_rows = len(rows_a) if rows_a is not None else int(co[-1])
    out = np.zeros((n_rows, H, dv), dtype=np.float64)
    args = (B, H, dqk, dv, _p(ho), _p(hk), _p(hv), _p(co), _p(q), _p(kc), _p(vc), _p(pt),
            0 if pt is None else len(pt), float(scale), _p(rows_a), n_rows, _p(out),
            threads or default_threads())
    if magnitude is None:
        rc = _load().oracle_attn_candidates(*args)
    else:
        rc = _load().oracle_attn_candidates_magnitude(*args, _MAGNITUDE_KIND[magnitude])
    if rc != 0:
        raise ValueError("oracle_attn_candidates: bad arguments")
    return out


def layernorm_gate(a, u, eps=1e-5, round_bf16=False, threads=None) -> np.ndarray:
    a, u = _f64(a), _f64(u)
    T, F = a.shape
    g = np.zeros((T, F), dtype=np.float64)
    _load().oracle_layernorm_gate(T, F, _p(a), _p(u), float(eps), int(bool(round_bf16)), _p(g),
                                  threads or default_threads())
    return g


def hstu_block(x0, seq_offsets, w_uvqk, w_o, timestamps, pos_table, time_table, scale,
               ln_eps=1e-5, H=4, dh=128, round_bf16=True, return_layers=False, threads=None,
               round_output=True):
    """Block stack: per layer X <- X + (LayerNorm(attn(SiLU(X W1))) * U) W2.

    round_bf16 rounds UVQK, A, G and X to bf16 where the GPU stores bf16;
    round_output=False leaves only the last layer's X unrounded."""
    x = _f64(x0).copy()
    off = _i64(seq_offsets)
    w1, w2 = _f64(w_uvqk), _f64(w_o)
    n_layers, dm = w1.shape[0], w1.shape[1]
    T = x.shape[0]
    ts = _i64(timestamps)
    pt, tt = _f64(pos_table), _f64(time_table)
    layers = np.zeros((n_layers, T, dm), dtype=np.float64) if return_layers else None
    rc = _load().oracle_hstu_block(T, len(off) - 1, _p(off), n_layers, dm, H, dh, _p(x), _p(w1),
                                   _p(w2), _p(ts), _p(pt), 0 if pt is None else len(pt), _p(tt),
                                   0 if tt is None else len(tt), float(scale), float(ln_eps),
                                   int(bool(round_bf16)), int(bool(round_output)), _p(layers),
                                   threads or default_threads())
    if rc != 0:
        raise ValueError("oracle_hstu_block failed (%d)" % rc)
    return (x, layers) if return_layers else x
