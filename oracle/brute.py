"""Independent numpy restatement of HSTU attention for tiny inputs.

TEST INFRASTRUCTURE ONLY.  Used to cross-check the C oracle (to ~1e-12) on
small shapes.  It is written differently on purpose: whole score matrices per
user, an explicit boolean mask, ``frexp`` for floor(log2) and a logistic
written as 0.5*(1+tanh(x/2)), so that a slip in one implementation does not
repeat in the other.
"""

from __future__ import annotations

import numpy as np


def _floor_log2_plus1(a: np.ndarray) -> np.ndarray:
    # floor(log2(a + 1)) for integer a >= 0: frexp gives a + 1 = m * 2^e, m in [0.5, 1)
    return np.frexp((a + 1).astype(np.float64))[1] - 1


def _logistic(x):
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def user_scores(q, k, pos_q, pos_k, ts_q, ts_k, pos_table, time_table):
    """S[h, i, j] = q_i . k_j + rab(i, j) for one user (fp64)."""
    s = np.einsum("ihe,jhe->hij", q, k)
    if pos_table is not None:
        dpos = np.abs(pos_q[:, None] - pos_k[None, :])
        b = np.minimum(_floor_log2_plus1(dpos), len(pos_table) - 1)
        s = s + np.asarray(pos_table, np.float64)[b][None]
    if time_table is not None:
        dt = np.maximum(ts_q[:, None] - ts_k[None, :], 0)
        b = np.minimum(_floor_log2_plus1(dt), len(time_table) - 1)
        s = s + np.asarray(time_table, np.float64)[b][None]
    return s


def causal(q, k, v, offsets, timestamps=None, pos_table=None, time_table=None, scale=1.0,
           magnitude=None):
    """magnitude "silu" / "score": |scale| * sum of |SiLU(s)| |v| / |s| |v| over the
    visible keys."""
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    if magnitude:
        v, scale = np.abs(v), abs(scale)
    out = np.zeros((q.shape[0], q.shape[1], v.shape[2]))
    for b in range(len(offsets) - 1):
        s0, e0 = int(offsets[b]), int(offsets[b + 1])
        L = e0 - s0
        pos = np.arange(L)
        ts = None if timestamps is None else np.asarray(timestamps[s0:e0], np.int64)
        S = user_scores(q[s0:e0], k[s0:e0], pos, pos, ts, ts, pos_table,
                        time_table if ts is not None else None)
        mask = pos[None, :] <= pos[:, None]
        W = np.where(mask[None], S if magnitude == "score" else S * _logistic(S), 0.0)
        if magnitude:
            W = np.abs(W)
        out[s0:e0] = np.einsum("hij,jhe->ihe", W, v[s0:e0]) * scale
    return out


def candidates(hist_k, hist_v, hist_offsets, q, k_cand, v_cand, cand_offsets, pos_table=None,
               scale=1.0, magnitude=None):
    hk, hv, q, kc, vc = (np.asarray(x, np.float64) for x in (hist_k, hist_v, q, k_cand, v_cand))
    if magnitude:
        hv, vc, scale = np.abs(hv), np.abs(vc), abs(scale)
    out = np.zeros((q.shape[0], q.shape[1], vc.shape[2]))
    for b in range(len(cand_offsets) - 1):
        hs, he = int(hist_offsets[b]), int(hist_offsets[b + 1])
        cs, ce = int(cand_offsets[b]), int(cand_offsets[b + 1])
        nh, nc = he - hs, ce - cs
        keys = np.concatenate([hk[hs:he], kc[cs:ce]])
        vals = np.concatenate([hv[hs:he], vc[cs:ce]])
        pos_k = np.concatenate([np.arange(nh), np.full(nc, nh)])
        pos_q = np.full(nc, nh)
        S = user_scores(q[cs:ce], keys, pos_q, pos_k, None, None, pos_table, None)
        mask = np.zeros((nc, nh + nc), bool)
        mask[:, :nh] = True
        mask[np.arange(nc), nh + np.arange(nc)] = True
        W = np.where(mask[None], S if magnitude == "score" else S * _logistic(S), 0.0)
        if magnitude:
            W = np.abs(W)
        out[cs:ce] = np.einsum("hij,jhe->ihe", W, vals) * scale
    return out
