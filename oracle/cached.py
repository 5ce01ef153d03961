"""KV-cached multi-layer serving step, defined by full recomputation (fp64 oracle).

TEST INFRASTRUCTURE ONLY (same rules as the rest of ``oracle/``).

Source: "NVIDIA Dynamo-Triton Gets End-to-End HSTU Generative Recommender
Workflow", sections "What the workflow combines" (KV caching keeps reusable
key-value state so long histories are not recomputed when new tokens arrive)
and the benchmark paragraph (the cached model is measured against the same
model without KV caching, so both compute the same result).

Definition used here: the cached step must equal the uncached block stack
(``oracle.hstu_block``, itself pinned in tests/test_oracle_block_kv.py) run over
whole sequences:
  * a new token of user b is its row of block([history_b; new_b]);
  * candidate c of user b is the last row of block([history_b; new_b; c]): in
    causal order that row sees the history, the new tokens and itself, at the
    position one past the last cached token, which is the candidate mask.
Every sequence of the batch goes through one call of the block oracle.
"""

from __future__ import annotations

import numpy as np

from . import hstu_block


def hstu_block_cached(x_hist, hist_offsets, x_new, new_offsets, x_cand, cand_offsets, w_uvqk, w_o,
                      pos_table, scale, ln_eps=1e-5, H=4, dh=128, round_bf16=True, threads=None,
                      round_output=True):
    """Returns (final new rows [T_new, d], final candidate rows [T_cand, d]) in fp64.

    x_hist / x_new / x_cand: layer-0 rows, jagged per user by the [B+1] offsets
    (x_cand / cand_offsets may be None).  round_output=False leaves the last
    layer's output unrounded (see ``oracle.hstu_block``)."""
    ho, no = np.asarray(hist_offsets, np.int64), np.asarray(new_offsets, np.int64)
    B = len(ho) - 1
    co = np.zeros(B + 1, np.int64) if cand_offsets is None else np.asarray(cand_offsets, np.int64)
    xh, xn = np.asarray(x_hist, np.float64), np.asarray(x_new, np.float64)
    xc = np.zeros((0, xh.shape[1])) if x_cand is None else np.asarray(x_cand, np.float64)
    seqs, new_rows, cand_rows = [], [], []
    start = 0
    for b in range(B):
        base = np.concatenate([xh[ho[b]:ho[b + 1]], xn[no[b]:no[b + 1]]])
        seqs.append(base)
        n_hist = int(ho[b + 1] - ho[b])
        new_rows.extend(range(start + n_hist, start + len(base)))
        start += len(base)
        for c in range(int(co[b]), int(co[b + 1])):
            seqs.append(np.concatenate([base, xc[c:c + 1]]))
            start += len(base) + 1
            cand_rows.append(start - 1)
    lengths = [len(s) for s in seqs]
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    x_all = np.concatenate(seqs) if seqs else np.zeros((0, xh.shape[1]))
    y = hstu_block(x_all, offsets, w_uvqk, w_o, None, pos_table, None, scale, ln_eps=ln_eps, H=H,
                   dh=dh, round_bf16=round_bf16, threads=threads, round_output=round_output)
    return y[np.asarray(new_rows, np.int64)], y[np.asarray(cand_rows, np.int64)]
