"""Beam-search decode attention over a shared context (fp64 oracle, test infrastructure only).

Source: "How Generative Recommenders Are Redefining RecSys at Scale", section
"Semantic ID-GR": a request's long context is shared by all beams, each beam
has a short decode history and an ancestry; beams are not treated as separate
long sequences.  The attention is the HSTU one.

Definition used here: beam j of request b at decode step s is the last row of
causal HSTU attention (``oracle.attn_causal``, pinned elsewhere) over the
sequence [context_b; the decode tokens of j's ancestors at steps 0 .. s-1; j's
own step-s token], at positions 0 .. L_b + s.  Ancestors follow
``beam_parent[t][row]`` = the index, within the request, of the step t-1 beam
that row ``row`` of step t extends.
"""

from __future__ import annotations

import numpy as np

from . import attn_causal


def ancestry(beam_parent, beam_offsets, b, j, step):
    """Rows (per step 0 .. step-1) of the ancestors of beam j of request b."""
    base = int(beam_offsets[b])
    rows, beam = [], j
    for t in range(step - 1, -1, -1):
        beam = int(beam_parent[t + 1][base + beam])
        rows.append(base + beam)
    return rows[::-1]


def attn_beam_decode(ctx_k, ctx_v, ctx_offsets, q, beam_offsets, step, beam_k, beam_v, beam_parent,
                     pos_table=None, scale=1.0, threads=None, magnitude=None):
    """Beam outputs of step `step`; magnitude as for ``oracle.attn_causal``."""
    ck, cv = np.asarray(ctx_k, np.float64), np.asarray(ctx_v, np.float64)
    bk, bv = np.asarray(beam_k, np.float64), np.asarray(beam_v, np.float64)
    co, bo = np.asarray(ctx_offsets, np.int64), np.asarray(beam_offsets, np.int64)
    ks, vs, lens = [], [], []
    for b in range(len(bo) - 1):
        for j in range(int(bo[b + 1] - bo[b])):
            anc = ancestry(beam_parent, bo, b, j, step)
            ks.append(np.concatenate([ck[co[b]:co[b + 1]]] + [bk[t][r][None] for t, r in enumerate(anc)]
                                     + [bk[step][bo[b] + j][None]]))
            vs.append(np.concatenate([cv[co[b]:co[b + 1]]] + [bv[t][r][None] for t, r in enumerate(anc)]
                                     + [bv[step][bo[b] + j][None]]))
            lens.append(len(ks[-1]))
    kv_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    q_off = np.arange(len(lens) + 1, dtype=np.int64)
    return attn_causal(np.asarray(q, np.float64), np.concatenate(ks), np.concatenate(vs), kv_off,
                       q_offsets=q_off, pos_table=pos_table, scale=scale, threads=threads,
                       magnitude=magnitude)
