"""Pins for oracle.beam.attn_beam_decode (beam decode attention over a shared context)."""

import numpy as np

import oracle
from oracle import brute
from oracle.beam import ancestry, attn_beam_decode


def _case(ctx, beams, step, H=2, d=8, seed=0):
    rng = np.random.default_rng(seed)
    co = np.concatenate([[0], np.cumsum(ctx)]).astype(np.int64)
    bo = np.concatenate([[0], np.cumsum(beams)]).astype(np.int64)
    T = int(bo[-1])
    ck, cv = rng.standard_normal((2, int(co[-1]), H, d))
    q = rng.standard_normal((T, H, d))
    bk, bv = rng.standard_normal((2, step + 1, T, H, d))
    parent = np.zeros((step + 1, T), np.int32)
    for t in range(1, step + 1):
        for b in range(len(beams)):
            parent[t, bo[b]:bo[b + 1]] = rng.integers(0, beams[b], size=beams[b])
    return dict(ctx_k=ck, ctx_v=cv, ctx_offsets=co, q=q, beam_offsets=bo, step=step, beam_k=bk,
                beam_v=bv, beam_parent=parent, pos_table=rng.normal(0, 0.1, 16), scale=0.1)


def test_step_zero_is_candidate_attention():
    c = _case([7, 20], [3, 5], step=0)
    got = attn_beam_decode(**c)
    ref = oracle.attn_candidates(c["ctx_k"], c["ctx_v"], c["ctx_offsets"], c["q"], c["beam_k"][0],
                                 c["beam_v"][0], c["beam_offsets"], pos_table=c["pos_table"],
                                 scale=c["scale"])
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_three_key_sets_add_up():
    """Independent restatement: context + ancestors + own token, summed directly."""
    c = _case([11, 4], [4, 6], step=2, seed=1)
    got = attn_beam_decode(**c)
    bo, co = c["beam_offsets"], c["ctx_offsets"]
    for b in range(2):
        L = int(co[b + 1] - co[b])
        for j in range(int(bo[b + 1] - bo[b])):
            r = int(bo[b] + j)
            anc = ancestry(c["beam_parent"], bo, b, j, 2)
            keys = [c["ctx_k"][co[b] + i] for i in range(L)] + [c["beam_k"][t][a] for t, a in enumerate(anc)] \
                + [c["beam_k"][2][r]]
            vals = [c["ctx_v"][co[b] + i] for i in range(L)] + [c["beam_v"][t][a] for t, a in enumerate(anc)] \
                + [c["beam_v"][2][r]]
            pos = np.arange(L + 3)
            s = brute.user_scores(c["q"][r][None], np.stack(keys), np.array([L + 2]), pos, None, None,
                                  c["pos_table"], None)[:, 0, :]          # [H, keys]
            w = s * brute._logistic(s)
            ref = np.einsum("hj,jhe->he", w, np.stack(vals)) * c["scale"]
            np.testing.assert_allclose(got[r], ref, rtol=1e-10, atol=1e-12)


def test_beams_with_the_same_path_and_tokens_agree():
    c = _case([9], [4], step=1, seed=2)
    c["beam_parent"][1] = [2, 2, 0, 1]
    c["beam_k"][1][1] = c["beam_k"][1][0]
    c["beam_v"][1][1] = c["beam_v"][1][0]
    c["q"][1] = c["q"][0]
    got = attn_beam_decode(**c)
    np.testing.assert_allclose(got[0], got[1], rtol=0, atol=0)
    assert not np.allclose(got[0], got[2])
