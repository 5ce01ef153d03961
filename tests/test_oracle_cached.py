"""Pins for oracle.cached.hstu_block_cached (the KV-cached multi-layer step, defined
as the uncached block stack over whole sequences).  CPU only."""

import numpy as np
import pytest

import oracle
from oracle import brute
from oracle.cached import hstu_block_cached


def _case(hist, new, cand, dm=16, H=2, dh=8, n_layers=2, seed=0):
    rng = np.random.default_rng(seed)
    off = lambda n: np.concatenate([[0], np.cumsum(n)]).astype(np.int64)
    xh = rng.standard_normal((sum(hist), dm))
    xn = rng.standard_normal((sum(new), dm))
    xc = rng.standard_normal((sum(cand), dm))
    w1 = rng.normal(0, 0.2, (n_layers, dm, 4 * H * dh))
    w2 = rng.normal(0, 0.2, (n_layers, H * dh, dm))
    pt = rng.normal(0, 0.1, 16)
    return dict(x_hist=xh, hist_offsets=off(hist), x_new=xn, new_offsets=off(new), x_cand=xc,
                cand_offsets=off(cand), w_uvqk=w1, w_o=w2, pos_table=pt, scale=0.05, H=H, dh=dh,
                round_bf16=False)


def test_no_history_no_candidates_is_the_block():
    c = _case([0, 0], [5, 9], [0, 0])
    got_new, got_c = hstu_block_cached(**c)
    ref = oracle.hstu_block(c["x_new"], c["new_offsets"], c["w_uvqk"], c["w_o"], None, c["pos_table"],
                            None, c["scale"], H=c["H"], dh=c["dh"], round_bf16=False)
    assert got_c.shape[0] == 0
    np.testing.assert_allclose(got_new, ref, rtol=0, atol=1e-12)


def test_candidates_are_exchangeable_and_independent():
    c = _case([6, 3], [2, 4], [3, 2], seed=1)
    _, out = hstu_block_cached(**c)
    # permute user 0's candidates
    c2 = dict(c)
    c2["x_cand"] = c["x_cand"][[2, 0, 1, 3, 4]]
    _, out2 = hstu_block_cached(**c2)
    np.testing.assert_allclose(out2, out[[2, 0, 1, 3, 4]], rtol=0, atol=1e-12)
    # drop user 1's first candidate: the others do not change
    c3 = dict(c)
    c3["x_cand"] = c["x_cand"][[0, 1, 2, 4]]
    c3["cand_offsets"] = np.array([0, 3, 4])
    _, out3 = hstu_block_cached(**c3)
    np.testing.assert_allclose(out3, out[[0, 1, 2, 4]], rtol=0, atol=1e-12)
    # two identical candidates score identically
    c4 = dict(c)
    xc = c["x_cand"].copy()
    xc[1] = xc[0]
    c4["x_cand"] = xc
    _, out4 = hstu_block_cached(**c4)
    np.testing.assert_allclose(out4[0], out4[1], rtol=0, atol=1e-12)


def _masked_single_pass(c, ln_eps=1e-5):
    """Independent restatement: one pass per user over [hist; new; cands] with an
    explicit mask (causal among history and new tokens; a candidate sees those and
    itself, at the position one past the last of them), numpy fp64."""
    H, dh = c["H"], c["dh"]
    F = H * dh
    ho, no, co = c["hist_offsets"], c["new_offsets"], c["cand_offsets"]
    outs_new, outs_c = [], []
    for b in range(len(ho) - 1):
        xh = c["x_hist"][ho[b]:ho[b + 1]]
        xn = c["x_new"][no[b]:no[b + 1]]
        xc = c["x_cand"][co[b]:co[b + 1]]
        n, m = len(xh) + len(xn), len(xc)
        x = np.concatenate([xh, xn, xc])
        pos = np.concatenate([np.arange(n), np.full(m, n)])
        mask = np.zeros((n + m, n + m), bool)
        mask[:n, :n] = np.tril(np.ones((n, n), bool))
        mask[n:, :n] = True
        mask[np.arange(n, n + m), np.arange(n, n + m)] = True
        for l in range(c["w_uvqk"].shape[0]):
            y = x @ c["w_uvqk"][l]
            y = y * brute._logistic(y)
            u, v, q, k = (y[:, i * F:(i + 1) * F].reshape(-1, H, dh) for i in range(4))
            s = brute.user_scores(q, k, pos, pos, None, None, c["pos_table"], None)
            w = np.where(mask[None], s * brute._logistic(s), 0.0)
            a = np.einsum("hij,jhe->ihe", w, v).reshape(-1, F) * c["scale"]
            mu = a.mean(1, keepdims=True)
            var = ((a - mu) ** 2).mean(1, keepdims=True)
            g = (a - mu) / np.sqrt(var + ln_eps) * u.reshape(-1, F)
            x = x + g @ c["w_o"][l]
        outs_new.append(x[len(xh):n])
        outs_c.append(x[n:])
    return np.concatenate(outs_new), np.concatenate(outs_c)


@pytest.mark.parametrize("hist,new,cand", [([7, 0, 12], [3, 5, 1], [2, 4, 1]), ([20], [0], [3])])
def test_matches_a_single_masked_pass(hist, new, cand):
    c = _case(hist, new, cand, seed=2)
    got_new, got_c = hstu_block_cached(**c)
    ref_new, ref_c = _masked_single_pass(c)
    np.testing.assert_allclose(got_new, ref_new, rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(got_c, ref_c, rtol=1e-9, atol=1e-10)
