"""Pins for the fp64 attention oracle (CPU only).

The pages print no worked example, so every pin here is a closed form, a
reduction to a library routine, a hand table, an invariant, or an independent
brute-force restatement (oracle/brute.py) on tiny inputs.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from workloads import jagged_case, offsets_from_lengths, tiny_fp32


def silu_math(x):
    return x / (1.0 + math.exp(-x))


def test_closed_form_two_tokens(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "closed_form_two_tokens.json")))
    q = np.array(g["q"]).reshape(2, 1, 1)
    k = np.array(g["k"]).reshape(2, 1, 1)
    v = np.array(g["v"]).reshape(2, 1, 1)
    out = oracle.attn_causal(q, k, v, [0, 2], pos_table=None, scale=1.0 / g["N"])
    np.testing.assert_allclose(out.ravel(), g["expected"], rtol=1e-15, atol=0)
    # the same with an all-zero 16-bucket table must not change anything
    out0 = oracle.attn_causal(q, k, v, [0, 2], pos_table=np.zeros(16), scale=0.5)
    assert np.array_equal(out0, out)


def test_bucket_table(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "bucket_table.json")))
    for delta, b in g["pos_n16"]:
        assert oracle.pos_bucket(delta, 16) == b, delta
    for delta, b in g["pos_n128"]:
        assert oracle.pos_bucket(delta, 128) == b, delta
    for dt, b in g["time_n64"]:
        assert oracle.time_bucket(dt, 64) == b, dt
    for dt, b in g["time_n8"]:
        assert oracle.time_bucket(dt, 8) == b, dt


def test_rab_hand_case():
    """Three tokens, d=1, q=0: scores are the rab alone; buckets worked out by hand."""
    pos_table = np.array([0.5, -0.25, 1.5, 0.75])               # n_pos = 4
    time_table = np.array([0.125, -0.5, 0.3125, 1.0, -1.0, 2.0, 0.0, 0.375, 3.0, -2.0])
    ts = np.array([100, 105, 1100], dtype=np.int64)
    v = np.array([1.0, 10.0, 100.0]).reshape(3, 1, 1)
    z = np.zeros((3, 1, 1))
    out = oracle.attn_causal(z, z, v, [0, 3], timestamps=ts, pos_table=pos_table,
                             time_table=time_table, scale=0.5).ravel()
    # pos buckets: |0|->0, |1|->1, |2|->1 ; time buckets: 0->0, 5->2, 995->9, 1000->9
    e0 = 0.5 * silu_math(0.5 + 0.125) * 1
    e1 = 0.5 * (silu_math(-0.25 + 0.3125) * 1 + silu_math(0.5 + 0.125) * 10)
    e2 = 0.5 * (silu_math(-0.25 + -2.0) * 1 + silu_math(-0.25 + -2.0) * 10
                + silu_math(0.5 + 0.125) * 100)
    np.testing.assert_allclose(out, [e0, e1, e2], rtol=1e-14)


def test_prefix_sum_reduction():
    """Q = 0 and rab = c everywhere: O_i = SiLU(c) * scale * sum_{j<=i} v_j (torch.cumsum)."""
    rng = np.random.default_rng(0)
    lengths = [5, 1, 9]
    off = offsets_from_lengths(lengths)
    T, H, d = int(off[-1]), 2, 3
    c = 0.7
    q = np.zeros((T, H, d))
    k = rng.standard_normal((T, H, d))
    v = rng.standard_normal((T, H, d))
    out = oracle.attn_causal(q, k, v, off, pos_table=np.full(16, c), scale=0.125)
    for b in range(3):
        s, e = off[b], off[b + 1]
        ref = torch.cumsum(torch.from_numpy(v[s:e]), dim=0).numpy() * silu_math(c) * 0.125
        np.testing.assert_allclose(out[s:e], ref, rtol=1e-13, atol=1e-15)


def test_k_zero_rab_zero_gives_zero():
    case = jagged_case(7, [3, 11], H=2, d=8, dtype="f32", n_pos=16)
    out = oracle.attn_causal(case.q, np.zeros_like(case.k), case.v, case.seq_offsets,
                             pos_table=np.zeros(16), scale=case.scale)
    assert np.all(out == 0.0)


def test_linear_regime_masked_matmul():
    """rab = 60 and |q.k| <= 10: sigmoid == 1 in fp64, so O = tril(QK^T + 60) V * scale."""
    rng = np.random.default_rng(1)
    L, H, d = 13, 2, 4
    q = rng.uniform(-0.5, 0.5, (L, H, d))
    k = rng.uniform(-0.5, 0.5, (L, H, d))
    v = rng.standard_normal((L, H, d))
    out = oracle.attn_causal(q, k, v, [0, L], pos_table=np.full(16, 60.0), scale=0.25)
    for h in range(H):
        Q, K, V = (torch.from_numpy(x[:, h]) for x in (q, k, v))
        S = torch.tril(Q @ K.T + 60.0)
        ref = (S @ V).numpy() * 0.25
        np.testing.assert_allclose(out[:, h], ref, rtol=1e-13)


def test_causality_future_perturbation_is_invisible():
    case = jagged_case(3, [20, 33], H=2, d=8, dtype="f32", n_pos=16, n_time=8)
    base = oracle.attn_causal(case.q, case.k, case.v, case.seq_offsets, timestamps=case.timestamps,
                              pos_table=case.pos_table, time_table=case.time_table, scale=case.scale)
    i = 25  # a token of the second user
    q, k, v = case.q.copy(), case.k.copy(), case.v.copy()
    k[i + 1:] += 3.0
    v[i + 1:] -= 2.0
    q[i + 1:] *= -1.0
    pert = oracle.attn_causal(q, k, v, case.seq_offsets, timestamps=case.timestamps,
                              pos_table=case.pos_table, time_table=case.time_table, scale=case.scale)
    assert np.array_equal(pert[: i + 1], base[: i + 1])
    assert not np.array_equal(pert[i + 1:], base[i + 1:])


def test_users_are_independent():
    case = jagged_case(4, [9, 14, 6], H=2, d=4, dtype="f32", n_pos=16)
    base = oracle.attn_causal(case.q, case.k, case.v, case.seq_offsets, pos_table=case.pos_table,
                              scale=case.scale)
    k = case.k.copy()
    s, e = case.seq_offsets[1], case.seq_offsets[2]
    k[s:e] += 1.0
    pert = oracle.attn_causal(case.q, k, case.v, case.seq_offsets, pos_table=case.pos_table,
                              scale=case.scale)
    assert np.array_equal(pert[:s], base[:s]) and np.array_equal(pert[e:], base[e:])
    assert not np.array_equal(pert[s:e], base[s:e])


def test_linearity_in_v_and_power_of_two_scale():
    case = jagged_case(5, [7, 12], H=2, d=4, dtype="f32", n_pos=16)
    rng = np.random.default_rng(2)
    v2 = rng.standard_normal(case.v.shape)
    f = lambda v, s=1.0: oracle.attn_causal(case.q, case.k, v, case.seq_offsets,
                                            pos_table=case.pos_table, scale=s)
    v1 = case.v.astype(np.float64)
    np.testing.assert_allclose(f(2.5 * v1 + v2), 2.5 * f(v1) + f(v2), rtol=1e-12, atol=1e-12)
    assert np.array_equal(f(case.v, 0.25), f(case.v) * 0.25)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_twin_causal(seed):
    rng = np.random.default_rng(100 + seed)
    lengths = rng.integers(1, 40, size=3)
    case = jagged_case(seed, lengths, H=2, d=int(rng.integers(1, 9)), dtype="f32",
                       n_pos=int(rng.integers(2, 20)), n_time=int(rng.integers(2, 20)))
    got = oracle.attn_causal(case.q, case.k, case.v, case.seq_offsets, timestamps=case.timestamps,
                             pos_table=case.pos_table, time_table=case.time_table, scale=case.scale)
    ref = brute.causal(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                       case.pos_table, case.time_table, case.scale)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_tiny_fp32_workload_matches_brute():
    case = tiny_fp32()
    assert case.T == 57 and case.H == 2 and case.d == 32 and case.scale == 1 / 40
    got = oracle.attn_causal(case.q, case.k, case.v, case.seq_offsets, pos_table=case.pos_table,
                             scale=case.scale)
    ref = brute.causal(case.q, case.k, case.v, case.seq_offsets, pos_table=case.pos_table,
                       scale=case.scale)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_sampled_rows_match_full():
    case = jagged_case(9, [15, 30], H=2, d=4, dtype="f32", n_pos=16)
    full = oracle.attn_causal(case.q, case.k, case.v, case.seq_offsets, pos_table=case.pos_table,
                              scale=case.scale)
    rows = np.array([44, 0, 15, 14, 29])
    part = oracle.attn_causal(case.q, case.k, case.v, case.seq_offsets, pos_table=case.pos_table,
                              scale=case.scale, rows=rows)
    assert np.array_equal(part, full[rows])


def test_suffix_queries_equal_last_rows_of_full():
    """Queries that are the last n_q tokens of a sequence == last rows of full causal."""
    case = jagged_case(11, [10, 21], H=2, d=4, dtype="f32", n_pos=16, n_time=8)
    full = oracle.attn_causal(case.q, case.k, case.v, case.seq_offsets, timestamps=case.timestamps,
                              pos_table=case.pos_table, time_table=case.time_table, scale=case.scale)
    nq = np.array([3, 21])
    q_off = offsets_from_lengths(nq)
    q = np.concatenate([case.q[7:10], case.q[10:31]])
    got = oracle.attn_causal(q, case.k, case.v, case.seq_offsets, q_offsets=q_off,
                             timestamps=case.timestamps, pos_table=case.pos_table,
                             time_table=case.time_table, scale=case.scale)
    assert np.array_equal(got, np.concatenate([full[7:10], full[10:31]]))


def _cand_case(seed, hist, n_cand, H=2, d=4, n_pos=16):
    rng = np.random.default_rng(seed)
    ho = offsets_from_lengths(hist)
    co = offsets_from_lengths(n_cand)
    Th, Tc = int(ho[-1]), int(co[-1])
    return dict(hist_k=rng.standard_normal((Th, H, d)), hist_v=rng.standard_normal((Th, H, d)),
                hist_offsets=ho, q=rng.standard_normal((Tc, H, d)),
                k_cand=rng.standard_normal((Tc, H, d)), v_cand=rng.standard_normal((Tc, H, d)),
                cand_offsets=co, pos_table=rng.normal(0, 0.1, n_pos), scale=0.03)


def test_candidates_equal_full_recompute():
    """Candidate c == last row of causal attention over [history, c] (cached = full)."""
    a = _cand_case(12, [6, 17], [3, 4])
    got = oracle.attn_candidates(**a)
    for b in range(2):
        hs, he = a["hist_offsets"][b], a["hist_offsets"][b + 1]
        for c in range(a["cand_offsets"][b], a["cand_offsets"][b + 1]):
            k = np.concatenate([a["hist_k"][hs:he], a["k_cand"][c:c + 1]])
            v = np.concatenate([a["hist_v"][hs:he], a["v_cand"][c:c + 1]])
            q = np.concatenate([np.zeros_like(a["hist_k"][hs:he]), a["q"][c:c + 1]])
            full = oracle.attn_causal(q, k, v, [0, len(k)], pos_table=a["pos_table"],
                                      scale=a["scale"])
            assert np.array_equal(got[c], full[-1])


def test_candidate_permutation_equivariance():
    a = _cand_case(13, [8], [6])
    got = oracle.attn_candidates(**a)
    perm = np.array([3, 0, 5, 1, 4, 2])
    b = dict(a)
    for key in ("q", "k_cand", "v_cand"):
        b[key] = a[key][perm]
    assert np.array_equal(oracle.attn_candidates(**b), got[perm])


def test_brute_force_twin_candidates():
    a = _cand_case(14, [0, 5, 23], [2, 1, 5], d=3, n_pos=6)
    np.testing.assert_allclose(oracle.attn_candidates(**a), brute.candidates(**a),
                               rtol=1e-12, atol=1e-12)


def test_sampled_candidate_rows():
    a = _cand_case(15, [4, 9], [3, 3])
    full = oracle.attn_candidates(**a)
    rows = np.array([5, 1])
    assert np.array_equal(oracle.attn_candidates(**a, rows=rows), full[rows])


# ------------------------------------------------------------------ magnitude sums
# |scale| * sum_j |SiLU(q.k_j + rab)| * |v_j| sizes the error bound of a GPU path
# whose per-term error is relative (bf16 P operand); it is pinned like the sum.

@pytest.mark.parametrize("kind", ["silu", "score"])
@pytest.mark.parametrize("seed", [0, 1])
def test_magnitude_matches_brute_force_twin(seed, kind):
    rng = np.random.default_rng(300 + seed)
    lengths = rng.integers(1, 30, size=3)
    case = jagged_case(seed, lengths, H=2, d=5, dtype="f32", n_pos=9, n_time=7)
    args = dict(timestamps=case.timestamps, pos_table=case.pos_table, time_table=case.time_table,
                scale=-case.scale)
    got = oracle.attn_causal(case.q, case.k, case.v, case.seq_offsets, magnitude=kind, **args)
    ref = brute.causal(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                       case.pos_table, case.time_table, -case.scale, magnitude=kind)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    a = _cand_case(310 + seed, [0, 5, 23], [2, 1, 5], d=3, n_pos=6)
    np.testing.assert_allclose(oracle.attn_candidates(**a, magnitude=kind),
                               brute.candidates(**a, magnitude=kind), rtol=1e-12, atol=1e-12)


def test_magnitude_bounds_the_sum_and_equals_it_for_nonnegative_terms():
    case = jagged_case(21, [13, 40], H=2, d=4, dtype="f32", n_pos=16)
    f = lambda v, mag, rab: oracle.attn_causal(case.q, case.k, v, case.seq_offsets,
                                               pos_table=np.full(16, rab), scale=case.scale,
                                               magnitude=mag)
    # triangle inequality, term by term; |SiLU(s)| <= |s| for every s
    assert np.all(f(case.v, "silu", 0.1) >= np.abs(f(case.v, None, 0.1)))
    assert np.all(f(case.v, "score", 0.1) >= f(case.v, "silu", 0.1))
    # rab = 60 keeps every SiLU argument positive (|q.k| < 60 here) and |v| >= 0:
    # every term is non-negative, so the magnitude is the sum itself, bit for bit
    s = np.einsum("ihe,jhe->ihj", case.q.astype(np.float64), case.k.astype(np.float64))
    assert np.max(np.abs(s)) < 60
    v_pos = np.abs(case.v)
    assert np.array_equal(f(v_pos, "silu", 60.0), f(v_pos, None, 60.0))
    a = _cand_case(22, [7, 3], [2, 4])
    a["hist_v"], a["v_cand"] = np.abs(a["hist_v"]), np.abs(a["v_cand"])
    a["pos_table"] = np.full(16, 60.0)
    assert np.array_equal(oracle.attn_candidates(**a, magnitude="silu"), oracle.attn_candidates(**a))
