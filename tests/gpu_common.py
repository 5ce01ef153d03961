"""Shared helpers for the GPU parity tests (tolerances from the build's contract)."""

import numpy as np
import torch

import workloads

BF16_MAX_ABS = 1e-2
BF16_REL_L2 = 5e-3
F32_REL = 1e-5


def dev(x, dtype=None):
    t = torch.as_tensor(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def storage(x, dtype: str):
    return workloads.to_torch(x, dtype).cuda()


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = got - ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    rel_l2 = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300)) if diff.size else 0.0
    max_rel = max_abs / max(float(np.max(np.abs(ref))), 1e-300) if diff.size else 0.0
    return max_abs, rel_l2, max_rel


# Rounding a value x to bf16 (round to nearest even) moves it by at most half an
# ulp, i.e. at most 2^-8 |x| (8 significand bits).
BF16_HALF_ULP_REL = 2.0 ** -8


def magnitudes(fn, *args, **kw):
    """The oracle's term-by-term magnitudes of an attention sum (``fn`` is
    oracle.attn_causal, oracle.attn_candidates or the beam oracle)."""
    return fn(*args, magnitude="silu", **kw), fn(*args, magnitude="score", **kw)


def assert_bf16_close(got, ref, what="", mag=None):
    """The contract bound: max-abs <= 1e-2 and rel-L2 <= 5e-3.

    mag = (silu, score) from ``magnitudes``: for edge-case inputs (few keys, so a
    large 1/N) the elementwise bound follows the kernel's arithmetic instead:
      |err| <= 1e-2 + 2^-8 |ref| + 2^-8 silu + 2^-11 score
    - 2^-8 |ref|: the final rounding of the output to bf16 (half an ulp);
    - 2^-8 silu: each SiLU weight P is rounded to bf16 before the tensor-core
      product (at most 2^-9 |P| per term, doubled for the fp32 sums);
    - 2^-11 score: SiLU(s) = h + h tanh(h) with h = s / 2 and tanh.approx.f32,
      whose error is at most ~2^-11 in absolute terms, i.e. 2^-12 |s| per term,
      doubled;
    where silu = |scale| sum_j |SiLU(s_j)| |v_j| and score = |scale| sum_j |s_j| |v_j|
    (the oracle's magnitudes).  rel-L2 stays 5e-3."""
    max_abs, rel_l2, _ = errors(got, ref)
    got64 = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got64)), what
    if mag is not None:
        ref64 = np.asarray(ref, dtype=np.float64)
        silu, score = (np.asarray(m, dtype=np.float64) for m in mag)
        bound = (BF16_MAX_ABS + BF16_HALF_ULP_REL * np.abs(ref64) + 2.0 ** -8 * silu +
                 2.0 ** -11 * score)
        excess = float(np.max(np.abs(got64 - ref64) - bound))
        assert excess <= 0 and rel_l2 <= BF16_REL_L2, \
            f"{what}: max_abs={max_abs:.3e} excess={excess:.3e} rel_l2={rel_l2:.3e}"
    else:
        assert max_abs <= BF16_MAX_ABS and rel_l2 <= BF16_REL_L2, \
            f"{what}: max_abs={max_abs:.3e} rel_l2={rel_l2:.3e}"
    return max_abs, rel_l2


def assert_f32_close(got, ref, what=""):
    _, rel_l2, max_rel = errors(got, ref)
    assert rel_l2 <= F32_REL and max_rel <= F32_REL, f"{what}: rel_l2={rel_l2:.3e} max_rel={max_rel:.3e}"
    return rel_l2, max_rel


def to_np(t):
    return t.detach().float().cpu().numpy()


def sample_rows(offsets, n_random, seed=0):
    """Rows to check at full size: first/last rows of every user and every 128-row tile
    boundary, plus random rows."""
    rng = np.random.default_rng(seed)
    rows = set()
    for b in range(len(offsets) - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        if e <= s:
            continue
        rows.update([s, e - 1])
        for t in range(s, e, 128):
            rows.update([t, min(t + 127, e - 1)])
    T = int(offsets[-1])
    if T:
        rows.update(rng.integers(0, T, size=n_random).tolist())
    return np.array(sorted(rows), dtype=np.int64)
