"""Pin of the block oracle's bf16 rounding points (CPU only).

The GPU block stores four bf16 tensors per layer: [U|V|Q|K] after SiLU, the
attention output A, the gate output G = LayerNorm(A) * U and the new residual
stream X.  The oracle rounds at exactly those points ("How Generative
Recommenders Are Redefining RecSys at Scale", section "HSTU": projection, SiLU,
SiLU attention, elementwise gate before the output projection), so they are
part of the parity contract.

Here one layer is rebuilt from pieces pinned elsewhere -- a float64 torch matmul
and torch's silu, the attention oracle, torch's layer_norm -- each result rounded
with torch's bf16 conversion, and ``oracle.hstu_block(round_bf16=True)`` must
agree bit for bit.  The weights are scaled so that every intermediate is O(1),
so a rounding point that is dropped, moved or added changes many outputs.
Planted mistakes (a modified copy of the oracle source, compiled into a
temporary directory) must all break the pin.
"""

import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
from workloads import draw_timestamps, offsets_from_lengths

H, DH = 2, 8
F = H * DH
DM = F
LENGTHS = [7, 19, 12]
EPS = 1e-5


def _bf(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float64)).to(torch.bfloat16).to(
        torch.float64).numpy()


def _case(seed=11):
    rng = np.random.default_rng(seed)
    off = offsets_from_lengths(LENGTHS)
    T = int(off[-1])
    ts = draw_timestamps(rng, LENGTHS)
    pos = rng.normal(0, 0.1, 16)
    tim = rng.normal(0, 0.1, 8)
    x = _bf(rng.standard_normal((T, DM)))
    w1 = _bf(rng.normal(0, 0.35, (1, DM, 4 * F)))
    w2 = _bf(rng.normal(0, 0.35, (1, F, DM)))
    return dict(x=x, off=off, ts=ts, pos=pos, tim=tim, w1=w1, w2=w2, scale=1.0 / max(LENGTHS))


def _from_pieces(c, round_output=True):
    """One layer from separately pinned pieces, rounded where the GPU stores bf16."""
    x, T = c["x"], c["x"].shape[0]
    z = torch.from_numpy(x) @ torch.from_numpy(c["w1"][0])                    # fp64 matmul
    uvqk = _bf(torch.nn.functional.silu(z).numpy())                          # rounding point 1
    U, V, Q, K = (uvqk[:, i * F:(i + 1) * F] for i in range(4))
    a = oracle.attn_causal(Q.reshape(T, H, DH), K.reshape(T, H, DH), V.reshape(T, H, DH), c["off"],
                           timestamps=c["ts"], pos_table=c["pos"], time_table=c["tim"],
                           scale=c["scale"]).reshape(T, F)
    A = _bf(a)                                                               # rounding point 2
    ln = torch.nn.functional.layer_norm(torch.from_numpy(A), (F,), eps=EPS).numpy()
    G = _bf(ln * U)                                                          # rounding point 3
    y = x + (torch.from_numpy(G) @ torch.from_numpy(c["w2"][0])).numpy()
    return _bf(y) if round_output else y                                     # rounding point 4


def _oracle_layer(c, fn=None, round_output=True):
    if fn is None:
        return oracle.hstu_block(c["x"], c["off"], c["w1"], c["w2"], c["ts"], c["pos"], c["tim"],
                                 c["scale"], ln_eps=EPS, H=H, dh=DH, round_bf16=True,
                                 round_output=round_output, threads=1)
    x = np.ascontiguousarray(c["x"], np.float64).copy()
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    w1, w2 = np.ascontiguousarray(c["w1"]), np.ascontiguousarray(c["w2"])
    off, ts = np.ascontiguousarray(c["off"]), np.ascontiguousarray(c["ts"])
    pos, tim = np.ascontiguousarray(c["pos"]), np.ascontiguousarray(c["tim"])
    rc = fn(x.shape[0], len(off) - 1, p(off), 1, DM, H, DH, p(x), p(w1), p(w2), p(ts), p(pos),
            len(pos), p(tim), len(tim), c["scale"], EPS, 1, int(round_output), None, 1)
    assert rc == 0
    return x


def test_block_rounding_points_match_pinned_pieces_bit_for_bit():
    for seed in (11, 12, 13):
        c = _case(seed)
        ref = _from_pieces(c)
        got = _oracle_layer(c)
        assert np.array_equal(got, ref), f"seed {seed}: {np.sum(got != ref)} values differ"


def test_block_unrounded_output_is_the_value_before_the_last_rounding():
    c = _case(14)
    pre = _oracle_layer(c, round_output=False)
    np.testing.assert_allclose(pre, _from_pieces(c, round_output=False), rtol=1e-13, atol=1e-13)
    assert np.array_equal(_bf(pre), _oracle_layer(c))
    assert not np.array_equal(pre, _bf(pre))


def test_block_rounding_changes_many_outputs():
    """The pin is sensitive: the unrounded stack differs from the rounded one almost everywhere."""
    c = _case(15)
    exact = oracle.hstu_block(c["x"], c["off"], c["w1"], c["w2"], c["ts"], c["pos"], c["tim"],
                              c["scale"], ln_eps=EPS, H=H, dh=DH, round_bf16=False)
    assert np.mean(exact != _oracle_layer(c)) > 0.5


# Planted mistakes: (what, text in the oracle source, replacement).  Rounding G a
# second time at the same point is idempotent (RNE of a bf16 value is itself),
# so the "extra rounding" mutants round at a different point instead.
MUTANTS = [
    ("UVQK not rounded",
     "gemm_ctx g1 = {x, w_uvqk + (int64_t)l * dm * N1, uvqk, dm, N1, 1, round_bf16};",
     "gemm_ctx g1 = {x, w_uvqk + (int64_t)l * dm * N1, uvqk, dm, N1, 1, 0};"),
    ("UVQK rounded before the SiLU",
     "        if (g->act_silu) s = oracle_silu(s);",
     "        if (g->act_silu) s = oracle_silu(g->round ? oracle_round_bf16(s) : s);"),
    ("A not rounded",
     "for (int64_t i = 0; i < T * F; i++) a[i] = oracle_round_bf16(a[i]);",
     "for (int64_t i = 0; i < T * F; i++) a[i] = a[i];"),
    ("G not rounded",
     "lngate_ctx lc = {a, uvqk, N1, g, F, ln_eps, round_bf16};",
     "lngate_ctx lc = {a, uvqk, N1, g, F, ln_eps, 0};"),
    ("LayerNorm(A) rounded before the gate",
     "double y = (a[f] - mean) * inv * u[f];",
     "double y = (c->round ? oracle_round_bf16((a[f] - mean) * inv) : (a[f] - mean) * inv) * u[f];"),
    ("G W2 rounded before the residual add",
     "double y = x[i] + d[i];",
     "double y = x[i] + (round_bf16 ? oracle_round_bf16(d[i]) : d[i]);"),
    ("X not rounded",
     "x[i] = round_x ? oracle_round_bf16(y) : y;",
     "x[i] = y;"),
]


@pytest.fixture(scope="module")
def oracle_source():
    with open(os.path.join(os.path.dirname(oracle.__file__), "hstu_oracle.c")) as f:
        return f.read()


@pytest.mark.parametrize("what,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_rounding_mistake_breaks_the_pin(tmp_path, oracle_source, what, old, new):
    assert oracle_source.count(old) == 1, f"mutation site for '{what}' not found"
    src = tmp_path / "mutant.c"
    src.write_text(oracle_source.replace(old, new))
    lib_path = str(tmp_path / "libmutant.so")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                           "-shared", "-pthread", "-o", lib_path, str(src), "-lm"])
    lib = ctypes.CDLL(lib_path)
    fn = lib.oracle_hstu_block
    fn.argtypes = oracle._load().oracle_hstu_block.argtypes
    fn.restype = ctypes.c_int
    caught = False
    for seed in (11, 12, 13):
        c = _case(seed)
        if not np.array_equal(_oracle_layer(c, fn), _from_pieces(c)):
            caught = True
            break
    assert caught, f"planted mistake '{what}' passes the rounding-point pin"
