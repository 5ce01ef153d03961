"""hstu_block_cached_step (KV-cached multi-layer serving) vs the oracle's full
recomputation, and vs the GPU's own uncached block.

The contract is per-layer parity, as for the uncached block: each layer runs as
its own cached step (prefill, then the step) and the oracle layer is fed the
GPU's own inputs to that layer (history, new and candidate rows), with every
bf16 rounding point except the final one; the bound is |err| <= 1e-2 + 2^-8
|ref| (half an ulp of the GPU's final rounding) and rel-L2 <= 5e-3.  Whole
multi-layer runs are reported as a diagnostic and checked with rel-L2 <= 5e-3
only: a rounding point that lands one bf16 ulp apart at one layer moves every
later layer."""

import numpy as np
import pytest
import torch

from oracle.cached import hstu_block_cached
from tests.gpu_common import BF16_HALF_ULP_REL, dev, storage, to_np

pytestmark = pytest.mark.gpu

DM, H, DH = 512, 4, 128


def _bf16(a):
    import workloads
    return workloads._as_storage(np.asarray(a, np.float32), "bf16")


def _offsets(n):
    return np.concatenate([[0], np.cumsum(n)]).astype(np.int64)


def _layer_close(got, ref, what):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    worst = float(np.max(err - (1e-2 + BF16_HALF_ULP_REL * np.abs(ref))))
    rel_l2 = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert np.all(np.isfinite(got)) and worst <= 0 and rel_l2 <= 5e-3, \
        f"{what}: worst excess={worst:.3e} max_abs={err.max():.3e} rel_l2={rel_l2:.3e}"


def _chain_diagnostic(got, ref, what):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    rel_l2 = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    print(f"{what}: chain max_abs={np.max(np.abs(got - ref)):.3e} rel_l2={rel_l2:.3e}")
    assert np.all(np.isfinite(got)) and rel_l2 <= 5e-3, f"{what}: rel_l2={rel_l2:.3e}"


def _setup(hist, new, cand, n_layers, seed):
    rng = np.random.default_rng(seed)
    c = dict(hist=np.array(hist), new=np.array(new), cand=np.array(cand))
    c["x_hist"] = _bf16(rng.standard_normal((sum(hist), DM)))
    c["x_new"] = _bf16(rng.standard_normal((sum(new), DM)))
    c["x_cand"] = _bf16(rng.standard_normal((sum(cand), DM)))
    c["w1"] = _bf16(rng.normal(0, 0.02, (n_layers, DM, 4 * H * DH)))
    c["w2"] = _bf16(rng.normal(0, 0.02, (n_layers, H * DH, DM)))
    c["pt"] = rng.normal(0, 0.1, 16).astype(np.float32)
    c["scale"] = 1.0 / int((c["hist"] + c["new"] + c["cand"]).max())
    return c


def _tables(c, layers):
    import generative_recommender_sequence_b200 as hstu
    B = len(c["hist"])
    total = c["hist"] + c["new"]
    mpp = int(np.max((total + 31) // 32)) + 2
    n_pages = int(np.sum((total + 31) // 32)) + 8
    return [hstu.KVTable(n_pages, H, DH, max_users=B, max_pages_per_user=mpp,
                         free_order=np.random.default_rng(40 + l).permutation(n_pages))
            for l in layers]


def _step(c, tables, layers, xh, x):
    """Prefill (history as new rows on empty tables) then the step, over `layers`;
    xh and x are updated in place."""
    import generative_recommender_sequence_b200 as hstu
    B = len(c["hist"])
    total = c["hist"] + c["new"]
    users = dev(np.arange(B, dtype=np.int64))
    w1 = [storage(c["w1"][l], "bf16") for l in layers]
    w2 = [storage(c["w2"][l], "bf16") for l in layers]
    pt = dev(c["pt"])
    if c["hist"].sum() > 0:
        hstu.block_cached_step(tables, users, xh, dev(_offsets(c["hist"])), int(c["hist"].max()),
                               None, 0, int(c["hist"].max()), w1, w2, pos_table=pt, scale=c["scale"])
    hstu.block_cached_step(tables, users, x, dev(_offsets(c["new"])), int(c["new"].max()),
                           dev(_offsets(c["cand"])), int(c["cand"].max()), int(total.max()), w1, w2,
                           pos_table=pt, scale=c["scale"], T_new=int(c["new"].sum()))
    torch.cuda.synchronize()
    assert hstu.last_device_error() == 0
    for t in tables:
        assert t.status() == 0


def _run_gpu(c, n_layers):
    """All layers in one cached call; returns (new rows, candidate rows) after the last."""
    tables = _tables(c, range(n_layers))
    xh = storage(c["x_hist"], "bf16")
    x = storage(np.concatenate([c["x_new"], c["x_cand"]]), "bf16")
    _step(c, tables, list(range(n_layers)), xh, x)
    for t in tables:
        t.close()
    T_new = int(c["new"].sum())
    out = to_np(x)
    return out[:T_new], out[T_new:]


def _run_gpu_layerwise(c, n_layers):
    """One cached call per layer; returns the inputs and outputs of every layer as
    (history rows, new rows, candidate rows)."""
    T_new = int(c["new"].sum())
    xh = storage(c["x_hist"], "bf16")
    x = storage(np.concatenate([c["x_new"], c["x_cand"]]), "bf16")
    ins, outs = [], []
    for l in range(n_layers):
        ins.append((to_np(xh).copy(), to_np(x)[:T_new].copy(), to_np(x)[T_new:].copy()))
        tables = _tables(c, [l])
        _step(c, tables, [l], xh, x)
        tables[0].close()
        outs.append((to_np(xh).copy(), to_np(x)[:T_new].copy(), to_np(x)[T_new:].copy()))
    return ins, outs


def _oracle(c, layers, x_hist, x_new, x_cand, round_output=True):
    l0, l1 = layers[0], layers[-1] + 1
    return hstu_block_cached(x_hist, _offsets(c["hist"]), x_new, _offsets(c["new"]),
                             x_cand, _offsets(c["cand"]), c["w1"][l0:l1], c["w2"][l0:l1], c["pt"],
                             c["scale"], H=H, dh=DH, round_bf16=True, round_output=round_output)


@pytest.mark.parametrize("hist,new,cand", [
    ([0, 37, 300], [16, 16, 5], [8, 3, 4]),    # a new user, a ragged page tail, several tiles
    ([130, 1], [1, 40], [1, 130]),             # single new token, candidates over one tile
])
def test_cached_step_matches_full_recompute(hist, new, cand):
    c = _setup(hist, new, cand, n_layers=2, seed=7)
    ins, outs = _run_gpu_layerwise(c, 2)
    for l in range(2):
        ref_new, ref_c = _oracle(c, [l], *ins[l], round_output=False)
        _layer_close(outs[l][1], ref_new, f"new rows, layer {l}")
        _layer_close(outs[l][2], ref_c, f"candidate rows, layer {l}")
    # the one-call two-layer step gives the layer-by-layer result, bit for bit
    got_new, got_c = _run_gpu(c, 2)
    assert np.array_equal(got_new, outs[1][1]) and np.array_equal(got_c, outs[1][2])
    ref_new, ref_c = _oracle(c, [0, 1], c["x_hist"], c["x_new"], c["x_cand"])
    _chain_diagnostic(got_new, ref_new, "new rows")
    _chain_diagnostic(got_c, ref_c, "candidate rows")


def test_cached_new_rows_match_the_uncached_gpu_block():
    """The new tokens' outputs equal the GPU's uncached block over [history; new]."""
    import generative_recommender_sequence_b200 as hstu
    c = _setup([200, 64], [24, 8], [0, 0], n_layers=3, seed=9)
    got_new, _ = _run_gpu(c, 3)
    seqs = []
    ho, no = _offsets(c["hist"]), _offsets(c["new"])
    for b in range(2):
        seqs.append(np.concatenate([c["x_hist"][ho[b]:ho[b + 1]], c["x_new"][no[b]:no[b + 1]]]))
    full = np.concatenate(seqs)
    lens = c["hist"] + c["new"]
    x = storage(full, "bf16")
    hstu.block_fwd(x, dev(_offsets(lens)), int(lens.max()),
                   [storage(c["w1"][l], "bf16") for l in range(3)],
                   [storage(c["w2"][l], "bf16") for l in range(3)], pos_table=dev(c["pt"]),
                   scale=c["scale"])
    torch.cuda.synchronize()
    y = to_np(x)
    fo = _offsets(lens)
    ref = np.concatenate([y[fo[b] + c["hist"][b]:fo[b + 1]] for b in range(2)])
    _chain_diagnostic(got_new, ref, "cached vs uncached GPU")
