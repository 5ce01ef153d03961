"""Beam decode attention over a shared paged context vs the oracle, steps 0-2."""

import numpy as np
import pytest
import torch

import workloads
from oracle.beam import attn_beam_decode as oracle_beam
from tests.gpu_common import assert_bf16_close, dev, magnitudes, storage, to_np

pytestmark = pytest.mark.gpu

H, D = 4, 128


def _bf16(rng, shape):
    return workloads._as_storage(rng.standard_normal(shape).astype(np.float32), "bf16")


@pytest.mark.parametrize("ctx,beams", [([300, 1000, 37], [16, 130, 5]), ([2048], [256])])
def test_beam_decode_steps_match_oracle(ctx, beams):
    import generative_recommender_sequence_b200 as hstu
    rng = np.random.default_rng(31)
    ctx, beams = np.array(ctx), np.array(beams)
    B = len(ctx)
    n_pages = int(np.sum((ctx + 31) // 32)) + 4
    t = hstu.KVTable(n_pages, H, D, max_users=B, max_pages_per_user=int((ctx.max() + 31) // 32) + 2,
                     free_order=rng.permutation(n_pages))
    users = dev(np.arange(B, dtype=np.int64))
    ck, cv = _bf16(rng, (int(ctx.sum()), H, D)), _bf16(rng, (int(ctx.sum()), H, D))
    co = workloads.offsets_from_lengths(ctx)
    t.alloc(users, dev(ctx.astype(np.int64)))
    t.append(users, storage(ck, "bf16"), storage(cv, "bf16"), dev(co), int(ctx.max()))
    bo = workloads.offsets_from_lengths(beams)
    T = int(bo[-1])
    steps = 3
    bk, bv = _bf16(rng, (steps, T, H, D)), _bf16(rng, (steps, T, H, D))
    parent = np.zeros((steps, T), np.int32)
    for s in range(1, steps):
        for b in range(B):
            parent[s, bo[b]:bo[b + 1]] = rng.integers(0, beams[b], size=beams[b])
    pt = rng.normal(0, 0.1, 16).astype(np.float32)
    scale = 1.0 / int(ctx.max() + steps)
    bk_d, bv_d, par_d = storage(bk, "bf16"), storage(bv, "bf16"), dev(parent)
    for s in range(steps):
        q = _bf16(rng, (T, H, D))
        out = hstu.attn_beam_decode(t, users, storage(q, "bf16"), dev(bo), int(beams.max()),
                                    int(ctx.max()), s, bk_d[:s + 1], bv_d[:s + 1],
                                    par_d[:s + 1] if s else None, pos_table=dev(pt), scale=scale)
        torch.cuda.synchronize()
        assert hstu.last_device_error() == 0 and t.status() == 0
        ref = oracle_beam(ck, cv, co, q, bo, s, bk[:s + 1], bv[:s + 1], parent[:s + 1],
                          pos_table=pt, scale=scale)
        mag = magnitudes(oracle_beam, ck, cv, co, q, bo, s, bk[:s + 1], bv[:s + 1], parent[:s + 1],
                         pos_table=pt, scale=scale)
        assert_bf16_close(to_np(out), ref, f"beam decode step {s}", mag=mag)
    t.close()
