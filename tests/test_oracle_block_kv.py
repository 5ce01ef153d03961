"""Pins for the bf16 rounding, LayerNorm gate, block stack and KV-table oracles (CPU only)."""

import json
import os

import numpy as np
import torch

import oracle
from oracle.kv import INVALID_ARG, OK, OUT_OF_PAGES, KVTableOracle, to_bits
from workloads import block_case, offsets_from_lengths


def test_round_bf16_matches_torch_on_fp32_values():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),   # fp32 subnormals
        (rng.standard_normal(2000) * 1e30).astype(np.float32),
        # exact ties: bf16 value + half an ulp, both parities of the kept bit
        (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        np.array([3.3895e38, 3.4e38, -3.4e38, 0.0, -0.0], dtype=np.float32),
    ])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_bf16(x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_layernorm_gate_with_unit_gate_is_layer_norm():
    rng = np.random.default_rng(1)
    a = rng.standard_normal((37, 512)) * 3 + 0.5
    got = oracle.layernorm_gate(a, np.ones_like(a), eps=1e-5)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(a), (512,), eps=1e-5).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    u = rng.standard_normal(a.shape)
    np.testing.assert_allclose(oracle.layernorm_gate(a, u), ref * u, rtol=1e-12, atol=1e-12)


def _tiny_block(n_layers=2, lengths=(5, 9), H=2, dh=4):
    return block_case(21, list(lengths), n_layers, d_model=H * dh, H=H, dh=dh)


def test_block_zero_output_projection_is_identity():
    c = _tiny_block()
    x = oracle.hstu_block(c.x0, c.seq_offsets, c.w_uvqk, np.zeros_like(c.w_o), c.timestamps,
                          c.pos_table, c.time_table, c.scale, H=c.H, dh=c.dh, round_bf16=False)
    assert np.array_equal(x, c.x0.astype(np.float64))


def test_block_selector_weights_reduce_to_pinned_pieces():
    """W1 copies slices of X into [U|V|Q|K] and W2 = I: one layer must equal
    X + layer_norm(attn(SiLU(X_q), SiLU(X_k), SiLU(X_v))) * SiLU(X_u),
    built from torch's silu / layer_norm and the (separately pinned) attention oracle."""
    H, dh = 2, 4
    F = H * dh
    rng = np.random.default_rng(3)
    lengths = [4, 7]
    off = offsets_from_lengths(lengths)
    T = int(off[-1])
    x = rng.standard_normal((T, F))
    # W1 columns: U <- x, V <- -x, Q <- 0.5 x, K <- x reversed
    w1 = np.zeros((1, F, 4 * F))
    w1[0, :, 0:F] = np.eye(F)
    w1[0, :, F:2 * F] = -np.eye(F)
    w1[0, :, 2 * F:3 * F] = 0.5 * np.eye(F)
    w1[0, :, 3 * F:4 * F] = np.eye(F)[::-1]
    w2 = np.eye(F)[None]
    pos_table = rng.normal(0, 0.1, 16)
    ts = np.arange(T, dtype=np.int64) * 7
    time_table = rng.normal(0, 0.1, 8)
    got = oracle.hstu_block(x, off, w1, w2, ts, pos_table, time_table, 0.1, H=H, dh=dh,
                            round_bf16=False)
    silu = lambda z: torch.nn.functional.silu(torch.from_numpy(z)).numpy()
    U, V, Q, K = silu(x), silu(-x), silu(0.5 * x), silu(x[:, ::-1].copy())
    A = oracle.attn_causal(Q.reshape(T, H, dh), K.reshape(T, H, dh), V.reshape(T, H, dh), off,
                           timestamps=ts, pos_table=pos_table, time_table=time_table,
                           scale=0.1).reshape(T, F)
    ln = torch.nn.functional.layer_norm(torch.from_numpy(A), (F,), eps=1e-5).numpy()
    np.testing.assert_allclose(got, x + ln * U, rtol=1e-12, atol=1e-12)


def test_block_rounding_points_are_bf16():
    c = _tiny_block(n_layers=1)
    x = oracle.hstu_block(c.x0, c.seq_offsets, c.w_uvqk, c.w_o, c.timestamps, c.pos_table,
                          c.time_table, c.scale, H=c.H, dh=c.dh, round_bf16=True)
    assert np.array_equal(oracle.round_bf16(x), x)
    x_exact = oracle.hstu_block(c.x0, c.seq_offsets, c.w_uvqk, c.w_o, c.timestamps, c.pos_table,
                                c.time_table, c.scale, H=c.H, dh=c.dh, round_bf16=False)
    assert np.max(np.abs(x - x_exact)) < 5e-2


def test_block_layers_compose():
    """Two layers at once == layer 1 applied to the output of layer 0."""
    c = _tiny_block(n_layers=2)
    args = (c.timestamps, c.pos_table, c.time_table, c.scale)
    x2, layers = oracle.hstu_block(c.x0, c.seq_offsets, c.w_uvqk, c.w_o, *args, H=c.H, dh=c.dh,
                                   return_layers=True)
    x1 = oracle.hstu_block(c.x0, c.seq_offsets, c.w_uvqk[:1], c.w_o[:1], *args, H=c.H, dh=c.dh)
    x2b = oracle.hstu_block(x1, c.seq_offsets, c.w_uvqk[1:], c.w_o[1:], *args, H=c.H, dh=c.dh)
    assert np.array_equal(layers[0], x1) and np.array_equal(x2, x2b) and np.array_equal(layers[1], x2)


# ---------------------------------------------------------------- KV table

def test_kv_hand_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "kv_hand_example.json")))
    H, d = 1, 2
    t = KVTableOracle(g["n_pages"], g["page_size"], H, d, g["max_users"], 8, g["free_order"])
    rng = np.random.default_rng(5)
    written = {0: [], 1: []}
    for st in g["steps"]:
        if st["op"] == "alloc":
            status, pages = t.alloc(st["users"], st["n_new"])
            assert status == st["status"] and pages == st["new_pages"], st
        elif st["op"] == "append":
            n = st["n_new"]
            kv = rng.standard_normal((2, sum(n), H, d)).astype(np.float32)
            kv = torch.from_numpy(kv).to(torch.bfloat16).float().numpy()
            assert t.append(st["users"], kv[0], kv[1], offsets_from_lengths(n)) == st["status"]
            o = offsets_from_lengths(n)
            for b, u in enumerate(st["users"]):
                written[u].append(kv[:, o[b]:o[b + 1]])
        else:
            lens, table, k, v = t.lookup(st["users"], st["max_pages"])
            assert lens.tolist() == st["lengths"] and table.tolist() == st["page_table"]
            ref = np.concatenate([np.concatenate(written[u], axis=1) for u in st["users"]], axis=1)
            assert np.array_equal(k, to_bits(ref[0], "bf16"))
            assert np.array_equal(v, to_bits(ref[1], "bf16"))
    # explicit slot placement from the hand derivation: user 1 token 4 -> page 4 slot 0
    k1 = np.concatenate(written[1], axis=1)[0]
    assert np.array_equal(t.pool[4, 0, :, 0, :], to_bits(k1[4], "bf16"))
    assert np.array_equal(t.pool[0, 0, :, 0, :], to_bits(k1[8], "bf16"))


def test_kv_roundtrip_and_page_accounting():
    rng = np.random.default_rng(6)
    P, H, d = 32, 2, 8
    t = KVTableOracle(200, P, H, d, 5, 64, rng.permutation(200))
    sent = {u: [] for u in range(5)}
    for step in range(4):
        users = rng.permutation(5)[:3]
        n = rng.integers(0, 70, size=3)
        assert t.alloc(users, n)[0] == OK
        kv = torch.from_numpy(rng.standard_normal((2, int(n.sum()), H, d)).astype(np.float32))
        kv = kv.to(torch.bfloat16).float().numpy()
        assert t.append(users, kv[0], kv[1], offsets_from_lengths(n)) == OK
        o = offsets_from_lengths(n)
        for b, u in enumerate(users):
            sent[u].append(kv[:, o[b]:o[b + 1]])
    users = np.arange(5)
    lens, table, k, v = t.lookup(users, 64)
    for u in range(5):
        held = int((table[u] >= 0).sum())
        assert held == -(-lens[u] // P)
    ref = np.concatenate([np.concatenate(sent[u], axis=1) for u in users], axis=1)
    assert np.array_equal(k, to_bits(ref[0], "bf16")) and np.array_equal(v, to_bits(ref[1], "bf16"))
    used = set(table[table >= 0].tolist())
    assert len(used) == int((table >= 0).sum()) and used.isdisjoint(t.stack)
    assert len(used) + t.n_free == 200


def test_kv_errors_leave_table_unchanged():
    t = KVTableOracle(4, 4, 1, 2, 3, 8, [0, 1, 2, 3])
    assert t.alloc([0, 1], [8, 9]) == (OUT_OF_PAGES, [])
    assert t.n_free == 4 and t.pages[0] == [] and t.pages[1] == []
    assert t.alloc([0, 0], [1, 1])[0] == INVALID_ARG
    assert t.alloc([0], [4]) == (OK, [3])
    kv = np.zeros((5, 1, 2), np.float32)
    assert t.append([0], kv, kv, [0, 5]) == INVALID_ARG   # only 4 slots reserved
    assert t.length[0] == 0


def test_kv_release_hand_example():
    # free order 0..5 (top = 5); pages of 4 tokens
    t = KVTableOracle(6, 4, 1, 2, 3, 8, [0, 1, 2, 3, 4, 5])
    assert t.alloc([0, 1], [9, 2]) == (OK, [5, 4, 3, 2])
    assert t.pages[0] == [5, 4, 3] and t.pages[1] == [2] and t.stack == [0, 1]
    # user 1 first, then user 0; each user's pages go back last to first
    assert t.release([1, 0]) == OK
    assert t.stack == [0, 1, 2, 3, 4, 5]
    assert t.pages[0] == [] and t.pages[1] == [] and t.length[0] == 0
    # the next user gets user 0's first pages back, in the same order
    assert t.alloc([2], [5]) == (OK, [5, 4])


def test_kv_release_errors_and_accounting():
    t = KVTableOracle(6, 4, 1, 2, 3, 8, [0, 1, 2, 3, 4, 5])
    assert t.alloc([0], [6])[0] == OK
    before = (list(t.stack), [list(p) for p in t.pages], list(t.length))
    assert t.release([0, 0]) == INVALID_ARG
    assert t.release([3]) == INVALID_ARG
    assert (t.stack, t.pages, t.length) == before
    # random alloc / append / release sequences keep every page exactly once
    rng = np.random.default_rng(8)
    t = KVTableOracle(64, 4, 1, 2, 6, 64, rng.permutation(64))
    for _ in range(40):
        users = rng.permutation(6)[:rng.integers(1, 4)].tolist()
        if rng.random() < 0.4:
            assert t.release(users) == OK
            assert all(t.length[u] == 0 and t.pages[u] == [] for u in users)
        else:
            n = rng.integers(0, 9, size=len(users))
            if t.alloc(users, n)[0] == OK:
                kv = np.zeros((int(n.sum()), 1, 2), np.float32)
                assert t.append(users, kv, kv, offsets_from_lengths(n)) == OK
        held = [p for u in range(6) for p in t.pages[u]]
        assert len(held) + t.n_free == 64 and set(held).isdisjoint(t.stack)
        assert all(len(t.pages[u]) == -(-t.length[u] // 4) for u in range(6))
