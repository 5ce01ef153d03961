"""The seeded input generators follow the five configurations they stand for:
shapes, length ranges, timestamp structure, page pools, weight scales, bf16-exact
storage values and seed determinism (no arithmetic of the method is involved)."""

import numpy as np

import workloads as W


def _bf16_exact(x: np.ndarray) -> bool:
    u = np.ascontiguousarray(x.reshape(-1)[:200_000], dtype=np.float32).view(np.uint32)
    return not np.any(u & 0xFFFF)


def test_tiny_fp32_is_config_1():
    c = W.tiny_fp32()
    assert c.lengths.tolist() == [17, 40] and c.H == 2 and c.d == 32 and c.dtype == "f32"
    assert c.q.shape == (57, 2, 32) and c.pos_table.shape == (16,)
    assert c.time_table is None and c.timestamps is None
    assert c.scale == 1.0 / 40


def test_jagged_bf16_is_config_2():
    c = W.jagged_bf16()
    assert c.B == 8 and c.H == 4 and c.d == 128 and c.dtype == "bf16"
    assert c.lengths.min() >= 256 and c.lengths.max() <= 2048
    assert c.pos_table.shape == (128,) and c.time_table.shape == (64,)
    assert abs(c.pos_table.std() - 0.1) < 0.03
    assert c.scale == 1.0 / c.max_len
    ts, off = c.timestamps, c.seq_offsets
    gaps = []
    for b in range(c.B):
        t = ts[off[b]:off[b + 1]]
        assert t[0] == W.TS0
        g = np.diff(t)
        assert g.min() >= 1                       # strictly increasing, whole seconds
        gaps.append(g)
    g = np.concatenate(gaps)
    assert abs(g.mean() - (W.GAP_MEAN_S + 0.5)) < 0.05 * W.GAP_MEAN_S   # 1 + floor(Exp(300))
    assert all(_bf16_exact(x) for x in (c.q, c.k, c.v))


def test_cached_cand_is_config_3():
    c = W.cached_cand()
    assert c.B == 8 and c.H == 4 and c.d == 128 and c.mode == 0
    assert c.hist_lengths.min() >= 1024 and c.hist_lengths.max() <= 4096
    assert np.all(c.n_new == 64) and np.all(c.n_cand == 128)
    assert c.hist_k.shape == (int(c.hist_lengths.sum()), 4, 128)
    assert c.new_k.shape == (8 * 64, 4, 128) and c.q_cand.shape == (8 * 128, 4, 128)
    need = int(np.sum((c.hist_lengths + 64 + W.PAGE - 1) // W.PAGE))
    assert c.n_pages >= need
    assert sorted(c.free_order.tolist()) == list(range(c.n_pages))   # a shuffled pool
    assert c.scale == 1.0 / int((c.hist_lengths + 64 + 128).max())
    assert all(_bf16_exact(x) for x in (c.hist_k, c.hist_v, c.new_k, c.q_cand, c.k_cand, c.v_cand))


def test_block_stack_is_config_4():
    c = W.block_stack()
    assert c.B == 8 and c.n_layers == 8 and c.d_model == 512 and c.H == 4 and c.dh == 128
    assert c.lengths.min() >= 512 and c.lengths.max() <= 4096
    assert c.x0.shape == (c.T, 512)
    assert c.w_uvqk.shape == (8, 512, 2048) and c.w_o.shape == (8, 512, 512)
    assert abs(c.w_uvqk.std() - 0.02) < 0.001 and abs(c.w_o.std() - 0.02) < 0.001
    assert abs(c.x0.std() - 1.0) < 0.02
    assert c.pos_table.shape == (128,) and c.time_table.shape == (64,)
    assert c.timestamps.shape == (c.T,)
    assert all(_bf16_exact(x) for x in (c.x0, c.w_uvqk, c.w_o))


def test_long_history_is_config_5():
    c = W.long_history()
    L = c.total_lengths
    assert c.B == 32 and c.H == 4 and c.d == 128 and c.mode == 1
    assert L.min() >= 64 and L.max() <= 16384
    assert np.all(c.n_new == 16)                       # each step appends 16 per user
    assert np.array_equal(c.n_q, L)                    # causal over the full history
    assert c.n_pages == 2 * 1024 * 1024 // W.PAGE      # the 2M-token pool
    assert sorted(c.free_order.tolist()) == list(range(c.n_pages))
    assert c.scale == 1.0 / int(L.max())
    assert all(_bf16_exact(x) for x in (c.q, c.hist_k, c.new_v))


def test_generators_are_seed_deterministic():
    a, b = W.cached_cand(), W.cached_cand()
    assert np.array_equal(a.hist_lengths, b.hist_lengths)
    assert np.array_equal(a.free_order, b.free_order)
    assert np.array_equal(a.q_cand, b.q_cand) and np.array_equal(a.hist_v, b.hist_v)
    c, d = W.tiny_fp32(), W.tiny_fp32()
    assert np.array_equal(c.q, d.q) and np.array_equal(c.pos_table, d.pos_table)
    e = W.cached_cand(seed=1004)
    assert not np.array_equal(e.hist_lengths, a.hist_lengths)
