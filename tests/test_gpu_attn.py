"""hstu_attn_fwd on the GPU vs the fp64 oracle (jagged causal attention)."""

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_common import (assert_bf16_close, assert_f32_close, dev, magnitudes, sample_rows,
                              storage, to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    import generative_recommender_sequence_b200 as hstu
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    hstu.device_check()


def case_magnitudes(case, rows=None):
    return magnitudes(oracle.attn_causal, case.q, case.k, case.v, case.seq_offsets,
                      timestamps=case.timestamps, pos_table=case.pos_table,
                      time_table=case.time_table, scale=case.scale, rows=rows)


def run_case(case, rows=None, stream=None):
    import generative_recommender_sequence_b200 as hstu
    q, k, v = (storage(x, case.dtype) for x in (case.q, case.k, case.v))
    off = dev(case.seq_offsets)
    pt = dev(case.pos_table)
    tt = dev(case.time_table) if case.time_table is not None else None
    ts = dev(case.timestamps) if case.timestamps is not None else None
    out = hstu.attn_fwd(q, k, v, off, case.max_len, pos_table=pt, time_table=tt, timestamps=ts,
                        scale=case.scale)
    torch.cuda.synchronize()
    assert hstu.last_device_error() == 0
    got = to_np(out)
    ref = oracle.attn_causal(case.q, case.k, case.v, case.seq_offsets, timestamps=case.timestamps,
                             pos_table=case.pos_table, time_table=case.time_table, scale=case.scale,
                             rows=rows)
    return (got if rows is None else got[rows]), ref


def test_tiny_fp32_workload():
    case = workloads.tiny_fp32()
    got, ref = run_case(case)
    assert_f32_close(got, ref, "tiny fp32")


@pytest.mark.parametrize("d", [32, 64, 128])
def test_fp32_head_dims(d):
    case = workloads.jagged_case(50 + d, [1, 70, 129, 5], H=3, d=d, dtype="f32", n_pos=16, n_time=8)
    got, ref = run_case(case)
    assert_f32_close(got, ref, f"fp32 d={d}")


@pytest.mark.parametrize("d", [32, 64])
def test_bf16_simt_head_dims(d):
    case = workloads.jagged_case(60 + d, [3, 100, 257], H=2, d=d, dtype="bf16", n_pos=32, n_time=16)
    got, ref = run_case(case)
    assert_bf16_close(got, ref, f"bf16 simt d={d}")


@pytest.mark.parametrize("lengths", [
    [128] * 300,                # many one-tile users: item-to-item hand-offs
    [256] * 64 + [1] * 7,       # two-tile users and single tokens
    [130, 300, 517],            # several tiles, ragged tails
    [1, 128, 129, 255, 256],    # tile-boundary edge cases
    [0, 7, 0, 384, 0],          # empty users
    [1000],
])
def test_bf16_tcgen05_pos_rab(lengths):
    # edge shapes: short users make scale = 1/max_len large, so outputs reach a few
    # units and one bf16 ulp exceeds 1e-2 -> the ulp-aware elementwise bound
    case = workloads.jagged_case(7, lengths, H=4, d=128, dtype="bf16", n_pos=16)
    got, ref = run_case(case)
    assert_bf16_close(got, ref, f"bf16 {lengths[:8]}...", mag=case_magnitudes(case))


@pytest.mark.parametrize("lengths", [[100, 50, 128, 1], [7]])
def test_bf16_tcgen05_few_short_users(lengths):
    """Few users of at most one query tile: fewer items than SMs, and no
    workspace to split keys into, so every item streams all of its keys."""
    case = workloads.jagged_case(14, lengths, H=4, d=128, dtype="bf16", n_pos=32, n_time=16)
    got, ref = run_case(case)
    assert_bf16_close(got, ref, f"short users {lengths}", mag=case_magnitudes(case))


def test_bf16_tcgen05_over_1024_users():
    """1100 short users: the launch runs as chunks of at most 1024 users over
    absolute rows (position + time bias)."""
    rng = np.random.default_rng(15)
    lengths = rng.integers(1, 40, size=1100)
    case = workloads.jagged_case(15, lengths, H=2, d=128, dtype="bf16", n_pos=16, n_time=8)
    got, ref = run_case(case)
    assert_bf16_close(got, ref, "1100 users", mag=case_magnitudes(case))


@pytest.mark.parametrize("lengths,what", [
    ([200] * 148, "8 rounds: the largest batch the round-balanced plan takes"),
    ([200] * 149, "9 rounds: decoded item by item in the snake order"),
    ([16500, 100, 3, 300], "129 query-tile levels: decoded item by item"),
])
def test_bf16_tcgen05_schedule_bounds(lengths, what):
    """Contiguous causal launches plan a round-balanced item order in every
    CTA when the batch fits the planner's tables (at most 8 rounds of the SM
    count, 128 query-tile levels) and otherwise decode the snake order one
    item at a time; both must cover every (user, head, query tile) once."""
    case = workloads.jagged_case(16, lengths, H=4, d=128, dtype="bf16", n_pos=16, n_time=8)
    rows = sample_rows(case.seq_offsets, 400)
    got, ref = run_case(case, rows=rows)
    assert_bf16_close(got, ref, what, mag=case_magnitudes(case, rows=rows))


def test_bf16_tcgen05_pos_time_rab():
    case = workloads.jagged_case(8, [200, 640, 37, 1100], H=4, d=128, dtype="bf16", n_pos=128,
                                 n_time=64)
    got, ref = run_case(case)
    assert_bf16_close(got, ref, "pos+time rab")


def _bucket_reach(ts, off, n):
    """Largest unclamped time bucket over visible pairs (floor(log2(max(dt,0)+1)))."""
    best = 0
    for b in range(len(off) - 1):
        t = ts[off[b]:off[b + 1]]
        dt = np.maximum(t[:, None] - t[None, :], 0)[np.tril_indices(len(t))]
        best = max(best, int(np.floor(np.log2(dt.max() + 1))))
    return best


EDGE_TS = [
    ("increasing", 3 * 86400, 128, 64),   # spans of years: integer time buckets
    ("unordered", 3, 128, 64),            # equal and decreasing neighbours: max(dt, 0)
    ("unordered", 300, 4, 4),             # both tables clamp at n - 1
    ("increasing", 20 * 86400, 4, 4),     # clamps on the integer time path
]


@pytest.mark.parametrize("kind,gap,n_pos,n_time", EDGE_TS)
def test_bf16_tcgen05_rab_edge_timestamps_and_tables(kind, gap, n_pos, n_time):
    """Time-gap bias branches that the workloads' Exp(300 s) gaps never reach."""
    lengths = [700, 129, 1500, 64]
    case = workloads.jagged_case(12, lengths, H=4, d=128, dtype="bf16", n_pos=n_pos,
                                 n_time=n_time, ts_gap_mean=gap, ts_kind=kind)
    ts, off = case.timestamps, case.seq_offsets
    spans = [int(ts[off[b + 1] - 1] - ts[off[b]]) for b in range(len(lengths))]
    steps = np.concatenate([np.diff(ts[off[b]:off[b + 1]]) for b in range(len(lengths))])
    if kind == "increasing" and gap > 86400:
        assert max(spans) > 2 ** 23            # offsets leave the exact float range
    if kind == "unordered":
        assert np.any(steps == 0) and np.any(steps < 0)
    if n_time == 4:
        assert _bucket_reach(ts, off, n_time) > n_time - 1   # the time clamp bites
        assert max(lengths) > 2 ** n_pos                      # so does the position clamp
    got, ref = run_case(case)
    assert_bf16_close(got, ref, f"{kind} gaps {gap}, tables {n_pos}/{n_time}")


@pytest.mark.parametrize("d,dtype", [(32, "f32"), (64, "bf16")])
@pytest.mark.parametrize("kind,gap", [("increasing", 3 * 86400), ("unordered", 3)])
def test_simt_rab_edge_timestamps_and_tables(d, dtype, kind, gap):
    case = workloads.jagged_case(13, [90, 300, 17], H=2, d=d, dtype=dtype, n_pos=4, n_time=4,
                                 ts_gap_mean=gap, ts_kind=kind)
    got, ref = run_case(case)
    if dtype == "f32":
        assert_f32_close(got, ref, f"simt fp32 {kind}")
    else:
        assert_bf16_close(got, ref, f"simt bf16 {kind}")


def test_bf16_no_rab_and_single_head():
    import generative_recommender_sequence_b200 as hstu
    case = workloads.jagged_case(9, [300, 45], H=1, d=128, dtype="bf16", n_pos=16)
    q, k, v = (storage(x, "bf16") for x in (case.q, case.k, case.v))
    out = hstu.attn_fwd(q, k, v, dev(case.seq_offsets), case.max_len, scale=case.scale)
    ref = oracle.attn_causal(case.q, case.k, case.v, case.seq_offsets, scale=case.scale)
    assert_bf16_close(to_np(out), ref, "no rab")


def test_jagged_bf16_workload_full_size_sampled():
    """The 8-user, L~U[256,2048] workload at full size; oracle on sampled rows."""
    case = workloads.jagged_bf16()
    rows = sample_rows(case.seq_offsets, 1500)
    got, ref = run_case(case, rows=rows)
    assert_bf16_close(got, ref, "jagged_bf16 workload")


def test_causality_and_determinism_on_gpu():
    import generative_recommender_sequence_b200 as hstu
    case = workloads.jagged_case(10, [600, 300], H=4, d=128, dtype="bf16", n_pos=16)
    q, k, v = (storage(x, "bf16") for x in (case.q, case.k, case.v))
    off, pt = dev(case.seq_offsets), dev(case.pos_table)
    a = hstu.attn_fwd(q, k, v, off, 600, pos_table=pt, scale=case.scale).clone()
    b = hstu.attn_fwd(q, k, v, off, 600, pos_table=pt, scale=case.scale).clone()
    assert torch.equal(a, b)
    i = 250
    k2, v2 = k.clone(), v.clone()
    k2[i + 1:600] = -k2[i + 1:600]
    v2[i + 1:600] += 1
    c = hstu.attn_fwd(q, k2, v2, off, 600, pos_table=pt, scale=case.scale)
    assert torch.equal(a[: i + 1], c[: i + 1])
    assert torch.equal(a[600:], c[600:])   # the other user is untouched


def test_k_zero_rab_zero_gives_zero_on_gpu():
    import generative_recommender_sequence_b200 as hstu
    case = workloads.jagged_case(11, [333], H=2, d=128, dtype="bf16", n_pos=16)
    q, v = storage(case.q, "bf16"), storage(case.v, "bf16")
    k = torch.zeros_like(q)
    out = hstu.attn_fwd(q, k, v, dev(case.seq_offsets), 333, pos_table=torch.zeros(16, device="cuda"),
                        scale=case.scale)
    assert torch.count_nonzero(out) == 0
