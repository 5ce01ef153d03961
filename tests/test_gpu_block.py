"""hstu_block_fwd (GEMM + SiLU, attention, LayerNorm gate, GEMM + residual) vs the oracle.

Tolerance for bf16 tensors whose magnitude exceeds 1: a rounding flip of one
bf16 ulp is 2^-7 |x| at |x| in [1, 2) and more above; both sides round X to
bf16 at the same points, so a value may land one ulp apart.  Hence
|err| <= 1e-2 + 2^-7 |ref| elementwise, and rel-L2 <= 5e-3 overall.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_common import dev, storage, to_np

pytestmark = pytest.mark.gpu

ATOL, RTOL, REL_L2 = 1e-2, 2.0 ** -7, 5e-3


def assert_block_close(got, ref, what):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    rel_l2 = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    worst = float(np.max(err - bound))
    assert np.all(np.isfinite(got)) and worst <= 0 and rel_l2 <= REL_L2, \
        f"{what}: worst excess={worst:.3e} max_abs={err.max():.3e} rel_l2={rel_l2:.3e}"


def gpu_layers(case, x0, layers):
    """Run the stack one layer at a time through the C ABI; returns X after each layer."""
    import generative_recommender_sequence_b200 as hstu
    x = storage(x0, "bf16")
    off = dev(case.seq_offsets)
    w1 = [storage(case.w_uvqk[l], "bf16") for l in range(case.n_layers)]
    w2 = [storage(case.w_o[l], "bf16") for l in range(case.n_layers)]
    pt, tt, ts = dev(case.pos_table), dev(case.time_table), dev(case.timestamps)
    outs = []
    for l in layers:
        hstu.block_fwd(x, off, int(case.lengths.max()), [w1[l]], [w2[l]], pos_table=pt,
                       time_table=tt, timestamps=ts, scale=case.scale, H=case.H, dh=case.dh)
        outs.append(to_np(x).copy())
    torch.cuda.synchronize()
    assert hstu.last_device_error() == 0
    return outs


def oracle_layer(case, x_in, l, rows_of=None):
    return oracle.hstu_block(x_in, case.seq_offsets, case.w_uvqk[l:l + 1], case.w_o[l:l + 1],
                             case.timestamps, case.pos_table, case.time_table, case.scale,
                             H=case.H, dh=case.dh, round_bf16=True)


def test_block_small_per_layer_and_chain():
    case = workloads.block_case(31, [130, 257, 40], n_layers=2)
    outs = gpu_layers(case, case.x0, range(2))
    # per layer: the oracle layer applied to the GPU's own input
    x_in = case.x0
    for l in range(2):
        ref = oracle_layer(case, x_in, l)
        assert_block_close(outs[l], ref, f"layer {l}")
        x_in = outs[l]
    chain = oracle.hstu_block(case.x0, case.seq_offsets, case.w_uvqk, case.w_o, case.timestamps,
                              case.pos_table, case.time_table, case.scale, H=case.H, dh=case.dh)
    assert_block_close(outs[-1], chain, "2-layer chain")


def test_block_all_layers_in_one_call_equals_layer_by_layer():
    import generative_recommender_sequence_b200 as hstu
    case = workloads.block_case(32, [300, 129], n_layers=3)
    outs = gpu_layers(case, case.x0, range(3))
    x = storage(case.x0, "bf16")
    hstu.block_fwd(x, dev(case.seq_offsets), int(case.lengths.max()),
                   [storage(w, "bf16") for w in case.w_uvqk], [storage(w, "bf16") for w in case.w_o],
                   pos_table=dev(case.pos_table), time_table=dev(case.time_table),
                   timestamps=dev(case.timestamps), scale=case.scale)
    assert np.array_equal(to_np(x), outs[-1])


def test_block_stack_workload_full_size_one_user():
    """8 layers, 8 users, L~U[512,4096]: users are independent, so the oracle checks the
    shortest user's rows, layer by layer on the GPU's own inputs, and the 8-layer chain."""
    case = workloads.block_stack()
    outs = gpu_layers(case, case.x0, range(case.n_layers))
    b = int(np.argmin(case.lengths))
    s, e = int(case.seq_offsets[b]), int(case.seq_offsets[b + 1])
    sub = workloads.BlockCase("one_user", case.lengths[b:b + 1], np.array([0, e - s]), case.d_model,
                              case.H, case.dh, case.n_layers, case.x0[s:e], case.w_uvqk, case.w_o,
                              case.pos_table, case.time_table, case.timestamps[s:e], case.scale)
    x_in = sub.x0
    for l in (0, 3, 7):
        x_in = case.x0[s:e] if l == 0 else outs[l - 1][s:e]
        ref = oracle_layer(sub, x_in, l)
        assert_block_close(outs[l][s:e], ref, f"full size, layer {l}")
    # the 8-layer chain: rounding differences compound through the residual stream, so
    # the elementwise bound is looser (per-layer parity above is the contract)
    chain = oracle.hstu_block(sub.x0, sub.seq_offsets, sub.w_uvqk, sub.w_o, sub.timestamps,
                              sub.pos_table, sub.time_table, sub.scale, H=sub.H, dh=sub.dh)
    got = np.asarray(outs[-1][s:e], np.float64)
    rel_l2 = np.linalg.norm(got - chain) / np.linalg.norm(chain)
    assert rel_l2 <= REL_L2 and np.max(np.abs(got - chain)) <= 0.1, rel_l2
