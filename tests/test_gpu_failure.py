"""Failure detection without a GPU fault: a bounded wait that runs out (an
mbarrier that nothing completes, a short limit) reports HSTU_ERR_TIMEOUT to the
host, the error word clears once read, and the same context keeps computing."""

import time

import pytest
import torch

import oracle
import workloads
from tests.gpu_common import assert_bf16_close, dev, magnitudes, storage, to_np

pytestmark = pytest.mark.gpu

HSTU_ERR_TIMEOUT = 5


def test_bounded_wait_timeout_is_reported_and_the_context_survives():
    import generative_recommender_sequence_b200 as hstu
    assert hstu.last_device_error() == 0
    t0 = time.perf_counter()
    hstu.wait_timeout_selftest(20000)              # 20 ms limit
    assert hstu.last_device_error() == HSTU_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 10.0
    assert hstu.last_device_error() == 0           # read once, then cleared
    # the tcgen05 attention still runs correctly in the same context
    case = workloads.jagged_case(71, [5, 130, 300], H=4, d=128, dtype="bf16", n_pos=16)
    q, k, v = (storage(x, "bf16") for x in (case.q, case.k, case.v))
    out = hstu.attn_fwd(q, k, v, dev(case.seq_offsets), case.max_len, pos_table=dev(case.pos_table),
                        scale=case.scale)
    torch.cuda.synchronize()
    assert hstu.last_device_error() == 0
    ref = oracle.attn_causal(case.q, case.k, case.v, case.seq_offsets, pos_table=case.pos_table,
                             scale=case.scale)
    mag = magnitudes(oracle.attn_causal, case.q, case.k, case.v, case.seq_offsets,
                     pos_table=case.pos_table, scale=case.scale)
    assert_bf16_close(to_np(out), ref, "attention after a reported timeout", mag=mag)
