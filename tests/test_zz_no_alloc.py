"""The allocation-free candidate-scoring entry point.

Callers that cannot allocate device memory while serving (a frozen allocator,
someone else's memory pool) call hstu_attn_cached_fwd_noalloc, which keeps its
split partial sums in a fixed array the library reserves at load time.  This
test calls it through the C ABI twice in a row and checks each result against
the regular entry point (which is given a caller-allocated workspace) within
the bf16 attention tolerance.  It lives in its own file, collected last, and
passes both alone in a fresh process and after the other GPU tests.
"""

import ctypes

import numpy as np
import pytest
import torch

import workloads
from tests.gpu_common import assert_bf16_close, dev, storage, to_np

pytestmark = pytest.mark.gpu


def test_noalloc_candidates_match_the_workspace_entry_point_twice():
    import generative_recommender_sequence_b200 as hstu
    lib = hstu.load()
    case = workloads.cached_cand(B=4, hmin=900, hmax=2600, n_new=48, n_cand=96, seed=11)
    mpp = int(np.max((case.total_lengths + 31) // 32)) + 2
    table = hstu.KVTable(case.n_pages, case.H, case.d, max_users=case.B, max_pages_per_user=mpp,
                         free_order=case.free_order)
    users = dev(case.users)
    hist = case.total_lengths
    ho = workloads.offsets_from_lengths(case.hist_lengths)
    table.alloc(users, dev(case.hist_lengths))
    table.append(users, storage(case.hist_k, "bf16"), storage(case.hist_v, "bf16"), dev(ho),
                 int(case.hist_lengths.max()))
    table.alloc(users, dev(case.n_new))
    table.append(users, storage(case.new_k, "bf16"), storage(case.new_v, "bf16"),
                 dev(workloads.offsets_from_lengths(case.n_new)), int(case.n_new.max()))
    assert table.status() == 0

    q, kc, vc = (storage(x, "bf16") for x in (case.q_cand, case.k_cand, case.v_cand))
    q_off = dev(case.q_offsets)
    pt = dev(case.pos_table)
    max_q, max_cached = int(case.n_cand.max()), int(hist.max())
    total_q = q.shape[0]

    ref = hstu.attn_cached_fwd(table, users, q, q_off, max_q, max_cached, hstu.HSTU_MASK_CANDIDATES,
                               k_cand=kc, v_cand=vc, pos_table=pt, scale=case.scale)
    torch.cuda.synchronize()
    need = table.workspace_size(case.B, total_q, max_q, max_cached, hstu.HSTU_MASK_CANDIDATES)
    assert 0 < need <= lib.hstu_attn_cached_noalloc_max_scratch()

    rab = hstu.HstuRab()
    rab.pos_table = pt.data_ptr()
    rab.n_pos_buckets = pt.numel()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        st = lib.hstu_attn_cached_fwd_noalloc(
            table.handle, users.data_ptr(), case.B, q.data_ptr(), kc.data_ptr(), vc.data_ptr(),
            q_off.data_ptr(), total_q, max_q, max_cached, hstu.HSTU_MASK_CANDIDATES,
            ctypes.byref(rab), float(case.scale), out.data_ptr(), stream)
        assert st == 0, f"call {call}: status {st}"
        torch.cuda.synchronize()
        assert table.status() == 0 and hstu.last_device_error() == 0
        assert_bf16_close(to_np(out), to_np(ref), f"noalloc call {call}")
    table.close()


def test_noalloc_rejects_work_beyond_its_scratch():
    """A problem whose split partials exceed the fixed array is refused on the host
    (no launch): one user whose 4096 query rows face a 60000-token history."""
    import generative_recommender_sequence_b200 as hstu
    lib = hstu.load()
    table = hstu.KVTable(64, 4, 128, max_users=2, max_pages_per_user=8)
    need = table.workspace_size(1, 4096, 128, 60000, hstu.HSTU_MASK_CANDIDATES)
    assert need > lib.hstu_attn_cached_noalloc_max_scratch()   # checked before any call
    dummy = torch.zeros(16, dtype=torch.int64, device="cuda")
    st = lib.hstu_attn_cached_fwd_noalloc(
        table.handle, dummy.data_ptr(), 1, dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(),
        dummy.data_ptr(), 4096, 128, 60000, hstu.HSTU_MASK_CANDIDATES, None, 1.0,
        dummy.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 4   # HSTU_ERR_UNSUPPORTED, refused before any launch
    table.close()
