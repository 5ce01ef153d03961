"""The allocation-free candidate-scoring entry point.

Callers that cannot allocate device memory while serving (a frozen allocator,
someone else's memory pool) call hstu_attn_cached_fwd_noalloc, which keeps its
split partial sums in a fixed array the library reserves at load time.  This
test calls it through the C ABI twice in a row and checks each result against
the regular entry point (which is given a caller-allocated workspace) within
the bf16 attention tolerance, and against the fp64 oracle; the device's free
memory is unchanged across the two calls.  It lives in its own file, collected
last, and passes both alone in a fresh process and after the other GPU tests.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_common import assert_bf16_close, dev, magnitudes, storage, to_np

pytestmark = pytest.mark.gpu


def _oracle_candidates(case, magnitude=None):
    ho = workloads.offsets_from_lengths(case.hist_lengths)
    no = workloads.offsets_from_lengths(case.n_new)
    ks, vs = [], []
    for b in range(case.B):
        ks += [case.hist_k[ho[b]:ho[b + 1]], case.new_k[no[b]:no[b + 1]]]
        vs += [case.hist_v[ho[b]:ho[b + 1]], case.new_v[no[b]:no[b + 1]]]
    return oracle.attn_candidates(np.concatenate(ks), np.concatenate(vs),
                                  workloads.offsets_from_lengths(case.total_lengths), case.q_cand,
                                  case.k_cand, case.v_cand, case.q_offsets,
                                  pos_table=case.pos_table, scale=case.scale, magnitude=magnitude)


def _noalloc(lib, table, users, case, q, kc, vc, q_off, max_q, max_cached, rab, out, mask=0):
    return lib.hstu_attn_cached_fwd_noalloc(
        table.handle, users.data_ptr(), case.B, q.data_ptr(), kc.data_ptr(), vc.data_ptr(),
        q_off.data_ptr(), q.shape[0], max_q, max_cached, mask, ctypes.byref(rab),
        float(case.scale), out.data_ptr(), torch.cuda.current_stream().cuda_stream)


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
    outs = [torch.full_like(q, float("nan")) for _ in range(3)]
    # warm-up call: loads the module and looks the scratch address up
    assert _noalloc(lib, table, users, case, q, kc, vc, q_off, max_q, max_cached, rab, outs[2]) == 0
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for call in range(2):
        st = _noalloc(lib, table, users, case, q, kc, vc, q_off, max_q, max_cached, rab, outs[call])
        assert st == 0, f"call {call}: status {st}"
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before   # the calls allocated nothing
    ref_oracle = _oracle_candidates(case)
    for call in range(2):
        assert table.status() == 0 and hstu.last_device_error() == 0
        assert_bf16_close(to_np(outs[call]), to_np(ref), f"noalloc call {call} vs workspace call")
        assert_bf16_close(to_np(outs[call]), ref_oracle, f"noalloc call {call} vs oracle")
    table.close()


def test_noalloc_over_1024_users():
    """1025 users: the first 1024 run without a key split, the last user alone
    splits its keys; the scratch must hold that chunk's partials and the result
    must match the workspace entry point and the oracle."""
    import generative_recommender_sequence_b200 as hstu
    from tests.test_gpu_cached import many_user_case, make_table, prefill
    lib = hstu.load()
    case = many_user_case()
    table = make_table(case)
    users = dev(case.users)
    prefill(table, case, users)
    q, kc, vc = (storage(x, "bf16") for x in (case.q_cand, case.k_cand, case.v_cand))
    q_off, pt = dev(case.q_offsets), dev(case.pos_table)
    max_cached = int(case.total_lengths.max())
    ref = hstu.attn_cached_fwd(table, users, q, q_off, 4, max_cached, hstu.HSTU_MASK_CANDIDATES,
                               k_cand=kc, v_cand=vc, pos_table=pt, scale=case.scale)
    rab = hstu.HstuRab()
    rab.pos_table = pt.data_ptr()
    rab.n_pos_buckets = pt.numel()
    out = torch.full_like(q, float("nan"))
    assert _noalloc(lib, table, users, case, q, kc, vc, q_off, 4, max_cached, rab, out) == 0
    torch.cuda.synchronize()
    assert table.status() == 0 and hstu.last_device_error() == 0
    assert torch.equal(out, ref)
    assert_bf16_close(to_np(out), _oracle_candidates(case), "noalloc, 1025 users",
                      mag=magnitudes(lambda **kw: _oracle_candidates(case, **kw)))
    table.close()


def test_noalloc_scratch_covers_the_largest_split_and_checks_arguments_first():
    """Key-split partial sums take one [128, 128] fp32 block per SM plus a small
    per-user table, whatever the history length, so even one user facing a
    60000-token history fits the fixed array.  Invalid arguments are reported
    as such, exactly as the workspace entry point reports them."""
    import generative_recommender_sequence_b200 as hstu
    lib = hstu.load()
    table = hstu.KVTable(64, 4, 128, max_users=2, max_pages_per_user=8)
    for mask in (hstu.HSTU_MASK_CANDIDATES, hstu.HSTU_MASK_CAUSAL_SUFFIX):
        need = table.workspace_size(1, 4096, 128, 60000, mask)
        assert 0 < need <= lib.hstu_attn_cached_noalloc_max_scratch()
    dummy = torch.zeros(16, dtype=torch.int64, device="cuda")
    for mask in (7, -1):
        st = lib.hstu_attn_cached_fwd_noalloc(
            table.handle, dummy.data_ptr(), 1, dummy.data_ptr(), dummy.data_ptr(),
            dummy.data_ptr(), dummy.data_ptr(), 4096, 128, 60000, mask, None, 1.0,
            dummy.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == 1   # HSTU_ERR_INVALID_ARG
    table.close()
