"""Named, capture-sized cases for profiling the kernels (e.g. under ncu).

    python profile_cases.py <case> [--iters N]

cases:
  long_history_small  paged causal attention: 8 users {16384, 8226, 4096, 2048,
                      910, 548, 309, 64} tokens, 4 x 128, 16-bucket position
                      rab, 65536-token pool (the long_history kernel, small)
  jagged              the 8-user jagged bf16 workload (pos 128 + time 64 rab)
  cached_cand         the cached-candidate step's attention + split reduce (8
                      users, 128 candidates each, paged history U[1024, 4096] + 64)
  block_layer         one HSTU block layer of the 8-user block workload (GEMM +
                      SiLU, attention, LayerNorm gate, GEMM + residual)
  kv_step             the cached-candidate step's KV step (alloc + append of 64
                      tokens per user + lookup rows, 8 users)
  kv_append_bulk      append of the long-history workload's whole histories
                      (77k tokens, 158 MB of K/V) into fresh pages
  beam_decode         one beam-search decode step at step 2 (8 requests x 5000
                      context tokens, 256 beams each)
Each case runs ``--iters`` calls (default 4) and synchronises; inputs come from
the seeded generators in ``workloads``.
"""

from __future__ import annotations

import argparse
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import generative_recommender_sequence_b200 as hstu  # noqa: E402
import workloads as W  # noqa: E402


def _dev(a, dt=None):
    return (torch.as_tensor(np.ascontiguousarray(a)) if dt is None else W.to_torch(a, dt)).cuda()


def _filled_table(c):
    mpp = int(np.max((c.total_lengths + 31) // 32)) + 2
    t = hstu.KVTable(c.n_pages, c.H, c.d, max_users=c.B, max_pages_per_user=mpp, free_order=c.free_order)
    u = _dev(c.users)
    t.alloc(u, _dev(c.hist_lengths))
    if int(c.hist_lengths.max()) > 0:
        t.append(u, _dev(c.hist_k, "bf16"), _dev(c.hist_v, "bf16"),
                 _dev(W.offsets_from_lengths(c.hist_lengths)), int(c.hist_lengths.max()))
    t.alloc(u, _dev(c.n_new))
    if int(c.n_new.sum()) > 0:
        t.append(u, _dev(c.new_k, "bf16"), _dev(c.new_v, "bf16"),
                 _dev(W.offsets_from_lengths(c.n_new)), int(c.n_new.max()))
    if t.status() != 0:
        raise RuntimeError("KV table device error")
    return t, u


def case_long_history_small(iters):
    c = W.long_history(lengths=[16384, 8226, 4096, 2048, 910, 548, 309, 64], pool_tokens=65536)
    t, u = _filled_table(c)
    q, qo, pt = _dev(c.q, "bf16"), _dev(c.q_offsets), _dev(c.pos_table)
    out = torch.empty_like(q)
    for _ in range(iters):
        hstu.attn_cached_fwd(t, u, q, qo, int(c.n_q.max()), int(c.total_lengths.max()),
                             hstu.HSTU_MASK_CAUSAL_SUFFIX, pos_table=pt, scale=c.scale, out=out)
    return c.flops()


def case_jagged(iters):
    c = W.jagged_bf16()
    q, k, v = (_dev(x, "bf16") for x in (c.q, c.k, c.v))
    args = dict(pos_table=_dev(c.pos_table), time_table=_dev(c.time_table),
                timestamps=_dev(c.timestamps), scale=c.scale)
    out = torch.empty_like(q)
    off = _dev(c.seq_offsets)
    for _ in range(iters):
        hstu.attn_fwd(q, k, v, off, c.max_len, out=out, **args)
    return c.flops()


def case_cached_cand(iters):
    c = W.cached_cand()
    t, u = _filled_table(c)
    q, kc, vc = (_dev(x, "bf16") for x in (c.q_cand, c.k_cand, c.v_cand))
    out = torch.empty_like(q)
    for _ in range(iters):
        hstu.attn_cached_fwd(t, u, q, _dev(c.q_offsets), 128, int(c.total_lengths.max()),
                             hstu.HSTU_MASK_CANDIDATES, k_cand=kc, v_cand=vc,
                             pos_table=_dev(c.pos_table), scale=c.scale, out=out)
    return c.flops()


def case_block_layer(iters):
    c = W.block_stack()
    x = _dev(c.x0, "bf16")
    w1, w2 = [_dev(c.w_uvqk[0], "bf16")], [_dev(c.w_o[0], "bf16")]
    for _ in range(iters):
        hstu.block_fwd(x, _dev(c.seq_offsets), int(c.lengths.max()), w1, w2,
                       pos_table=_dev(c.pos_table), time_table=_dev(c.time_table),
                       timestamps=_dev(c.timestamps), scale=c.scale)
    return c.flops() / c.n_layers


def case_kv_step(iters):
    c = W.cached_cand()
    mpp = int(np.max((c.total_lengths + 31) // 32)) + 2
    t = hstu.KVTable(c.n_pages, c.H, c.d, max_users=c.B, max_pages_per_user=mpp,
                     free_order=c.free_order)
    u = _dev(c.users)
    hist, hoff = _dev(c.hist_lengths), _dev(W.offsets_from_lengths(c.hist_lengths))
    hk, hv = _dev(c.hist_k, "bf16"), _dev(c.hist_v, "bf16")
    nk, nv = _dev(c.new_k, "bf16"), _dev(c.new_v, "bf16")
    noff = _dev(W.offsets_from_lengths(c.n_new))
    lens = torch.empty(c.B, dtype=torch.int64, device="cuda")
    ptab = torch.empty((c.B, mpp), dtype=torch.int32, device="cuda")
    for _ in range(iters):
        # back to the prefilled state, then the step
        t.release(u)
        t.alloc(u, hist)
        t.append(u, hk, hv, hoff, int(c.hist_lengths.max()))
        t.step(u, nk, nv, noff, int(c.n_new.max()), lens, ptab)
    if t.status() != 0:
        raise RuntimeError("KV table device error")
    return 0.0


def case_kv_append_bulk(iters):
    c = W.long_history()
    mpp = int(np.max((c.total_lengths + 31) // 32)) + 2
    t = hstu.KVTable(c.n_pages, c.H, c.d, max_users=c.B, max_pages_per_user=mpp,
                     free_order=c.free_order)
    u = _dev(c.users)
    hist, hoff = _dev(c.hist_lengths), _dev(W.offsets_from_lengths(c.hist_lengths))
    hk, hv = _dev(c.hist_k, "bf16"), _dev(c.hist_v, "bf16")
    for _ in range(iters):
        t.release(u)
        t.alloc(u, hist)
        t.append(u, hk, hv, hoff, int(c.hist_lengths.max()))
    if t.status() != 0:
        raise RuntimeError("KV table device error")
    return 0.0


def case_beam_decode(iters):
    rng = np.random.default_rng(77)
    B, L, Wb, steps, H, D = 8, 5000, 256, 3, 4, 128
    bf = lambda shape: W.to_torch(W._as_storage(rng.standard_normal(shape).astype(np.float32),
                                                "bf16"), "bf16").cuda()
    t = hstu.KVTable(B * ((L + 31) // 32) + 4, H, D, max_users=B, max_pages_per_user=(L + 31) // 32 + 2)
    u = torch.arange(B, dtype=torch.int64, device="cuda")
    t.alloc(u, torch.full((B,), L, dtype=torch.int64, device="cuda"))
    t.append(u, bf((B * L, H, D)), bf((B * L, H, D)),
             torch.arange(0, B * L + 1, L, dtype=torch.int64, device="cuda"), L)
    T = B * Wb
    q, bk, bv = bf((T, H, D)), bf((steps, T, H, D)), bf((steps, T, H, D))
    par = np.zeros((steps, T), np.int32)
    for s_ in range(1, steps):
        par[s_] = np.concatenate([rng.integers(0, Wb, size=Wb) for _ in range(B)])
    parent = torch.as_tensor(par).cuda()
    bo = torch.arange(0, T + 1, Wb, dtype=torch.int64, device="cuda")
    pt = torch.as_tensor(rng.normal(0, 0.1, 16).astype(np.float32)).cuda()
    out = torch.empty_like(q)
    for _ in range(iters):
        hstu.attn_beam_decode(t, u, q, bo, Wb, L, steps - 1, bk, bv, parent, pos_table=pt,
                              scale=1.0 / (L + steps), out=out)
    if t.status() != 0:
        raise RuntimeError("KV table device error")
    return float(T) * (L + steps) * H * D * 4


CASES = {"long_history_small": case_long_history_small, "jagged": case_jagged,
         "cached_cand": case_cached_cand, "block_layer": case_block_layer,
         "kv_step": case_kv_step, "kv_append_bulk": case_kv_append_bulk,
         "beam_decode": case_beam_decode}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=sorted(CASES))
    ap.add_argument("--iters", type=int, default=4)
    a = ap.parse_args()
    torch.cuda.set_device(0)
    flops = CASES[a.case](a.iters)
    torch.cuda.synchronize()
    if hstu.last_device_error() != 0:
        raise RuntimeError("a device wait timed out")
    print(f"{a.case}: ok ({flops:.3e} flop per call)")


if __name__ == "__main__":
    main()
