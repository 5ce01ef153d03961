"""Named, capture-sized cases for profiling the kernels (e.g. under ncu).

    python -m generative_recommender_sequence_b200.profile_cases <case> [--iters N]

cases:
  long_history_small  paged causal attention: 8 users {16384, 8226, 4096, 2048,
                      910, 548, 309, 64} tokens, 4 x 128, 16-bucket position
                      rab, 65536-token pool (the long_history kernel, small)
  jagged              the 8-user jagged bf16 workload (pos 128 + time 64 rab)
  cached_cand         the cached-candidate step's attention (8 users, 128
                      candidates each, paged history U[1024, 4096] + 64)
  block_layer         one HSTU block layer of the 8-user block workload
Each case runs ``--iters`` calls (default 4) and synchronises; inputs come from
the seeded generators in ``workloads``.
"""

from __future__ import annotations

import argparse
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
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


CASES = {"long_history_small": case_long_history_small, "jagged": case_jagged,
         "cached_cand": case_cached_cand, "block_layer": case_block_layer}


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
