#!/usr/bin/env python
"""Benchmark of the HSTU attention hot path on B200.

One step = one pass of the hot path over one batch of synthetic input:
  1. jagged causal HSTU attention, workload ``jagged_bf16`` (8 users,
     L ~ U[256, 2048], 4 heads x 128, bf16, 128-bucket position + 64-bucket
     time-gap rab, scale 1/max_len);
  2. cached-candidate scoring, workload ``cached_cand`` (8 users with a paged
     history L ~ U[1024, 4096], 100% KV hit): KV alloc + append of 64 new
     tokens per user, lookup, then 128 candidates per user attend to the whole
     cached history plus themselves (K/V read page by page in the kernel).
Every step appends into fresh pages (the pool is sized for all steps), so the
history grows by 64 tokens per user per step; FLOPs/bytes are counted from the
actual lengths of every step.

value = attention FLOPs of all steps (both parts, unmasked pairs only) / time,
in TFLOP/s.  Cached candidates/s and the HBM fraction of the candidate step are
reported beside it.  Inputs are resident in HBM; L2 is flushed (256 MiB write)
between steps, outside the per-step CUDA events.

``--impl reference`` times the fp64 CPU oracle (the only reference this build
has) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HSTU attn TFLOP/s (% bf16 peak) & cached candidates/sec (% HBM BW), 1 B200"
WORKLOAD = ("jagged_bf16 (B=8, L~U[256,2048], H=4, d=128, bf16, pos128+time64 rab) + "
            "cached_cand (B=8, paged history U[1024,4096], +64 appended, 128 candidates/user)")


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained"), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if self.proc is None:
            return out
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return out
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        out.update(sm_mhz=float(np.median(sm)) if sm else None, sm_max_mhz=max(mx) if mx else None,
                   reasons=sorted(reasons), samples=len(rows))
        return out


def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


class Workloads:
    """Device-resident inputs of both parts of the step, plus a KV table sized for all steps."""

    def __init__(self, n_steps_total):
        import torch
        import generative_recommender_sequence_b200 as hstu
        import workloads as W
        self.hstu = hstu
        c2 = W.jagged_bf16()
        self.c2 = c2
        dev = lambda a, dt=None: (torch.as_tensor(np.ascontiguousarray(a)) if dt is None else
                                  W.to_torch(a, dt)).cuda()
        self.q, self.k, self.v = (dev(x, "bf16") for x in (c2.q, c2.k, c2.v))
        self.off = dev(c2.seq_offsets)
        self.pt, self.tt, self.ts = dev(c2.pos_table), dev(c2.time_table), dev(c2.timestamps)
        self.out = torch.empty_like(self.q)
        self.c2_flops = c2.flops()
        # cached candidates
        c3 = W.cached_cand()
        self.c3 = c3
        extra = c3.B * n_steps_total * ((int(c3.n_new[0]) + 31) // 32 + 1)
        n_pages = c3.n_pages + extra
        rng = np.random.default_rng(77)
        order = np.concatenate([c3.free_order, c3.n_pages + rng.permutation(extra)]).astype(np.int32)
        max_hist = int(c3.hist_lengths.max()) + n_steps_total * int(c3.n_new.max())
        self.max_ppu = (max_hist + 31) // 32 + 2
        self.table = hstu.KVTable(n_pages, c3.H, c3.d, max_users=c3.B, max_pages_per_user=self.max_ppu,
                                  free_order=order)
        self.users = dev(c3.users)
        hist_off = W.offsets_from_lengths(c3.hist_lengths)
        self.table.alloc(self.users, dev(c3.hist_lengths))
        self.table.append(self.users, dev(c3.hist_k, "bf16"), dev(c3.hist_v, "bf16"), dev(hist_off),
                          int(c3.hist_lengths.max()))
        assert self.table.status() == 0
        self.n_new = dev(c3.n_new)
        self.new_off = dev(W.offsets_from_lengths(c3.n_new))
        self.new_k, self.new_v = dev(c3.new_k, "bf16"), dev(c3.new_v, "bf16")
        self.q_c, self.k_c, self.v_c = (dev(x, "bf16") for x in (c3.q_cand, c3.k_cand, c3.v_cand))
        self.q_off = dev(c3.q_offsets)
        self.pt3 = dev(c3.pos_table)
        self.out_c = torch.empty_like(self.q_c)
        self.cached_len = torch.empty(c3.B, dtype=torch.int64, device="cuda")
        self.page_table = torch.empty((c3.B, self.max_ppu), dtype=torch.int32, device="cuda")
        self.hist_now = c3.hist_lengths.copy()
        self.max_cached = max_hist + int(c3.n_new.max())
        need = self.table.workspace_size(c3.B, int(c3.q_offsets[-1]), 128, self.max_cached, 0)
        self.ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
        self.flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")

    def c3_units(self):
        """(flops, algorithmic bytes) of the next candidate step (history before the append)."""
        c3 = self.c3
        L = (self.hist_now + c3.n_new).astype(np.float64)
        flops = float((c3.n_cand * (L + 1)).sum() * c3.H * 4 * c3.d)
        row = c3.H * c3.d * 2
        bytes_ = float((L * 2 * row).sum() + (c3.n_new * 2 * row * 2).sum()
                       + c3.n_cand.sum() * row * 4)
        return flops, bytes_

    def flush(self):
        self.flush_buf.fill_(1)

    def part_c2(self, stream=None):
        self.hstu.attn_fwd(self.q, self.k, self.v, self.off, self.c2.max_len, pos_table=self.pt,
                           time_table=self.tt, timestamps=self.ts, scale=self.c2.scale, out=self.out,
                           stream=stream)

    def part_c3(self, stream=None):
        h, t = self.hstu, self.table
        t.alloc(self.users, self.n_new, stream=stream)
        t.append(self.users, self.new_k, self.new_v, self.new_off, int(self.c3.n_new.max()), stream=stream)
        t.lookup(self.users, self.cached_len, self.page_table, stream=stream)
        h.attn_cached_fwd(t, self.users, self.q_c, self.q_off, 128, self.max_cached,
                          h.HSTU_MASK_CANDIDATES, k_cand=self.k_c, v_cand=self.v_c,
                          pos_table=self.pt3, scale=self.c3.scale, out=self.out_c,
                          workspace=self.ws, stream=stream)
        self.hist_now = self.hist_now + self.c3.n_new


def run_gpu(args):
    import torch
    rank, world, local = dist_setup(args.gpus)
    hbm_peak, tf_peak, tf_sus, peak_src = load_peaks()
    wl = Workloads(args.warmup + args.steps + 2)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        wl.flush()
        wl.part_c2()
        wl.part_c3()
    torch.cuda.synchronize()
    if wl.table.status() != 0 or wl.hstu.last_device_error() != 0:
        raise RuntimeError("device error during warm-up")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    flops_total, c3_flops, c3_bytes = 0.0, 0.0, 0.0
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    if rank == 0:
        sampler.start()
        time.sleep(0.25)
    wall0 = time.perf_counter()
    for i in range(args.steps):
        wl.flush()
        f3, b3 = wl.c3_units()
        ev[i][0].record()
        wl.part_c2()
        ev[i][1].record()
        wl.part_c3()
        ev[i][2].record()
        flops_total += wl.c2_flops + f3
        c3_flops += f3
        c3_bytes += b3
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - wall0
    clocks = sampler.stop() if rank == 0 else None
    t_c2 = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3
    t_c3 = sum(e[1].elapsed_time(e[2]) for e in ev) / 1e3
    t_step = t_c2 + t_c3
    if wl.table.status() != 0 or wl.hstu.last_device_error() != 0:
        raise RuntimeError("device error during the timed steps")
    t_max = max_over_ranks(t_step, world)
    flops_all = sum_over_ranks(flops_total, world)
    value = flops_all / t_max / 1e12
    c2_tflops = wl.c2_flops * args.steps / t_c2 / 1e12
    cand_per_s = float(wl.c3.n_cand.sum()) * args.steps / t_c3
    c3_gbs = c3_bytes / t_c3 / 1e9

    e2e = run_e2e(wl, args) if rank == 0 else None
    cpu = cpu_baseline(args) if (rank == 0 and world == 1 and not args.no_cpu) else None
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_step / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; shapes of the pages' benchmark, KuaiRand-1K not available)",
            "config": {"workload": WORKLOAD, "global_batch": 16 * world, "seq_len": int(wl.c2.max_len),
                       "parallelism": f"dp{world} (users sharded, no collective on the data path)",
                       "l2": "flushed between steps (256 MiB write, outside the step events)"},
            "parts": {
                "jagged_causal": {"ms": round(t_c2 / args.steps * 1e3, 4), "tflops": round(c2_tflops, 2),
                                  "frac_of_bf16_peak": round(c2_tflops / tf_peak, 4)},
                "cached_candidates": {"ms": round(t_c3 / args.steps * 1e3, 4),
                                      "candidates_per_s": round(cand_per_s, 1),
                                      "hbm_gbs": round(c3_gbs, 1), "frac_of_hbm": round(c3_gbs * 1e9 / (hbm_peak * 1e9), 4)},
            },
            "cached_candidates_per_s": round(cand_per_s * world, 1),
            "roofline": {"bound": "tensor", "kernel": "hstu_attn_sm100_kernel (jagged causal part)",
                         "achieved": round(c2_tflops, 2), "peak": tf_peak, "unit": "TFLOP/s",
                         "frac": round(c2_tflops / tf_peak, 4), "traffic": None,
                         "peak_source": f"{peak_src} bf16 dense (burst)"},
            "gpu_launches": args.steps * 6,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "wall_s": round(wall, 3),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(wl, args):
    """Same metric through the public API with host (pinned) inputs: H2D of the step's
    inputs and D2H of its outputs are inside the timed region."""
    import torch
    hq = [x.cpu().pin_memory() for x in (wl.q, wl.k, wl.v, wl.q_c, wl.k_c, wl.v_c, wl.new_k, wl.new_v)]
    dq = [torch.empty_like(x, device="cuda") for x in hq]
    ho = torch.empty_like(wl.out, device="cpu").pin_memory()
    hoc = torch.empty_like(wl.out_c, device="cpu").pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in hq)
    d2h = ho.numel() * ho.element_size() + hoc.numel() * hoc.element_size()
    saved = (wl.q, wl.k, wl.v, wl.q_c, wl.k_c, wl.v_c, wl.new_k, wl.new_v)
    wl.q, wl.k, wl.v, wl.q_c, wl.k_c, wl.v_c, wl.new_k, wl.new_v = dq
    steps = max(3, min(args.steps, 10))
    flops = 0.0
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    tot = 0.0
    for _ in range(steps):
        wl.flush()
        f3, _ = wl.c3_units()
        t0.record()
        for h, d in zip(hq, dq):
            d.copy_(h, non_blocking=True)
        wl.part_c2()
        wl.part_c3()
        ho.copy_(wl.out, non_blocking=True)
        hoc.copy_(wl.out_c, non_blocking=True)
        t1.record()
        torch.cuda.synchronize()
        tot += t0.elapsed_time(t1) / 1e3
        flops += wl.c2_flops + f3
    wl.q, wl.k, wl.v, wl.q_c, wl.k_c, wl.v_c, wl.new_k, wl.new_v = saved
    return {"value": round(flops / tot / 1e12, 4), "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps}


def cpu_sample_units():
    """A bounded sample of both parts for the fp64 oracle: a few query rows of every
    user of the jagged workload and a few candidates of every cached user."""
    import workloads as W
    c2 = W.jagged_bf16()
    rng = np.random.default_rng(5)
    rows2 = []
    for b in range(c2.B):
        s, e = int(c2.seq_offsets[b]), int(c2.seq_offsets[b + 1])
        rows2 += rng.integers(s, e, size=24).tolist()
    rows2 = np.array(sorted(rows2), dtype=np.int64)
    f2 = 0.0
    for r in rows2:
        b = int(np.searchsorted(c2.seq_offsets, r, side="right") - 1)
        f2 += (r - c2.seq_offsets[b] + 1) * c2.H * 4 * c2.d
    c3 = W.cached_cand()
    rows3 = np.array([b * 128 + j for b in range(c3.B) for j in (0, 64)], dtype=np.int64)
    L = c3.hist_lengths + c3.n_new
    f3 = sum(float(L[r // 128] + 1) * c3.H * 4 * c3.d for r in rows3)
    return c2, rows2, f2, c3, rows3, f3


def run_oracle_sample(c2, rows2, c3, rows3, threads):
    import oracle
    import workloads as W
    oracle.attn_causal(c2.q, c2.k, c2.v, c2.seq_offsets, timestamps=c2.timestamps,
                       pos_table=c2.pos_table, time_table=c2.time_table, scale=c2.scale, rows=rows2,
                       threads=threads)
    ho = W.offsets_from_lengths(c3.hist_lengths)
    no = W.offsets_from_lengths(c3.n_new)
    k = np.concatenate([np.concatenate([c3.hist_k[ho[b]:ho[b + 1]], c3.new_k[no[b]:no[b + 1]]])
                        for b in range(c3.B)])
    v = np.concatenate([np.concatenate([c3.hist_v[ho[b]:ho[b + 1]], c3.new_v[no[b]:no[b + 1]]])
                        for b in range(c3.B)])
    oracle.attn_candidates(k, v, W.offsets_from_lengths(c3.total_lengths), c3.q_cand, c3.k_cand,
                           c3.v_cand, c3.q_offsets, pos_table=c3.pos_table, scale=c3.scale,
                           rows=rows3, threads=threads)


def cpu_baseline(args):
    import oracle
    threads = oracle.default_threads()
    c2, rows2, f2, c3, rows3, f3 = cpu_sample_units()
    t0 = time.perf_counter()
    run_oracle_sample(c2, rows2, c3, rows3, threads)
    dt = time.perf_counter() - t0
    return {"value": round((f2 + f3) / dt / 1e12, 6), "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle",
            "sample": f"fp64 C oracle on {len(rows2)} query rows of jagged_bf16 (24 per user) + "
                      f"{len(rows3)} candidates of cached_cand (2 per user); {dt:.1f} s"}


def run_reference(args):
    """The oracle as the reference arm: same metric and config, bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    threads = oracle.default_threads()
    c2, rows2, f2, c3, rows3, f3 = cpu_sample_units()
    for _ in range(args.warmup):
        run_oracle_sample(c2, rows2[:8], c3, rows3[:2], threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run_oracle_sample(c2, rows2, c3, rows3, threads)
    dt = time.perf_counter() - t0
    value = (f2 + f3) * args.steps / dt / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": WORKLOAD, "global_batch": 16, "seq_len": int(c2.max_len),
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"per step: {len(rows2)} query rows of jagged_bf16 + {len(rows3)} candidates"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU baseline leg")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
