#!/usr/bin/env python
"""Benchmark of the HSTU attention hot path on B200.

One step = one pass of the hot path over one batch of synthetic input, in the
two configurations the metric is quoted on:
  A. long histories, workload ``long_history``: 32 users with Zipf(1.2)
     lengths clipped to [64, 16384] (T ~ 77k tokens), 4 heads x 128, bf16,
     16-bucket position rab, a 2M-token paged KV pool.  Per step: KV alloc +
     append of 16 new tokens per user, lookup, then causal HSTU attention of
     every user's last L_b tokens over its whole cached history, K/V read page
     by page inside the kernel ("TFLOP/s on long sequences");
  B. cached-candidate scoring, workload ``cached_cand``: 8 users with a paged
     history L ~ U[1024, 4096] (100% KV hit); per step KV alloc + append of 64
     tokens per user, lookup, then 128 candidates per user attend to the whole
     cached history plus themselves ("cached candidates/sec").
Every step appends into fresh pages (the pools are sized for all steps), so the
histories grow; FLOPs and bytes are counted from the actual lengths of every
step.  value = attention FLOPs of both parts (unmasked pairs only) / step time,
in TFLOP/s.  The 8-user jagged workload (``jagged_bf16``) is timed separately
and reported under parts.  Inputs are resident in HBM; L2 is flushed (256 MiB
write) between steps, outside the per-step CUDA events.

``--impl reference`` times the fp64 CPU oracle (the only reference this build
has) on a bounded sample of the same workloads.
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
WORKLOAD = ("long_history (B=32, L=clip(zipf(1.2),64,16384), H=4, d=128, bf16, pos16 rab, paged "
            "2M-token pool, +16 appended/user, causal over full history) + cached_cand (B=8, paged "
            "history U[1024,4096], +64 appended, 128 candidates/user)")


TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "roofline_traffic.json")
KERNEL_SOURCES = [os.path.join(ROOT, "generative_recommender_sequence_b200", "csrc", f)
                  for f in ("attn_sm100.cu", "attn.h", "sm100.cuh")]


def kernel_source_digest() -> str:
    """SHA-256 over the attention kernel's sources (what an ncu capture was taken of)."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic():
    """DRAM bytes per launch of the dominant kernel from the committed ncu record,
    or None when the record is missing or was taken on other kernel sources."""
    try:
        with open(TRAFFIC_RECORD) as f:
            rec = json.load(f)
        if rec.get("kernel_source_sha256") != kernel_source_digest():
            return None
        return int(rec["dram_bytes_per_launch"])
    except (OSError, ValueError, KeyError):
        return None


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
    from generative_recommender_sequence_b200.sharding import global_step_time
    return global_step_time(x, device="cuda") if world > 1 else x


def sum_over_ranks(x, world):
    from generative_recommender_sequence_b200.sharding import global_units
    return global_units(x, device="cuda") if world > 1 else x


def _dev(a, dt=None):
    import torch
    import workloads as W
    return (torch.as_tensor(np.ascontiguousarray(a)) if dt is None else W.to_torch(a, dt)).cuda()


class PagedPart:
    """A cached workload (long_history or cached_cand) with a KV table sized for all steps."""

    def __init__(self, case, n_steps_total, seed):
        import torch
        import generative_recommender_sequence_b200 as hstu
        import workloads as W
        self.hstu, self.case = hstu, case
        per_step_pages = int(np.max((case.n_new + 31) // 32)) + 1
        extra = case.B * n_steps_total * per_step_pages
        rng = np.random.default_rng(seed)
        order = np.concatenate([case.free_order, case.n_pages + rng.permutation(extra)]).astype(np.int32)
        self.max_cached = int(case.total_lengths.max()) + n_steps_total * int(case.n_new.max())
        self.max_ppu = (self.max_cached + 31) // 32 + 2
        self.table = hstu.KVTable(case.n_pages + extra, case.H, case.d, max_users=case.B,
                                  max_pages_per_user=self.max_ppu, free_order=order)
        self.users = _dev(case.users)
        hist_off = W.offsets_from_lengths(case.hist_lengths)
        self.table.alloc(self.users, _dev(case.hist_lengths))
        if int(case.hist_lengths.max()) > 0:
            self.table.append(self.users, _dev(case.hist_k, "bf16"), _dev(case.hist_v, "bf16"),
                              _dev(hist_off), int(case.hist_lengths.max()))
        assert self.table.status() == 0
        self.n_new = _dev(case.n_new)
        self.new_off = _dev(W.offsets_from_lengths(case.n_new))
        self.new_k, self.new_v = _dev(case.new_k, "bf16"), _dev(case.new_v, "bf16")
        if case.mode == 0:
            self.q, self.k_c, self.v_c = (_dev(x, "bf16") for x in (case.q_cand, case.k_cand, case.v_cand))
            self.n_q = case.n_cand.copy()
        else:
            self.q, self.k_c, self.v_c = _dev(case.q, "bf16"), None, None
            self.n_q = case.n_q.copy()
        self.q_off = _dev(case.q_offsets)
        self.pt = _dev(case.pos_table)
        self.out = torch.empty_like(self.q)
        self.cached_len = torch.empty(case.B, dtype=torch.int64, device="cuda")
        self.page_table = torch.empty((case.B, self.max_ppu), dtype=torch.int32, device="cuda")
        self.hist_now = case.hist_lengths.copy()
        need = self.table.workspace_size(case.B, int(case.q_offsets[-1]), int(self.n_q.max()),
                                         self.max_cached, case.mode)
        self.ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")

    def units(self):
        """(attention flops, algorithmic bytes, queries) of the next step."""
        c = self.case
        Lk = (self.hist_now + c.n_new).astype(np.float64)
        nq = self.n_q.astype(np.float64)
        if c.mode == 0:
            pairs = (nq * (Lk + 1)).sum()
        else:
            pairs = (nq * (Lk - nq) + nq * (nq + 1) / 2).sum()
        row = c.H * c.d * 2
        bytes_ = float((Lk * 2 * row).sum() + (c.n_new * 2 * row * 2).sum()
                       + nq.sum() * row * (4 if c.mode == 0 else 2))
        return float(pairs * c.H * 4 * c.d), bytes_, float(nq.sum())

    def kv_ops(self, stream=None):
        """alloc + append + lookup rows of this step's new tokens (one hstu_kv_step call)."""
        self.table.step(self.users, self.new_k, self.new_v, self.new_off, int(self.case.n_new.max()),
                        self.cached_len, self.page_table, stream=stream)

    def launch_attention(self, stream=None):
        h, c = self.hstu, self.case
        h.attn_cached_fwd(self.table, self.users, self.q, self.q_off, int(self.n_q.max()), self.max_cached,
                          c.mode, k_cand=self.k_c, v_cand=self.v_c, pos_table=self.pt, scale=c.scale,
                          out=self.out, workspace=self.ws, stream=stream)

    def advance(self):
        """Host-side record of the cached lengths after one more step."""
        self.hist_now = self.hist_now + self.case.n_new

    def attention(self, stream=None):
        self.launch_attention(stream)
        self.advance()


class JaggedPart:
    def __init__(self):
        import torch
        import generative_recommender_sequence_b200 as hstu
        import workloads as W
        self.hstu = hstu
        c = W.jagged_bf16()
        self.c = c
        self.q, self.k, self.v = (_dev(x, "bf16") for x in (c.q, c.k, c.v))
        self.off = _dev(c.seq_offsets)
        self.pt, self.tt, self.ts = _dev(c.pos_table), _dev(c.time_table), _dev(c.timestamps)
        self.out = torch.empty_like(self.q)
        self.flops = c.flops()

    def run(self):
        c = self.c
        self.hstu.attn_fwd(self.q, self.k, self.v, self.off, c.max_len, pos_table=self.pt,
                           time_table=self.tt, timestamps=self.ts, scale=c.scale, out=self.out)


class CachedServingPart:
    """KV-cached multi-layer serving vs the same stack without the cache (the
    pages' benchmark, on synthetic inputs): 8 users with histories U[1024, 8192]
    cached per layer, each request adding 64 new tokens and scoring 128
    candidates; hidden 512, 4 heads of 128, bf16.  The uncached path runs the
    block over each user's whole sequence [history; new; candidates].  Both are
    replayed from CUDA graphs; the prefill of the caches is not timed."""

    def __init__(self, n_layers, n_runs, seed=2024):
        import torch
        import generative_recommender_sequence_b200 as hstu
        import workloads as W
        rng = np.random.default_rng(seed)
        self.hstu, self.n_layers = hstu, n_layers
        B, n_new, n_cand, dm = 8, 64, 128, 512
        hist = rng.integers(1024, 8193, B).astype(np.int64)
        bf = lambda a: W.to_torch(W._as_storage(np.asarray(a, np.float32), "bf16"), "bf16").cuda()
        off = lambda n: torch.as_tensor(np.concatenate([[0], np.cumsum(n)]).astype(np.int64)).cuda()
        x_hist = bf(rng.standard_normal((int(hist.sum()), dm)))
        x_new = bf(rng.standard_normal((B * n_new, dm)))
        x_cand = bf(rng.standard_normal((B * n_cand, dm)))
        self.w1 = [bf(rng.normal(0, 0.02, (dm, 2048))) for _ in range(n_layers)]
        self.w2 = [bf(rng.normal(0, 0.02, (512, dm))) for _ in range(n_layers)]
        self.pt = torch.as_tensor(rng.normal(0, 0.1, 16).astype(np.float32)).cuda()
        full_len = hist + n_new + n_cand
        self.scale = 1.0 / int(full_len.max())
        grow = n_new * (n_runs + 4)
        self.max_cached = int(hist.max()) + grow
        mpp = (self.max_cached + 31) // 32 + 2
        n_pages = int(np.sum((hist + grow + 31) // 32)) + 8
        self.tables = [hstu.KVTable(n_pages, 4, 128, max_users=B, max_pages_per_user=mpp)
                       for _ in range(n_layers)]
        self.users = torch.arange(B, dtype=torch.int64, device="cuda")
        hstu.block_cached_step(self.tables, self.users, x_hist, off(hist), int(hist.max()), None, 0,
                               int(hist.max()), self.w1, self.w2, pos_table=self.pt, scale=self.scale)
        self.new_off, self.cand_off = off(np.full(B, n_new)), off(np.full(B, n_cand))
        self.n_new, self.n_cand, self.T_new = n_new, n_cand, B * n_new
        self.x0 = torch.cat([x_new, x_cand])
        self.x = self.x0.clone()
        self.ws = torch.empty(hstu.block_cached_workspace_size(self.tables, B, B * n_new, B * n_cand,
                                                                n_cand, self.max_cached),
                              dtype=torch.uint8, device="cuda")
        # uncached: every user's whole sequence, candidates last
        xh = x_hist.split(hist.tolist())
        xn, xc = x_new.split(n_new), x_cand.split(n_cand)
        self.full0 = torch.cat([torch.cat([xh[b], xn[b], xc[b]]) for b in range(B)])
        self.full = self.full0.clone()
        self.full_off, self.full_max = off(full_len), int(full_len.max())
        self.ws_full = torch.empty(hstu.block_workspace_size(int(full_len.sum()), dm, 4, 128),
                                   dtype=torch.uint8, device="cuda")
        torch.cuda.synchronize()

    def cached(self):
        self.hstu.block_cached_step(self.tables, self.users, self.x, self.new_off, self.n_new,
                                    self.cand_off, self.n_cand, self.max_cached, self.w1, self.w2,
                                    pos_table=self.pt, scale=self.scale, T_new=self.T_new,
                                    workspace=self.ws)

    def uncached(self):
        self.hstu.block_fwd(self.full, self.full_off, self.full_max, self.w1, self.w2,
                            pos_table=self.pt, scale=self.scale, workspace=self.ws_full)

    def measure(self, runs):
        import torch
        self.cached()
        self.uncached()
        torch.cuda.synchronize()
        g_c, g_u = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_c):
            self.cached()
        with torch.cuda.graph(g_u):
            self.uncached()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        res = {}
        for name, g, x, x0 in (("cached", g_c, self.x, self.x0), ("uncached", g_u, self.full, self.full0)):
            tot = 0.0
            for _ in range(runs):
                x.copy_(x0)
                e0.record(); g.replay(); e1.record()
                torch.cuda.synchronize()
                tot += e0.elapsed_time(e1)
            res[name + "_ms"] = round(tot / runs, 4)
        for t in self.tables:
            if t.status():
                raise RuntimeError("KV table error in the cached serving measurement")
        res["speedup"] = round(res["uncached_ms"] / res["cached_ms"], 2)
        return res


class BeamDecodePart:
    """Beam-search decode attention (the pages' Semantic ID workload shape, on
    synthetic inputs): 8 requests with 5000-token contexts in the paged table,
    256 beams each, 3 decode steps; 4 heads of 128, bf16.  Per step: latency,
    FLOP rate, and the bytes that must move (context K/V once, the beams' Q, K,
    V and output) as a fraction of HBM bandwidth."""

    def __init__(self, seed=77, B=8, L=5000, W=256, steps=3):
        import torch
        import generative_recommender_sequence_b200 as hstu
        import workloads as W_
        rng = np.random.default_rng(seed)
        self.hstu, self.B, self.L, self.W, self.steps = hstu, B, L, W, steps
        H, D = 4, 128
        bf = lambda shape: W_.to_torch(W_._as_storage(rng.standard_normal(shape).astype(np.float32),
                                                      "bf16"), "bf16").cuda()
        n_pages = B * ((L + 31) // 32) + 4
        self.table = hstu.KVTable(n_pages, H, D, max_users=B, max_pages_per_user=(L + 31) // 32 + 2)
        self.users = torch.arange(B, dtype=torch.int64, device="cuda")
        lens = torch.full((B,), L, dtype=torch.int64, device="cuda")
        self.table.alloc(self.users, lens)
        off = torch.arange(0, B * L + 1, L, dtype=torch.int64, device="cuda")
        self.table.append(self.users, bf((B * L, H, D)), bf((B * L, H, D)), off, L)
        T = B * W
        self.q = bf((T, H, D))
        self.bk, self.bv = bf((steps, T, H, D)), bf((steps, T, H, D))
        par = np.zeros((steps, T), np.int32)
        for t in range(1, steps):
            par[t] = np.concatenate([rng.integers(0, W, size=W) for _ in range(B)])
        self.parent = torch.as_tensor(par).cuda()
        self.bo = torch.arange(0, T + 1, W, dtype=torch.int64, device="cuda")
        self.pt = torch.as_tensor(rng.normal(0, 0.1, 16).astype(np.float32)).cuda()
        self.out = torch.empty_like(self.q)
        self.ws = torch.empty(max(1 << 20, hstu.load().hstu_attn_beam_decode_workspace_size(
            self.table.handle, B, T, W, L, steps - 1)), dtype=torch.uint8, device="cuda")
        torch.cuda.synchronize()

    def run(self, s):
        self.hstu.attn_beam_decode(self.table, self.users, self.q, self.bo, self.W, self.L, s,
                                   self.bk[:s + 1], self.bv[:s + 1], self.parent[:s + 1] if s else None,
                                   pos_table=self.pt, scale=1.0 / (self.L + self.steps), out=self.out,
                                   workspace=self.ws)

    def measure(self, flush_buf, hbm_peak, tf_peak, reps=5):
        import torch
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        res = {}
        T, F = self.B * self.W, 4 * 128
        for s in range(self.steps):
            self.run(s)
            tot = 0.0
            for _ in range(reps):
                flush_buf.fill_(1)
                e0.record(); self.run(s); e1.record()
                torch.cuda.synchronize()
                tot += e0.elapsed_time(e1) / 1e3
            t = tot / reps
            flops = float(T) * (self.L + s + 1) * F * 4
            bytes_ = float(self.B) * self.L * F * 2 * 2 + T * F * 2 * (3 + 2 * s + 1)
            res[f"step_{s}"] = {"us": round(t * 1e6, 2), "tflops": round(flops / t / 1e12, 2),
                                "frac_of_bf16_peak": round(flops / t / 1e12 / tf_peak, 4),
                                "gbs": round(bytes_ / t / 1e9, 1),
                                "frac_of_hbm": round(bytes_ / t / 1e9 / hbm_peak, 4)}
        if self.table.status() or self.hstu.last_device_error():
            raise RuntimeError("device error in the beam decode measurement")
        return res


def run_gpu(args):
    import torch
    import workloads as W
    rank, world, local = dist_setup(args.gpus)
    hbm_peak, tf_peak, tf_sus, peak_src = load_peaks()
    n_total = args.warmup + args.steps + 12
    # weak scaling: every rank owns one per-GPU batch of distinct users (its own
    # seeds; rank 0 draws the reference workloads), no data-path collective
    A = PagedPart(W.long_history(seed=1005 + 7919 * rank), n_total, seed=55 + rank)
    Bp = PagedPart(W.cached_cand(seed=1003 + 7919 * rank), n_total, seed=77 + rank)
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        flush_buf.fill_(1)
        A.kv_ops(); A.attention(); Bp.kv_ops(); Bp.attention()
    torch.cuda.synchronize()
    if A.table.status() or Bp.table.status() or A.hstu.last_device_error():
        raise RuntimeError("device error during warm-up")

    # The step's launches as CUDA graphs (capture does not execute them): the KV
    # ops read and advance the table state on the device, so every replay
    # appends into fresh slots exactly like a direct call.
    g_akv, g_aat, g_b = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_akv):
        A.kv_ops()
    with torch.cuda.graph(g_aat):
        A.launch_attention()
    with torch.cuda.graph(g_b):
        Bp.kv_ops()
        Bp.launch_attention()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    fa = fb = bb = qb = 0.0
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    if rank == 0:
        sampler.start()
        time.sleep(0.25)
    wall0 = time.perf_counter()
    for i in range(args.steps):
        flush_buf.fill_(1)
        f_a, _, _ = A.units()
        f_b, b_b, q_b = Bp.units()
        ev[i][0].record()
        g_akv.replay()
        ev[i][1].record()
        g_aat.replay()
        ev[i][2].record()
        g_b.replay()
        ev[i][3].record()
        A.advance()
        Bp.advance()
        fa += f_a; fb += f_b; bb += b_b; qb += q_b
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - wall0
    clocks = sampler.stop() if rank == 0 else None
    t_akv = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3
    t_aat = sum(e[1].elapsed_time(e[2]) for e in ev) / 1e3
    t_b = sum(e[2].elapsed_time(e[3]) for e in ev) / 1e3
    t_step = t_akv + t_aat + t_b
    if A.table.status() or Bp.table.status() or A.hstu.last_device_error():
        raise RuntimeError("device error during the timed steps")
    t_max = max_over_ranks(t_step, world)
    value = sum_over_ranks(fa + fb, world) / t_max / 1e12
    a_tflops = fa / (t_akv + t_aat) / 1e12
    a_attn_tflops = fa / t_aat / 1e12
    cand_per_s = qb / t_b
    b_gbs = bb / t_b / 1e9

    # the jagged workload, reported beside the step (not part of value)
    J = JaggedPart()
    for _ in range(3):
        J.run()
    jt = 0.0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(max(3, args.steps // 2)):
        flush_buf.fill_(1)
        e0.record(); J.run(); e1.record()
        torch.cuda.synchronize()
        jt += e0.elapsed_time(e1) / 1e3
    jsteps = max(3, args.steps // 2)

    # KV-cached multi-layer serving vs the uncached stack, reported beside the step
    serving = {}
    if not args.no_serving:
        for n_layers in (3, 8):
            part = CachedServingPart(n_layers, n_runs=5)
            serving[f"layers_{n_layers}"] = part.measure(runs=5)
            del part

    beam = {} if args.no_serving else BeamDecodePart().measure(flush_buf, hbm_peak, tf_peak)

    # the cached-candidate step at larger batches (same per-user shapes): how far
    # the fixed per-step latencies are amortised once a step moves more bytes
    # (single-GPU runs only: the 128-user case draws ~1.3 GB of host inputs)
    by_batch = {}
    if not args.no_serving and world == 1:
        for nb in (32, 128):
            part = PagedPart(W.cached_cand(B=nb, seed=2003 + 7919 * rank), 12, seed=91 + rank)
            for _ in range(3):
                part.kv_ops(); part.attention()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                part.kv_ops()
                part.launch_attention()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            tot = byt = nq = 0.0
            for _ in range(5):
                flush_buf.fill_(1)
                _, b_, q_ = part.units()
                e0.record(); g.replay(); e1.record()
                torch.cuda.synchronize()
                tot += e0.elapsed_time(e1) / 1e3
                byt += b_
                nq += q_
                part.advance()
            if part.table.status():
                raise RuntimeError("KV table error in the batch-scaling measurement")
            by_batch[f"B_{nb}"] = {"ms": round(tot / 5 * 1e3, 4),
                                   "candidates_per_s": round(nq / tot, 1),
                                   "hbm_gbs": round(byt / tot / 1e9, 1),
                                   "frac_of_hbm": round(byt / tot / 1e9 / hbm_peak, 4)}
            del g, part

    # every rank runs the end-to-end steps: whole-job units over the slowest rank
    e2e_local = run_e2e(A, Bp, flush_buf, args)
    e2e_t = max_over_ranks(e2e_local.pop("seconds"), world)
    e2e_units = sum_over_ranks(e2e_local.pop("flops"), world)
    e2e_h2d = sum_over_ranks(float(e2e_local["h2d_bytes_per_step"]), world)
    e2e_d2h = sum_over_ranks(float(e2e_local["d2h_bytes_per_step"]), world)
    e2e = {"value": round(e2e_units / e2e_t / 1e12, 4), "unit": "TFLOP/s",
           "h2d_bytes_per_step": int(e2e_h2d), "d2h_bytes_per_step": int(e2e_d2h),
           "steps": e2e_local["steps"]}
    cpu = cpu_baseline(args) if (rank == 0 and world == 1 and not args.no_cpu) else None
    if rank == 0:
        c5 = A.case
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_step / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; shapes of the pages' benchmark, KuaiRand-1K not available)",
            "config": {"workload": WORKLOAD, "global_batch": (c5.B + Bp.case.B) * world,
                       "seq_len": int(c5.total_lengths.max()),
                       "parallelism": f"dp{world} (users sharded, no collective on the data path)",
                       "l2": "flushed between steps (256 MiB write, outside the step events)",
                       "timing": "CUDA-graph replay of each part, CUDA events between replays"},
            "parts": {
                "long_history": {"ms": round((t_akv + t_aat) / args.steps * 1e3, 4),
                                 "kv_ops_ms": round(t_akv / args.steps * 1e3, 4),
                                 "attention_ms": round(t_aat / args.steps * 1e3, 4),
                                 "tflops": round(a_tflops, 2), "attention_tflops": round(a_attn_tflops, 2),
                                 "frac_of_bf16_peak": round(a_attn_tflops / tf_peak, 4)},
                "cached_candidates": {"ms": round(t_b / args.steps * 1e3, 4),
                                      "candidates_per_s": round(cand_per_s, 1),
                                      "hbm_gbs": round(b_gbs, 1), "frac_of_hbm": round(b_gbs / hbm_peak, 4)},
                "cached_candidates_by_batch": by_batch,
                "cached_serving": serving,
                "beam_decode": beam,
                "jagged_bf16": {"ms": round(jt / jsteps * 1e3, 4),
                                "tflops": round(J.flops * jsteps / jt / 1e12, 2),
                                "frac_of_bf16_peak": round(J.flops * jsteps / jt / 1e12 / tf_peak, 4)},
            },
            "cached_candidates_per_s": round(cand_per_s * world, 1),
            "roofline": {"bound": "tensor", "kernel": "hstu_attn_sm100_kernel<paged, causal> (long_history)",
                         "achieved": round(a_attn_tflops, 2), "peak": tf_peak, "unit": "TFLOP/s",
                         "frac": round(a_attn_tflops / tf_peak, 4), "traffic": recorded_traffic(),
                         "peak_source": f"{peak_src} bf16 dense (burst)"},
            "gpu_launches": args.steps * 9,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "wall_s": round(wall, 3),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(A, Bp, flush_buf, args):
    """Same metric through the public API with host (pinned) inputs: H2D of each
    step's inputs and D2H of its outputs are inside the timed region.  Returns
    this rank's device seconds, FLOPs and bytes per step (the caller reduces
    them over ranks)."""
    import torch
    parts = [(A, ["q", "new_k", "new_v"]), (Bp, ["q", "k_c", "v_c", "new_k", "new_v"])]
    host, saved = [], []
    for part, names in parts:
        for n in names:
            t = getattr(part, n)
            host.append((part, n, t.cpu().pin_memory(), torch.empty_like(t)))
            saved.append((part, n, t))
    outs = [(A.out, torch.empty_like(A.out, device="cpu").pin_memory()),
            (Bp.out, torch.empty_like(Bp.out, device="cpu").pin_memory())]
    h2d = sum(h.numel() * h.element_size() for _, _, h, _ in host)
    d2h = sum(h.numel() * h.element_size() for _, h in outs)
    for part, n, _, d in host:
        setattr(part, n, d)
    steps = max(3, min(args.steps, 5))
    flops, tot = 0.0, 0.0
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(steps):
        flush_buf.fill_(1)
        fa, _, _ = A.units()
        fb, _, _ = Bp.units()
        t0.record()
        for _, _, h, d in host:
            d.copy_(h, non_blocking=True)
        A.kv_ops(); A.attention(); Bp.kv_ops(); Bp.attention()
        for dsrc, h in outs:
            h.copy_(dsrc, non_blocking=True)
        t1.record()
        torch.cuda.synchronize()
        tot += t0.elapsed_time(t1) / 1e3
        flops += fa + fb
    for part, n, t in saved:
        setattr(part, n, t)
    return {"seconds": tot, "flops": flops, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps}


def cpu_sample_units(rows_per_user=6, cands_per_user=2):
    """A bounded sample of both parts for the fp64 oracle: a few query rows of every
    long-history user (spread over its positions) and a few candidates per cached user."""
    import workloads as W
    c5 = W.long_history()
    rng = np.random.default_rng(5)
    qo = c5.q_offsets
    rows5 = []
    for b in range(c5.B):
        s0, e0 = int(qo[b]), int(qo[b + 1])
        rows5 += sorted(set(rng.integers(s0, e0, size=min(rows_per_user, e0 - s0)).tolist()))
    rows5 = np.array(rows5, dtype=np.int64)
    f5 = 0.0
    for r in rows5:
        b = int(np.searchsorted(qo, r, side="right") - 1)
        f5 += (r - qo[b] + 1) * c5.H * 4 * c5.d  # n_q == cached length: position r - qo[b]
    c3 = W.cached_cand()
    rows3 = np.array([b * 128 + j for b in range(c3.B) for j in range(0, 128, 128 // cands_per_user)],
                     dtype=np.int64)
    L = c3.hist_lengths + c3.n_new
    f3 = sum(float(L[r // 128] + 1) * c3.H * 4 * c3.d for r in rows3)
    return c5, rows5, f5, c3, rows3, f3


def _joined_kv(c):
    import workloads as W
    ho, no = W.offsets_from_lengths(c.hist_lengths), W.offsets_from_lengths(c.n_new)
    k = np.concatenate([np.concatenate([c.hist_k[ho[b]:ho[b + 1]], c.new_k[no[b]:no[b + 1]]]) for b in range(c.B)])
    v = np.concatenate([np.concatenate([c.hist_v[ho[b]:ho[b + 1]], c.new_v[no[b]:no[b + 1]]]) for b in range(c.B)])
    return k, v, W.offsets_from_lengths(c.total_lengths)


def run_oracle_sample(c5, rows5, c3, rows3, threads, kv5=None, kv3=None):
    import oracle
    k5, v5, o5 = kv5 if kv5 is not None else _joined_kv(c5)
    oracle.attn_causal(c5.q, k5, v5, o5, q_offsets=c5.q_offsets, pos_table=c5.pos_table,
                       scale=c5.scale, rows=rows5, threads=threads)
    k3, v3, o3 = kv3 if kv3 is not None else _joined_kv(c3)
    oracle.attn_candidates(k3, v3, o3, c3.q_cand, c3.k_cand, c3.v_cand, c3.q_offsets,
                           pos_table=c3.pos_table, scale=c3.scale, rows=rows3, threads=threads)


def cpu_baseline(args):
    import oracle
    threads = oracle.default_threads()
    # about 10-15 s of fp64 work on a 16-core host
    c5, rows5, f5, c3, rows3, f3 = cpu_sample_units(rows_per_user=2500, cands_per_user=32)
    kv5, kv3 = _joined_kv(c5), _joined_kv(c3)
    t0 = time.perf_counter()
    run_oracle_sample(c5, rows5, c3, rows3, threads, kv5, kv3)
    dt = time.perf_counter() - t0
    return {"value": round((f5 + f3) / dt / 1e12, 6), "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle",
            "sample": f"fp64 C oracle on {len(rows5)} query rows of long_history (up to 2500 per user) + "
                      f"{len(rows3)} candidates of cached_cand (32 per user); {dt:.1f} s"}


def run_reference(args):
    """The oracle as the reference arm: same metric and config, bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    threads = oracle.default_threads()
    c5, rows5, f5, c3, rows3, f3 = cpu_sample_units()
    kv5, kv3 = _joined_kv(c5), _joined_kv(c3)
    for _ in range(args.warmup):
        run_oracle_sample(c5, rows5[:4], c3, rows3[:1], threads, kv5, kv3)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run_oracle_sample(c5, rows5, c3, rows3, threads, kv5, kv3)
    dt = time.perf_counter() - t0
    value = (f5 + f3) * args.steps / dt / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": WORKLOAD, "global_batch": 40, "seq_len": int(c5.total_lengths.max()),
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"per step: {len(rows5)} query rows of long_history + {len(rows3)} candidates"},
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
    ap.add_argument("--no-serving", action="store_true",
                    help="skip the cached vs uncached multi-layer serving report")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
