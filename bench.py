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
Before every step (outside the timed region) both tables are put back to the
state after their prefill: the users are released and their histories
allocated and appended again, so every timed step sees exactly the workloads'
cached lengths (history + this step's append).  value = attention FLOPs of both
parts (unmasked pairs only) / step time, in TFLOP/s.  The 8-user jagged workload
(``jagged_bf16``), the 8-layer block stack (``block_stack``) and the KV append
path are timed separately and reported under parts.  Inputs are resident in
HBM; L2 is flushed (256 MiB write) between steps, outside the per-step CUDA
events.

``--gpus N`` without an outer launcher re-executes this script under
torch.distributed.run with N local ranks (one process per GPU); under a
launcher, WORLD_SIZE must equal N.

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


def launcher_command(n_gpus, argv, port=None):
    """The torch.distributed.run command that starts one rank per GPU of this node."""
    port = port if port is not None else 29500 + (os.getpid() % 2000)
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n_gpus}", "--master-addr", "127.0.0.1",
            "--master-port", str(port), os.path.abspath(__file__), *argv]


def check_world(n_gpus, env):
    """Rank layout from the launcher's environment; refuses a --gpus / WORLD_SIZE mismatch."""
    world = int(env.get("WORLD_SIZE", "1"))
    if "WORLD_SIZE" in env and world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but the launcher started WORLD_SIZE={world} ranks")
    return int(env.get("RANK", "0")), world, int(env.get("LOCAL_RANK", "0"))


def dist_setup(n_gpus):
    import torch
    rank, world, local = check_world(n_gpus, os.environ)
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
    """A cached workload (long_history or cached_cand) in its own KV table.

    reset() puts the table back to the state after the prefill (release every
    user, then allocate and append the history again), so each step appends
    the workload's new tokens onto exactly the workload's history."""

    def __init__(self, case, seed):
        import torch
        import generative_recommender_sequence_b200 as hstu
        import workloads as W
        self.hstu, self.case = hstu, case
        # room for the history + one step's append, plus a spare page per user
        n_pages = max(case.n_pages, int(np.sum((case.total_lengths + 31) // 32)) + case.B)
        rng = np.random.default_rng(seed)
        order = rng.permutation(n_pages).astype(np.int32)
        self.max_cached = int(case.total_lengths.max())
        self.max_ppu = (self.max_cached + 31) // 32 + 2
        self.table = hstu.KVTable(n_pages, case.H, case.d, max_users=case.B,
                                  max_pages_per_user=self.max_ppu, free_order=order)
        self.users = _dev(case.users)
        self.hist_len = _dev(case.hist_lengths)
        self.hist_off = _dev(W.offsets_from_lengths(case.hist_lengths))
        self.hist_k, self.hist_v = _dev(case.hist_k, "bf16"), _dev(case.hist_v, "bf16")
        self.reset()
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
        need = self.table.workspace_size(case.B, int(case.q_offsets[-1]), int(self.n_q.max()),
                                         self.max_cached, case.mode)
        self.ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")

    def reset(self, stream=None):
        """Back to the prefilled state: release every user, re-append its history."""
        c = self.case
        self.table.release(self.users, stream=stream)
        self.table.alloc(self.users, self.hist_len, stream=stream)
        if int(c.hist_lengths.max()) > 0:
            self.table.append(self.users, self.hist_k, self.hist_v, self.hist_off,
                              int(c.hist_lengths.max()), stream=stream)

    def units(self):
        """(attention flops, algorithmic bytes, queries) of one step."""
        c = self.case
        Lk = (c.hist_lengths + c.n_new).astype(np.float64)
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

    def attention(self, stream=None):
        self.launch_attention(stream)


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


class BlockStackPart:
    """The 8-layer HSTU block stack of workload ``block_stack`` (B=8, L~U[512,4096],
    d_model 512, 4 heads x 128, bf16, position + time rab): one hstu_block_fwd
    call over all layers, replayed from a CUDA graph after an L2 flush.  The
    attention alone (the same lengths and rab on contiguous Q/K/V) and one layer
    are timed too, so GEMMs + LayerNorm gate = layer - attention."""

    def __init__(self):
        import torch
        import generative_recommender_sequence_b200 as hstu
        import workloads as W
        self.hstu = hstu
        c = W.block_stack()
        self.c = c
        self.x0 = _dev(c.x0, "bf16")
        self.x = self.x0.clone()
        self.off = _dev(c.seq_offsets)
        self.w1 = [_dev(c.w_uvqk[l], "bf16") for l in range(c.n_layers)]
        self.w2 = [_dev(c.w_o[l], "bf16") for l in range(c.n_layers)]
        self.pt, self.tt, self.ts = _dev(c.pos_table), _dev(c.time_table), _dev(c.timestamps)
        self.ws = torch.empty(hstu.block_workspace_size(c.T, c.d_model, c.H, c.dh),
                              dtype=torch.uint8, device="cuda")
        rng = np.random.default_rng(4)
        qkv = lambda: _dev(W._as_storage(rng.standard_normal((c.T, c.H, c.dh), dtype=np.float32),
                                         "bf16"), "bf16")
        self.q, self.k, self.v = qkv(), qkv(), qkv()
        self.a_out = torch.empty_like(self.q)

    def stack(self, n_layers):
        self.hstu.block_fwd(self.x, self.off, int(self.c.lengths.max()), self.w1[:n_layers],
                            self.w2[:n_layers], pos_table=self.pt, time_table=self.tt,
                            timestamps=self.ts, scale=self.c.scale, workspace=self.ws)

    def attention(self):
        self.hstu.attn_fwd(self.q, self.k, self.v, self.off, int(self.c.lengths.max()),
                           pos_table=self.pt, time_table=self.tt, timestamps=self.ts,
                           scale=self.c.scale, out=self.a_out)

    def measure(self, flush_buf, tf_peak, reps=5):
        import torch
        c = self.c
        res = {}
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        T = float(c.T)
        gemm = 2 * T * c.d_model * (4 * c.H * c.dh) + 2 * T * (c.H * c.dh) * c.d_model
        L = c.lengths.astype(np.float64)
        attn = float((L * (L + 1) / 2).sum() * c.H * 4 * c.dh)
        for name, fn, flops in (("stack", lambda: self.stack(c.n_layers), c.flops()),
                                ("one_layer", lambda: self.stack(1), gemm + attn),
                                ("attention", self.attention, attn)):
            fn()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            tot = 0.0
            for _ in range(reps):
                self.x.copy_(self.x0)
                flush_buf.fill_(1)
                e0.record(); g.replay(); e1.record()
                torch.cuda.synchronize()
                tot += e0.elapsed_time(e1) / 1e3
            t = tot / reps
            res[name + "_ms"] = round(t * 1e3, 4)
            res[name + "_tflops"] = round(flops / t / 1e12, 2)
            del g
        res["gemm_ln_per_layer_ms"] = round(res["one_layer_ms"] - res["attention_ms"], 4)
        res["frac_of_bf16_peak"] = round(res["stack_tflops"] / tf_peak, 4)
        res["tokens"] = int(c.T)
        if self.hstu.last_device_error():
            raise RuntimeError("device error in the block stack measurement")
        return res


def kv_append_measure(A, Bp, flush_buf, hbm_peak, reps=5):
    """The KV append path: (1) the serving steps' hstu_kv_step (alloc + append +
    lookup rows: 8 users x 64 tokens, 32 users x 16 tokens), (2) a bulk append
    of every long-history user's whole history into fresh pages (prefill /
    onboarding).  Algorithmic bytes: each appended token's K and V read once
    and written once (2 x H x d x 2 bytes each way)."""
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    res = {}
    for name, part in (("step_cached_cand", Bp), ("step_long_history", A)):
        c = part.case
        tok = float(c.n_new.sum())
        byt = tok * c.H * c.d * 2 * 2 * 2
        tot = 0.0
        for _ in range(reps):
            part.reset()
            flush_buf.fill_(1)
            e0.record(); part.kv_ops(); e1.record()
            torch.cuda.synchronize()
            tot += e0.elapsed_time(e1) / 1e3
        t = tot / reps
        res[name] = {"tokens": int(tok), "us": round(t * 1e6, 2), "gbs": round(byt / t / 1e9, 1),
                     "frac_of_hbm": round(byt / t / 1e9 / hbm_peak, 4)}
    c = A.case
    tok = float(c.hist_lengths.sum())
    byt = tok * c.H * c.d * 2 * 2 * 2
    tot = 0.0
    for _ in range(reps):
        A.table.release(A.users)
        A.table.alloc(A.users, A.hist_len)
        flush_buf.fill_(1)
        e0.record()
        A.table.append(A.users, A.hist_k, A.hist_v, A.hist_off, int(c.hist_lengths.max()))
        e1.record()
        torch.cuda.synchronize()
        tot += e0.elapsed_time(e1) / 1e3
    t = tot / reps
    res["bulk_append_long_history"] = {"tokens": int(tok), "us": round(t * 1e6, 2),
                                       "gbs": round(byt / t / 1e9, 1),
                                       "frac_of_hbm": round(byt / t / 1e9 / hbm_peak, 4)}
    A.reset()
    torch.cuda.synchronize()
    if A.table.status() or Bp.table.status():
        raise RuntimeError("KV table error in the append measurement")
    return res


def rank_seeds(rank):
    """Weak scaling: every rank owns one per-GPU batch of distinct users, drawn
    from its own seeds (rank 0 draws the reference workloads)."""
    return {"long_history": 1005 + 7919 * rank, "cached_cand": 1003 + 7919 * rank,
            "pool_long": 55 + rank, "pool_cand": 77 + rank}


def run_gpu(args):
    import torch
    import workloads as W
    rank, world, local = dist_setup(args.gpus)
    hbm_peak, tf_peak, tf_sus, peak_src = load_peaks()
    seeds = rank_seeds(rank)
    A = PagedPart(W.long_history(seed=seeds["long_history"]), seed=seeds["pool_long"])
    Bp = PagedPart(W.cached_cand(seed=seeds["cached_cand"]), seed=seeds["pool_cand"])
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        A.reset(); Bp.reset()
        flush_buf.fill_(1)
        A.kv_ops(); A.attention(); Bp.kv_ops(); Bp.attention()
    torch.cuda.synchronize()
    if A.table.status() or Bp.table.status() or A.hstu.last_device_error():
        raise RuntimeError("device error during warm-up")

    # The step's launches as CUDA graphs (capture does not execute them): the KV
    # step reads the table state on the device, so every replay after a reset
    # appends onto exactly the prefilled history.
    g_akv, g_aat, g_b = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_akv):
        A.kv_ops()
    with torch.cuda.graph(g_aat):
        A.launch_attention()
    with torch.cuda.graph(g_b):
        Bp.kv_ops()
        Bp.launch_attention()
    torch.cuda.synchronize()
    # kernels of this library per step: long history KV step + attention; cached
    # candidates KV step + attention + split reduce (when its keys are split)
    # (a split leaves partial sums in the workspace, so a non-zero workspace
    # size means the reduce kernel runs)
    split = lambda P: P.table.workspace_size(P.case.B, int(P.case.q_offsets[-1]), int(P.n_q.max()),
                                             P.max_cached, P.case.mode) > 0
    launches_per_step = 2 + int(split(A)) + 2 + int(split(Bp))

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    fa, _, _ = A.units()
    fb, bb, qb = Bp.units()
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    if rank == 0:
        sampler.start()
        time.sleep(0.25)
    wall0 = time.perf_counter()
    for i in range(args.steps):
        A.reset(); Bp.reset()
        flush_buf.fill_(1)
        ev[i][0].record()
        g_akv.replay()
        ev[i][1].record()
        g_aat.replay()
        ev[i][2].record()
        g_b.replay()
        ev[i][3].record()
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
    value = sum_over_ranks((fa + fb) * args.steps, world) / t_max / 1e12
    a_tflops = fa * args.steps / (t_akv + t_aat) / 1e12
    a_attn_tflops = fa * args.steps / t_aat / 1e12
    cand_per_s = qb * args.steps / t_b
    b_gbs = bb * args.steps / t_b / 1e9

    # the candidate kernels alone (attention + split reduce, no KV step): the
    # bytes they must move are the cached K/V (history + append) and the
    # candidates' Q, K, V in and O out
    g_bat = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_bat):
        Bp.launch_attention()
    t_bat = 0.0
    nb_at = max(5, args.steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c3 = Bp.case
    Lk3 = (c3.hist_lengths + c3.n_new).astype(np.float64)
    row3 = c3.H * c3.d * 2
    b_at = float((Lk3 * 2 * row3).sum() + c3.n_cand.sum() * row3 * 4)
    for _ in range(nb_at):
        flush_buf.fill_(1)
        e0.record(); g_bat.replay(); e1.record()
        torch.cuda.synchronize()
        t_bat += e0.elapsed_time(e1) / 1e3
    t_bat /= nb_at
    del g_bat

    # the jagged workload, reported beside the step (not part of value)
    J = JaggedPart()
    for _ in range(3):
        J.run()
    jt = 0.0
    jsteps = max(3, args.steps // 2)
    for _ in range(jsteps):
        flush_buf.fill_(1)
        e0.record(); J.run(); e1.record()
        torch.cuda.synchronize()
        jt += e0.elapsed_time(e1) / 1e3

    block = {} if args.no_serving else BlockStackPart().measure(flush_buf, tf_peak)
    kv_append = kv_append_measure(A, Bp, flush_buf, hbm_peak)

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
            part = PagedPart(W.cached_cand(B=nb, seed=2003 + 7919 * rank), seed=91 + rank)
            for _ in range(3):
                part.reset(); part.kv_ops(); part.attention()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                part.kv_ops()
                part.launch_attention()
            tot = 0.0
            _, b_, q_ = part.units()
            for _ in range(5):
                part.reset()
                flush_buf.fill_(1)
                e0.record(); g.replay(); e1.record()
                torch.cuda.synchronize()
                tot += e0.elapsed_time(e1) / 1e3
            if part.table.status():
                raise RuntimeError("KV table error in the batch-scaling measurement")
            by_batch[f"B_{nb}"] = {"ms": round(tot / 5 * 1e3, 4),
                                   "candidates_per_s": round(q_ * 5 / tot, 1),
                                   "hbm_gbs": round(b_ * 5 / tot / 1e9, 1),
                                   "frac_of_hbm": round(b_ * 5 / tot / 1e9 / hbm_peak, 4)}
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
                       "timing": "tables reset to the prefilled state before every step (outside "
                                 "the events); CUDA-graph replay of each part, CUDA events between replays"},
            "parts": {
                "long_history": {"ms": round((t_akv + t_aat) / args.steps * 1e3, 4),
                                 "kv_ops_ms": round(t_akv / args.steps * 1e3, 4),
                                 "attention_ms": round(t_aat / args.steps * 1e3, 4),
                                 "tflops": round(a_tflops, 2), "attention_tflops": round(a_attn_tflops, 2),
                                 "frac_of_bf16_peak": round(a_attn_tflops / tf_peak, 4)},
                "cached_candidates": {"ms": round(t_b / args.steps * 1e3, 4),
                                      "candidates_per_s": round(cand_per_s, 1),
                                      "hbm_gbs": round(b_gbs, 1), "frac_of_hbm": round(b_gbs / hbm_peak, 4),
                                      "attention_only_us": round(t_bat * 1e6, 2),
                                      "attention_only_gbs": round(b_at / t_bat / 1e9, 1),
                                      "attention_only_frac_of_hbm": round(b_at / t_bat / 1e9 / hbm_peak, 4)},
                "cached_candidates_by_batch": by_batch,
                "kv_append": kv_append,
                "block_stack": block,
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
            "gpu_launches": args.steps * launches_per_step,
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
    fa, _, _ = A.units()
    fb, _, _ = Bp.units()
    for _ in range(steps):
        A.reset(); Bp.reset()
        flush_buf.fill_(1)
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
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start the ranks here (users are sharded by rank)
        cmd = launcher_command(args.gpus, sys.argv[1:])
        sys.exit(subprocess.call(cmd))
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
