"""Host-side pieces of bench.py that need no GPU: the committed DRAM-traffic record
is reported only for the kernel sources it was captured on, and the roofline
peaks come from the measured file (with the stated fallback)."""

import json

import bench


def test_traffic_record_is_consistent():
    """A one-pass capture whose per-launch bytes add up; reported only while the
    kernel sources still hash to the recorded digest (else the bench says null)."""
    rec = json.load(open(bench.TRAFFIC_RECORD))
    assert rec["passes"] == 1
    assert rec["dram_bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    if rec["kernel_source_sha256"] == bench.kernel_source_digest():
        assert bench.recorded_traffic() == rec["dram_bytes_per_launch"]
    else:
        assert bench.recorded_traffic() is None


def test_traffic_is_withheld_for_other_sources(tmp_path, monkeypatch):
    rec = json.load(open(bench.TRAFFIC_RECORD))
    rec["kernel_source_sha256"] = "0" * 64
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", str(path))
    assert bench.recorded_traffic() is None
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", str(tmp_path / "missing.json"))
    assert bench.recorded_traffic() is None


def test_kernel_digest_covers_every_listed_source(tmp_path, monkeypatch):
    files = []
    for i in range(3):
        f = tmp_path / f"s{i}.cu"
        f.write_text(f"source {i}")
        files.append(str(f))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", files)
    d0 = bench.kernel_source_digest()
    (tmp_path / "s2.cu").write_text("source 2 changed")
    assert bench.kernel_source_digest() != d0


def test_peaks_fall_back_when_the_measured_file_is_absent(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    hbm, tf, tf_sus, src = bench.load_peaks()
    assert (hbm, tf, src) == (6650.0, 1590.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6000.0, "bf16_tflops": 1500.0}))
    hbm, tf, tf_sus, src = bench.load_peaks()
    assert (hbm, tf, src) == (6000.0, 1500.0, "measured")


def test_launcher_command_starts_one_rank_per_gpu():
    cmd = bench.launcher_command(4, ["--gpus", "4", "--steps", "3"], port=12345)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--nnodes=1" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[cmd.index("--master-port") + 1] == "12345"
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"] and cmd[-5].endswith("bench.py")


def test_world_mismatch_is_refused():
    import pytest
    assert bench.check_world(1, {}) == (0, 1, 0)
    assert bench.check_world(2, {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"}) == (1, 2, 1)
    with pytest.raises(SystemExit):
        bench.check_world(8, {"WORLD_SIZE": "1", "RANK": "0"})


def _rank_worker(rank, world, port, q):
    import os
    import hashlib
    import torch.distributed as dist
    import workloads as W
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    r, w, local = bench.check_world(world, os.environ)
    dist.init_process_group("gloo", rank=r, world_size=w)
    seeds = bench.rank_seeds(r)
    c = W.cached_cand(seed=seeds["cached_cand"])
    digest = hashlib.sha256(c.hist_k[:64].tobytes() + c.q_cand[:64].tobytes()).hexdigest()
    q.put((r, local, seeds, c.hist_lengths.tolist(), digest))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_get_distinct_user_batches():
    """Weak scaling: each rank of a 2-rank launch reads its rank from the
    launcher's environment and draws its own batch of users; rank 0's batch is
    the reference workload."""
    import os
    import torch.multiprocessing as mp
    import workloads as W
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 31500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_rank_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, l0, s0, h0, d0), (r1, l1, s1, h1, d1) = res
    assert (r0, l0, r1, l1) == (0, 0, 1, 1)
    assert s0 != s1 and d0 != d1
    assert h0 == W.cached_cand().hist_lengths.tolist()
