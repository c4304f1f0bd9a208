"""The benchmark's multi-rank logic (replicas, max-over-ranks timing, rank-0
output) on two gloo ranks on the CPU."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.sync_barrier(dist, lambda: None)
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slow replica
        ms_max = bench.reduce_max(dist, ms, "cpu")
        value = bench.job_throughput(world, steps=4, layers=3, tokens=2, ms_max=ms_max)
        q.put((rank, ms_max, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]
    # 2 ranks x 4 steps x 3 layers x 2 tokens in 15 ms
    assert all(abs(r[2] - 48 / 0.015) < 1e-6 for r in res)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(None, 3.5, "cpu") == 3.5
    bench.sync_barrier(None, lambda: None)
    assert bench.job_throughput(1, 10, 48, 1, 100.0) == 4800.0


def test_reference_arm_line_on_the_host():
    """`bench.py --impl reference` times the oracle on the host and prints one JSON line
    with the contract's keys and the workload keys of the GPU arm's config."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_q8", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    import bench
    import synth
    want = bench.workload_config(synth.WORKLOADS["tiny_q8"], 1, 1, 1)
    assert {k: d["config"][k] for k in want} == want


def test_traffic_is_reported_only_for_the_captured_kernel_source(monkeypatch):
    """The roofline's `traffic` comes from profiles/traffic.json only while the kernel
    sources hash to the sha the ncu capture was taken on; otherwise it is null."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    key, entry = next(iter(rec.items()))
    stage, wl_name = key.split(":")
    monkeypatch.setattr(bench, "kernel_source_sha", lambda files=None: entry["source_sha"])
    assert bench.kernel_traffic(stage, wl_name) == entry["bytes_per_launch"]
    assert entry["bytes_per_launch"] == entry["dram_read"] + entry["dram_write"]
    assert bench.traffic_source(stage, wl_name)["status"] == "captured on this kernel source"
    monkeypatch.setattr(bench, "kernel_source_sha", lambda files=None: "0" * 16)
    assert bench.kernel_traffic(stage, wl_name) is None
    src = bench.traffic_source(stage, wl_name)
    assert src["captured_sha"] == entry["source_sha"] and src["kernel_source_sha"] == "0" * 16
    assert "changed" in src["status"] and src["command"] == entry["command"]
    assert bench.kernel_traffic(stage, "no_such_workload") is None
    assert "no ncu capture" in bench.traffic_source(stage, "no_such_workload")["status"]
    # each record names the kernel source files its sha covers (with every shared header)
    monkeypatch.undo()
    for k, e in rec.items():
        assert e["source_files"] and all(f.endswith(".cu") for f in e["source_files"]), k
        assert e["bytes_per_launch"] == e["dram_read"] + e["dram_write"], k


def test_reference_arm_under_torchrun_prints_once_from_rank_0(repo_tmp):
    """Launched like the scaling run (two ranks, 127.0.0.1): rank 0 alone times the oracle
    and prints the line; the other rank exits 0 without work."""
    import json
    import subprocess
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--workload", "tiny_q8", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, TMPDIR=str(repo_tmp))  # torchrun's log directory stays in the repository
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
