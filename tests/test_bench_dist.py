"""The benchmark's multi-rank logic on CPU: two gloo ranks.

bench.py runs one replica of the workload per GPU (the layer forward has no
exchange step), takes the slowest rank's device time and reports the units
all ranks processed over it. These tests drive that aggregation with gloo
processes on the host, and check that the CPU reference arm does its work on
rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, times, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    try:
        # the same collective steps, in the same order, as bench.main
        ms_max = bench.max_over_ranks(torch, dist, WORLD, times[rank][0], "cpu")
        e_max = bench.max_over_ranks(torch, dist, WORLD, times[rank][1], "cpu")
        q.put((rank, ms_max, e_max))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_gloo():
    times = [(12.5, 40.0), (13.75, 31.0)]          # per rank: device ms, e2e ms
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, times, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(WORLD))
    for rank, ms_max, e_max in got:
        assert ms_max == 13.75 and e_max == 40.0, (rank, ms_max, e_max)

    sys.path.insert(0, ROOT)
    import bench
    # 2 replicas x 10 steps x 1e9 bytes over the slowest rank's 13.75 ms
    v = bench.job_rate(1e9, 10, WORLD, 13.75, 1e9)
    assert v == pytest.approx(2 * 10 * 1e9 / 13.75e-3 / 1e9)
    # one rank alone over the same time reports half
    assert bench.job_rate(1e9, 10, 1, 13.75, 1e9) == pytest.approx(v / 2)


def test_max_over_ranks_single_process():
    import torch
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(torch, None, 1, 3.25, "cpu") == 3.25


def test_reference_arm_runs_on_rank0_only():
    """Under torchrun only rank 0 times the oracle; other ranks exit 0 silently."""
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "3", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_line_rank0():
    """Rank 0 prints one JSON line with the reference fields (tiny workload)."""
    env = dict(os.environ, RANK="0", LOCAL_RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "3", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 3 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["value"] > 0


def test_item_groups_pick_layers_sharing_input():
    """Grouped runs: q, k, v and gate, up of the Qwen2.5-3B set share their
    input; other workloads have no groups."""
    sys.path.insert(0, ROOT)
    import bench
    items = [(f"{n}/M=1", None, 1) for n in ("q", "k", "v", "o", "gate", "up", "down")]
    assert bench.item_groups("qwen25_3b", items) == [(0, 1, 2), (4, 5)]
    assert bench.item_groups("mamba2", [("in_proj/M=1", None, 1), ("out_proj/M=1", None, 1)]) == []
    # a group with one member left is no group
    assert bench.item_groups("qwen25_3b", [("q/M=1", None, 1), ("o/M=1", None, 1)]) == []


def test_reference_arm_encoder_line():
    """--impl reference --encoder: the oracle's k-means rounds and encode,
    one JSON line with the encoder metric and the reference fields."""
    env = dict(os.environ, RANK="0", LOCAL_RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--encoder", "tiny", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == "HXQ encoder weights/s" and d["unit"] == "weights/s"
    assert d["config"]["workload"].startswith("encode 256x256 mode 0, k=256")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["value"] > 0


def test_run_env_never_raises():
    import torch
    sys.path.insert(0, ROOT)
    import bench
    env = bench.run_env(torch, 0)
    assert ("gpu" in env and "torch" in env) or "error" in env


def test_cpu_baseline_times_cpp_oracle_on_one_and_all_threads():
    """The CPU baseline times the plain C++ oracle (compiled for the host) on
    one thread and on every host thread, on the bench's own workload."""
    sys.path.insert(0, ROOT)
    import bench
    items = bench.workload("tiny", 0, 1)
    r1, ra, n_all, desc = bench.oracle_sample(items, budget_s=0.3)
    assert n_all == (os.cpu_count() or 1)
    assert r1[0] > 0 and ra[0] > 0 and r1[2] >= 1 and ra[2] >= 1
    assert "C++ oracle" in desc and bench.cpu_model()
