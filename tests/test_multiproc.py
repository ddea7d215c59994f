"""The N>1 path of the benchmark on CPU: world-size-2 gloo ranks. The layer shards as
independent replicas (no data-path collective); what crosses ranks is the timing reduction
(max over ranks) and the whole-job aggregate, plus the reference arm's rank-0-only rule."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out_q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.reduce_max_over_ranks(times[rank], dist, world, device="cpu")
        out_q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_timing_reduction_takes_the_slowest_rank():
    world = 2
    times = [[10.0, 3.0, 7.0], [12.0, 2.5, 9.5]]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert res[r] == [12.0, 3.0, 9.5]


def test_whole_job_aggregate_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_tops(77.3e9, 1, 0.05)
    two = bench.whole_job_tops(77.3e9, 2, 0.05)
    assert two == pytest.approx(2 * one)
    assert one == pytest.approx(77.3e9 / 0.05e-3 / 1e12)


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny_256"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env0 = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    r0 = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                         "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny_256"],
                        capture_output=True, text=True, env=env0, timeout=300)
    assert r0.returncode == 0
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TOPS" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    # the JSON line's contract: every key present, the baseline described
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["steps"] == 1 and line["warmup"] >= 3 and line["higher_is_better"] is True
    assert line["config"]["workload"] == "tiny_256"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == line["value"]
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["unit"] == line["unit"]

