"""bench.py's N > 1 plumbing on the CPU: two gloo ranks on 127.0.0.1 take the job time as the
slowest rank's and report the throughput of all replicas; a rank other than 0 of the reference
arm leaves without work or output, and rank 0 of it prints one line of the bench contract."""
import datetime
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, queue):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        job_ms = bench.max_over_ranks(100.0 + 50.0 * rank, world, torch.device("cpu"))
        value = bench.job_throughput(1000, world, 10, job_ms)
        dist.barrier()
        queue.put((rank, job_ms, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_report_the_slowest_rank():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    got = sorted(queue.get(timeout=10) for _ in procs)
    assert [r for r, _, _ in got] == [0, 1]
    for _, job_ms, value in got:
        assert job_ms == 150.0  # every rank sees the slower rank's time
        assert value == pytest.approx(1000 * 2 * 10 / 0.150)  # both replicas' tokens


def test_single_rank_needs_no_process_group():
    import torch
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, 1, torch.device("cpu")) == 12.5
    assert bench.job_throughput(4096, 1, 3, 12.5) == pytest.approx(4096 * 3 / 0.0125)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout == ""


def test_reference_arm_rank0_prints_one_contract_line():
    import json
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "C0", "--steps", "2", "--warmup", "3",
                        "--cpu-seconds", "0.2"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = r.stdout.strip().splitlines()
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["higher_is_better"]
    assert d["steps"] == 2 and d["warmup"] == 3 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert "C0" in d["config"]["workload"]
