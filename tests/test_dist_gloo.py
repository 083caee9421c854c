"""Multi-process logic of bench.py on CPU (gloo, world size 2): the barrier,
the max-over-ranks of the timings and the whole-job throughput; and the
reference arm printing on rank 0 only.  No GPU."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.rank_barrier(world)
        ms = 10.0 + 5.0 * rank                     # rank 1 is the slow one
        mx = bench.max_over_ranks_value(ms, world, "cpu")
        out[rank] = (mx, bench.job_throughput(world, 1e12, 4, mx))
        bench.rank_barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world, port = 2, free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 15.0
    # 2 ranks x 1e12 flop x 4 steps over the slowest rank's 15 ms
    assert abs(out[0][1] - 2 * 1e12 * 4 / 15e-3 / 1e12) < 1e-9
    assert out[0][1] == out[1][1]


def test_job_throughput_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks_value(3.5, 1, "cpu") == 3.5
    assert abs(bench.job_throughput(1, 2e12, 10, 20.0) - 1000.0) < 1e-9


def _run_reference(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--gpus", "2", "--steps", "2", "--warmup", "1", "--workload", "tiny",
                           "--ref-budget-s", "1"],
                          capture_output=True, text=True, env=env, timeout=300)


def test_reference_arm_rank1_is_silent():
    r = _run_reference(1)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line():
    r = _run_reference(0)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
