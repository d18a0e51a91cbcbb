"""Multi-rank host logic of bench.py on CPU: two gloo ranks as spawned processes.

The SageSLA path has no exchange step, so N GPUs run N batch elements independently. What must
hold across ranks: every rank takes the same collective steps, the job's step time is the
slowest rank's, the reported value counts the work of all ranks, and only rank 0 prints.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, step_ms, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w, local = bench.rank_env()
    bench.init_ranks(w, "gloo", timeout_s=60)
    dist.barrier()
    mx = bench.max_over_ranks_of(step_ms[r], w)
    value = bench.whole_job_tops(1e12, w, mx)
    dist.barrier()
    dist.destroy_process_group()
    out_q.put((r, w, local, mx, value))


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_whole_job_value(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    step_ms = [1.5, 2.5]
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, step_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, (rank, w, local, mx, value) in enumerate(res):
        assert (rank, w, local) == (r, world, r)
        assert mx == max(step_ms)                 # every rank sees the slowest rank's time
        assert value == pytest.approx(world * 1e12 / (max(step_ms) * 1e-3) / 1e12)


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    bench.init_ranks(1, "gloo")                   # no process group for one rank
    assert bench.max_over_ranks_of(3.0, 1) == 3.0
    assert bench.whole_job_tops(2e12, 1, 1000.0) == pytest.approx(2.0)


def test_reference_arm_prints_only_on_rank_zero():
    # Under torchrun every rank runs bench.py; the CPU oracle arm runs on rank 0 alone and
    # the other ranks exit 0 without work or output.
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_line_on_tiny_workload():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "cpu_baseline", "e2e", "config"):
        assert key in line
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
