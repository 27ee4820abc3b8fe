"""Multi-rank host logic of bench.py, run as two `gloo` ranks on the CPU.

The attention work units are independent, so `bench.py --gpus N` runs one
replica of the step per rank with no data-path collective; the only
cross-rank steps are the barrier around the timed region and the max-over-
ranks reduction of the measured time.  These tests drive exactly those
helpers with ranks that report different times, and check that the
reference arm leaves every rank but 0 without work.
"""

import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

WORLD = 2


def _rank_main(rank, world, port, times, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = bench.max_over_ranks(times[rank], dist, torch.device("cpu"))
        val = bench.whole_job_tflops(world, 1e12, 4, ms)
        q.put((rank, ms, val))
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("times", [(10.0, 25.0), (40.0, 7.5), (3.25, 3.25)])
def test_max_over_ranks_gloo(times):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, WORLD, port, times, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(WORLD))
    want = max(times)
    for rank, ms, val in got:
        # every rank sees the slowest rank's time
        assert ms == want
        # 2 ranks x 4 steps x 1 TFLOP each, over the slowest rank's seconds
        assert val == pytest.approx(WORLD * 4 / (want / 1e3))


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(12.5, None, torch.device("cpu")) == 12.5
    assert bench.whole_job_tflops(1, 2e12, 5, 1000.0) == pytest.approx(10.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
