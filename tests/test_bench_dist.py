"""The multi-rank path of bench.py on CPU with gloo, world_size 2.

With N ranks each rank runs its own replica of the parameter set (the step
has no exchange step); the job's time is the max over ranks of the
device-timed region and its value is that time per parameter set over all
ranks.  Here the timings are planted per rank on the host.
"""
import os
import socket
import subprocess
import sys
from pathlib import Path

import pytest
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, str(ROOT))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank 1 is the slow one on the first number, rank 0 on the second
        mine = [10.0 + 5.0 * rank, 7.0 - 2.0 * rank]
        got = bench.reduce_max(mine, world)
        q.put((rank, got, bench.job_value(got[0], 4, world)))
    finally:
        dist.destroy_process_group()


def test_reduce_max_and_job_value_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, got, value in res:
        assert got == [15.0, 7.0], (rank, got)
        assert value == pytest.approx(15.0 / 4 / 2)


def test_job_value_single_rank():
    sys.path.insert(0, str(ROOT))
    import bench
    assert bench.job_value(100.0, 50, 1) == pytest.approx(2.0)
    assert bench.reduce_max([3.0, 4.0], 1) == [3.0, 4.0]


def test_reference_arm_under_torchrun_two_ranks():
    """--impl reference under torchrun: rank 0 times the oracle and prints
    one JSON line, the other rank exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), str(ROOT / "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--workload", "single-256x512-fp32"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    import json
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
