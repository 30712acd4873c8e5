"""The multi-rank host logic of bench.py on the CPU: two gloo ranks (world size 2).

Every rank runs its own full workload (heads are independent: weak scaling, no collective on the
data path); a multi-rank step takes the slowest rank's time (max over ranks) and the whole-job
throughput counts the units of all ranks. The reference (oracle) arm runs on rank 0 only.
"""
import os
import socket
import subprocess
import sys
from datetime import timedelta

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        ms = bench.reduce_max(10.0 + 5.0 * rank, world, device="cpu")  # rank 1 is the slower one
        rate = bench.weak_scaling_rate(1000.0, world, ms)
        dist.barrier()
        out.put((rank, ms, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = sorted(out.get(timeout=5) for _ in range(2))
    for rank, ms, rate in got:
        assert ms == 15.0  # every rank reports the slowest rank's time
        assert rate == pytest.approx(1000.0 * 2 / 0.015)  # units of both ranks over that time


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.weak_scaling_rate(10.0, 1, 2.0) == pytest.approx(5000.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1"], cwd=ROOT, env=env,
                       capture_output=True, timeout=300)
    assert r.returncode == 0, r.stderr.decode()[-2000:]
    assert r.stdout.strip() == b""
