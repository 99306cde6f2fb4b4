"""The multi-process path of the benchmark on CPU ranks (gloo, world size 2).

The operator is single-GPU and runs replicas only: under torchrun every rank
processes its own volume, ranks exchange nothing on the data path, the step
time is the maximum over ranks and the whole-job value counts every rank's
tokens.  These tests run that host logic on two gloo processes."""
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


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    per_rank_ms = [1.25, 2.5][rank]            # the second replica is the slower one
    ms = bench.max_over_ranks(per_rank_ms, world)
    value = bench.replica_value(65536, world, ms)
    bench.barrier(world)
    q.put((rank, ms, value))
    dist.destroy_process_group()


def test_replica_step_time_is_max_over_ranks_and_value_counts_all_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in got:
        assert ms == 2.5
        assert value == pytest.approx(65536 * 2 / 2.5e-3)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
