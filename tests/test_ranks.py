"""The replica (N>1) path of bench.py on CPU: world-size-2 gloo process groups.

The layer does not shard (every rank runs the whole workload on its own GPU),
so what multi-rank runs add is the timing rule: the device time of a run is the
largest over ranks, and the throughput is every rank's token rows over it.
"""
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, values, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(dist, values[rank], "cpu")
        out.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    values = [3.25, 7.5]
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, values, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: 7.5, 1: 7.5}          # every rank sees the slowest rank's time


def test_max_over_ranks_without_group():
    assert bench.max_over_ranks(None, 4.0, "cpu") == 4.0


def test_replica_throughput_counts_every_rank():
    # 2 ranks x 4 token rows x 100 steps in 50 ms
    assert bench.replica_throughput(2, 4, 100, 50.0) == pytest.approx(16000.0)
    assert bench.replica_throughput(1, 4, 100, 50.0) == pytest.approx(8000.0)


def test_reference_arm_other_ranks_exit_without_work():
    # Under torchrun only rank 0 times the oracle and prints; rank 1 prints nothing.
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "1"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
