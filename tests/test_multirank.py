"""The bench's multi-rank path on CPU: two gloo ranks, each with its own
independent layer (weak scaling).  Only the timing maximum and the work sum
cross ranks; the reference arm runs on rank 0 alone."""
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


def _rank_main(rank, world, port, out):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        total_ms = 100.0 + 10.0 * rank     # rank 1 is the slower one
        e2e_ms = 200.0 - 50.0 * rank       # rank 0 is slower end to end
        flops = 1e12 * (rank + 1)
        res = bench.aggregate(total_ms, e2e_ms, flops, world, torch.device("cpu"))
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_aggregate_takes_max_time_and_sums_work():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        total, e2e, flops = out[r]
        assert total == 110.0
        assert e2e == 200.0
        assert flops == 3e12


def test_single_rank_aggregate_is_identity():
    import torch
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate(5.0, 7.0, 3.0, 1, torch.device("cpu")) == (5.0, 7.0, 3.0)


@pytest.mark.parametrize("rank", ["1"])
def test_reference_arm_other_ranks_exit_without_work(rank):
    env = dict(os.environ, RANK=rank, WORLD_SIZE="2", LOCAL_RANK=rank)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
