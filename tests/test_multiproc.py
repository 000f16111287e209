"""The N > 1 plumbing of bench.py (replicas, max-over-ranks timing, whole-job
tokens/s) on CPU with world-size-2 gloo process groups."""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        assert bench.dist_env() == (world, rank, rank)
        cpu = torch.device("cpu")
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        bench.barrier(cpu)
        worst = bench.max_over_ranks(local_ms, cpu)
        value = bench.aggregate_tokens_per_s(224, 10, worst, world)
        q.put((rank, worst, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, worst, value in got:
        assert worst == 15.0                      # max over ranks, every rank sees it
        assert value == pytest.approx(2 * 224 * 10 / 15e-3)   # both replicas' tokens / slowest time


def test_single_process_helpers():
    sys.path.insert(0, ROOT)
    import torch
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.aggregate_tokens_per_s(224, 100, 50.0, 1) == pytest.approx(224 * 100 / 0.05)
    with pytest.raises(SystemExit):
        bench.main(["--gpus", "2", "--steps", "1", "--warmup", "3"])
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])
