"""The multi-GPU bench path is replicas only (independent problems per rank, no collective on the
data path).  Its host logic -- max-over-ranks timing, the whole-job aggregate, per-rank seeds and
the reference arm's rank-0-only behaviour -- runs here as two gloo ranks on the CPU."""
import io
import os
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                      # the slowest rank defines the job time
        mx = bench.max_over_ranks(torch, world, ms, device="cpu")
        val = bench.job_throughput(world, 32768, 4, mx)
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.replica_seed(1, rank))
        q.put((rank, mx, val, seeds))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, val, seeds in res:
        assert mx == 15.0
        assert val == pytest.approx(2 * 32768 * 4 / 0.015)
        assert len(set(seeds)) == 2       # independent problems per rank


def test_reference_arm_only_rank0_prints(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"])
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main()
    assert buf.getvalue() == ""
