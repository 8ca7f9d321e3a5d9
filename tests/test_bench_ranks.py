"""The bench's cross-rank logic on two gloo ranks (CPU): the job time is the slowest rank's,
the job rate counts every rank's units, and the reference arm runs on rank 0 alone."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    ms = bench.rank_max(5.0 + 3.0 * rank, dist, "cpu")   # rank 0: 5 ms, rank 1: 8 ms
    rate = bench.job_rate(2.0e12, world, ms)
    os.environ["RANK"] = str(rank)
    ref = bench.run_reference(type("A", (), {})()) if rank != 0 else None
    dist.barrier()
    dist.destroy_process_group()
    torch.save({"ms": ms, "rate": rate, "ref": ref}, os.path.join(out, f"r{rank}.pt"))


@pytest.mark.timeout(120)
def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [torch.load(os.path.join(tmp_path, f"r{r}.pt")) for r in range(world)]
    for r in res:
        assert r["ms"] == 8.0                       # the slowest rank's time, on every rank
        assert r["rate"] == pytest.approx(2.0e12 * 2 / 8e-3 / 1e12)
    assert res[1]["ref"] == 0                       # the reference arm: rank 1 exits without work


def test_launch_count_follows_the_grouping_path():
    """Five kernels per call, six when pw_group renumbers windows first (rows of more than 8
    words that would take more than 2112 words of shared memory per warp staged whole)."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.launches_per_call(32, 128) == 6   # 64K tokens, W = 128
    assert bench.launches_per_call(32, 256) == 6
    assert bench.launches_per_call(32, 64) == 5    # 32 x 65 = 2080 words: staged
    assert bench.launches_per_call(16, 128) == 5   # 32K tokens: 16 x 129 = 2064 words
    assert bench.launches_per_call(8, 256) == 5    # at most 8 words: always staged
    assert bench.launches_per_call(1, 32) == 5
