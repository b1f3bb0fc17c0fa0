"""bench.py's multi-rank plumbing on CPU: two `gloo` ranks (the path runs as
independent replicas; the only collectives are the timing reduction and the
barriers around the timed region)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, values, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        got = bench.max_over_ranks(values[rank], "cpu")
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    values = [3.25, 7.5]                     # per-rank step times (ms)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank, args=(r, 2, port, values, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in ps), [p.exitcode for p in ps]
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: 7.5, 1: 7.5}           # every rank reports the slowest rank's time


def test_max_over_ranks_without_a_group():
    assert bench.max_over_ranks(2.5, "cpu") == 2.5


@pytest.mark.parametrize("world", [1, 2, 8])
def test_whole_job_rate_counts_every_rank(world):
    # 4096 tokens per rank in 0.1 ms (the max over ranks): the job's rate
    assert bench.whole_job_rate(4096, world, 0.1) == pytest.approx(4096 * world / 1e-4)
