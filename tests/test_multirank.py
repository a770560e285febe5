"""Multi-GPU bookkeeping of bench.py, run as two gloo ranks on the CPU.

The decode path does not shard a block: blocks are independent, so N GPUs
run N replicas on disjoint blocks (no data-path collective).  What the ranks
share is the measurement: the device time is the maximum over ranks, the
bytes and weights are summed, and the job throughput divides the summed units
by the slowest rank's time.  These tests run that code with world size 2 on
the gloo backend.
"""
import datetime
import os
import socket

import pytest

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        maxima, sums = bench.reduce_over_ranks([1.5 + rank, 10.0 * rank], [100.0 * (rank + 1), 7.0])
        q.put((rank, maxima, sums, bench.rank_seed(rank), bench.rank_seed(rank, per_rank=32)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_and_seed():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in procs:
            rank, maxima, sums, seed, seed32 = q.get(timeout=120)
            got[rank] = (maxima, sums, seed, seed32)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    for rank in (0, 1):
        maxima, sums, _, _ = got[rank]
        assert maxima == [2.5, 10.0]            # max over ranks
        assert sums == [300.0, 14.0]            # summed over ranks
    assert [got[r][2] for r in (0, 1)] == [1000, 1001]      # one block per rank
    assert [got[r][3] for r in (0, 1)] == [1000, 1032]      # 32-block streams do not overlap


def test_single_process_is_identity():
    assert bench.reduce_over_ranks([3.0], [4.0, 5.0]) == ([3.0], [4.0, 5.0])


@pytest.mark.parametrize("units,steps,ms,want", [(300e9, 10, 1000.0, 3000.0), (1e9, 1, 1.0, 1000.0)])
def test_job_rate(units, steps, ms, want):
    assert bench.job_rate(units, steps, ms) == pytest.approx(want)

