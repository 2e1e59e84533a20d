"""Host logic of the N-GPU benchmark on CPU: two gloo ranks on 127.0.0.1.

The path has no collective on its data (every (batch, head) pair is independent, so N GPUs run N
replicas); the only cross-rank steps are the barriers around the timed region and the maximum of the
per-rank timings, which these tests exercise with world size 2.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        # rank r reports (10 + r, 20 - r): the job time is each column's slowest rank
        got = bench.max_over_ranks([10.0 + rank, 20.0 - rank], "cpu")
        value = bench.whole_job_tokens_per_s(32768, world, got[0])
        dist.barrier()
        out.put((rank, got, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_max_over_ranks_and_whole_job_value_two_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    world, port = 2, _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=150) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, value in res:
        assert got == [11.0, 20.0]
        # 2 replicas x 32768 tokens in 11 ms
        assert value == pytest.approx(2 * 32768 / 11e-3)


def test_max_over_ranks_without_process_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.5, 7], "cpu") == [3.5, 7.0]
    assert bench.whole_job_tokens_per_s(1000, 1, 2.0) == pytest.approx(5e5)
