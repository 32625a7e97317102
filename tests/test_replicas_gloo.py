"""Multi-process path of bench.py on CPU: world_size 2 over gloo.

A multi-GPU bench run is N independent replicas of the training step; the
ranks meet only to take the slowest rank's time.  This checks that reduction
and the whole-job throughput on two gloo ranks (no GPU, no data collective).
"""
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


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    mine = [10.0 + 5.0 * rank, 20.0 - 3.0 * rank]  # rank 1 slower in the first, faster in the second
    got = bench.max_over_ranks(mine, "cpu")
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got))


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[0] == out[1] == [15.0, 20.0]


def test_replica_throughput_is_whole_job():
    sys.path.insert(0, ROOT)
    import bench
    # 2 replicas x 10 steps x 32768 tokens in a slowest-rank time of 2 s
    assert bench.replica_throughput(32768, 10, 2, 2000.0) == pytest.approx(327680.0)
