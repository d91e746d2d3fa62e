"""Host side of bench.py's multi-GPU runs, on CPU with gloo.

Under torchrun every rank runs an independent replica of the layer on its
own tokens (the layer shards by tokens with no exchange).  The reported time
is the max over ranks and the throughput counts the tokens of all ranks;
this checks that reduction with two gloo ranks.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        # rank r was slower on the first timer, faster on the second
        got = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 0.25], "cpu")
        results[rank] = got
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world, start_method="spawn")
    assert results[0] == results[1] == [2.0, 5.0, 0.25]


def test_whole_job_throughput_counts_every_rank():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.whole_job_tokens_per_s(4096, 1, 2.0) == pytest.approx(2048000.0)
    assert bench.whole_job_tokens_per_s(4096, 8, 2.0) == pytest.approx(8 * 2048000.0)
    assert bench.max_over_ranks([3.0, 1.5], "cpu") == [3.0, 1.5]  # no process group: unchanged
