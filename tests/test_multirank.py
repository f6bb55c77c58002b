"""Multi-rank host logic of the benchmark, on CPU with the gloo backend.

The scan's sequences are independent, so N GPUs each run their own batch
(weak scaling) and the only cross-rank work is timing: a barrier and a max of
the elapsed times.  Two gloo ranks check that the reduction returns the
slowest rank's time on every rank, that ranks draw different batches, and
that the whole-job throughput counts every rank's tokens.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        elapsed = 10.0 + 5.0 * rank                     # rank 1 is the slow one
        got = bench.max_over_ranks(elapsed, world, "cpu")
        w = bench.workload()
        out[rank] = (got, bench.rank_seed(w, rank))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_to_the_slowest_and_draw_distinct_batches():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] != res[1][1]


def test_whole_job_throughput_counts_every_rank():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    one = bench.tokens_per_second(1, 64, 65536, 10, 30.0)
    assert one == pytest.approx(64 * 65536 * 10 / 0.03)
    assert bench.tokens_per_second(4, 64, 65536, 10, 30.0) == pytest.approx(4 * one)
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
