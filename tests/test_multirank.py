"""The multi-rank plumbing of bench.py on CPU: world size 2 over gloo.

The path has no exchange step, so `bench.py --gpus N` runs N independent replicas; what the ranks
share is the timing rule (the step time is the slowest rank's) and the whole-job value (all ranks'
work over that time).  These tests run those two pieces in two real processes.
"""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        ms = bench.max_over_ranks(dist, times[rank])
        value = bench.whole_job_value(2.0e12, world, ms)
        out.put((rank, ms, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_step_time_is_the_slowest_rank_and_value_counts_every_rank():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    times = [7.5, 9.25]
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, out)) for r in range(2)]
    for p in procs:
        p.start()
    got = [out.get(timeout=100) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in got:
        assert ms == max(times)
        # 2e12 flops per rank per step, two ranks, 9.25 ms per step
        assert value == pytest.approx(2 * 2.0e12 / 9.25e-3 / 1e12)


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(None, 3.5) == 3.5
    assert bench.whole_job_value(1.0e12, 1, 1.0) == pytest.approx(1000.0)
