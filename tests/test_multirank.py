"""The N > 1 path of the benchmark on the CPU: two gloo ranks (one process each,
as torchrun launches them) combine their timings with the same helpers the GPU
run uses -- the slowest rank's time, the whole job's units over it -- and every
rank takes the same collective steps.  Batch-1 decode runs as independent
replicas, so these are the only collectives."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms_local = 10.0 + 5.0 * rank        # rank 1 is the slower one
        ms = bench.max_over_ranks(ms_local, world, device="cpu")
        dist.barrier()
        e2e = bench.max_over_ranks(1.0 + rank, world, device="cpu")
        value = bench.whole_job_rate(6 * 3, world, ms / 1e3)
        out.put((rank, ms, e2e, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=90) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, ms, e2e, value in res:
        assert ms == 15.0 and e2e == 2.0           # every rank sees the maximum
        assert value == pytest.approx(6 * 3 * world / 0.015)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(10, 1, 2.0) == 5.0
