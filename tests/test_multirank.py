"""The bench's multi-GPU logic on CPU: two gloo ranks (127.0.0.1). The path
shards into independent problems, so ranks exchange only their timings: the
step time is the max over ranks and throughput counts every rank's tokens."""
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
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # each rank measured something different; all must agree on the max
        ms, kms = bench.max_over_ranks([1.0 + rank, 0.5 * (world - rank)])
        value = bench.whole_job_throughput(16384, world, ms)
        out[rank] = (ms, kms, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_weak_scaling(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        ms, kms, value = out[r]
        assert ms == float(world)            # max of 1 + rank
        assert kms == 0.5 * world            # max of 0.5 * (world - rank)
        assert value == pytest.approx(16384 * world / (world * 1e-3))


def test_single_process_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert bench.whole_job_throughput(100, 1, 2.0) == pytest.approx(50000.0)
