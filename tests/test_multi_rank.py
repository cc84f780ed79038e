"""The multi-GPU path of the benchmark on CPU: two gloo ranks, each timing its
own replica, agree on the slowest rank's time and on the whole-job value."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch.distributed as dist
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    local = [10.0 + rank, 1.0 + 2 * rank, 5.0 - rank]      # rank-specific timings
    agg = bench.max_over_ranks(local)
    val = bench.whole_job_tflops(1e12, 100, world, agg[0])
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, agg, val))


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_whole_job_value(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, agg, val in res:
        assert agg == [11.0, 3.0, 5.0]
        # 2 replicas x 100 steps x 1e12 flops in 11 ms
        assert abs(val - 2 * 100 * 1e12 / 11e-3 / 1e12) < 1e-6


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert abs(bench.whole_job_tflops(2e12, 10, 1, 20.0) - 1000.0) < 1e-9
