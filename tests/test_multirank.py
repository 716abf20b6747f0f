"""The multi-rank path of bench.py on CPU: two gloo ranks reduce their
timings to the max over ranks and report whole-job throughput (replicas:
no data-path collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 5.0])
    value = bench.whole_job_gbs(10 ** 9, 4, world, got[0])
    dist.destroy_process_group()
    q.put((rank, got, value))


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_gloo(world):
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
    for _, got, value in res:
        assert got == [2.0, 10.0, 5.0]
        # 2 ranks x 1 GB x 4 steps over the slowest rank's 2 ms
        assert abs(value - 2 * 4 / 2e-3) < 1e-6


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert bench.whole_job_gbs(2 * 10 ** 9, 10, 1, 1000.0) == 20.0
