"""The multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, ms_list, q):
    import sys
    import datetime
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms_max = bench.max_over_ranks(ms_list[rank], world, "cpu")
        value = bench.whole_job_tflops(1e12, 10, world, ms_max)
        dist.barrier()
        q.put((rank, ms_max, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_whole_job_value():
    world, port = 2, _free_port()
    ms = [40.0, 50.0]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms_max, value in got:
        assert ms_max == 50.0                          # every rank sees the slowest time
        assert value == pytest.approx(2 * 1e12 * 10 / 0.050 / 1e12)  # all ranks' work


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.whole_job_tflops(2e12, 5, 1, 10.0) == pytest.approx(1000.0)
