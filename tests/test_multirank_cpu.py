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


def test_bench_launch_plan():
    """`bench.py --gpus N` starts its own ranks when nothing else did, runs in place when
    torch.distributed.run started it with a matching world size, and refuses a mismatch."""
    import sys
    import bench
    assert bench.launch_plan(1, {}, ["--gpus", "1"]) is None
    assert bench.launch_plan(2, {"WORLD_SIZE": "2", "RANK": "1"}, ["--gpus", "2"]) is None
    cmd = bench.launch_plan(4, {}, ["--gpus", "4", "--steps", "5"], port=29511)
    assert cmd[:3] == [sys.executable, "-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert "--master-port=29511" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "5"] and cmd[-5].endswith("bench.py")
    with pytest.raises(ValueError, match="WORLD_SIZE=2"):
        bench.launch_plan(4, {"WORLD_SIZE": "2"}, [])
    with pytest.raises(ValueError):
        bench.launch_plan(0, {}, [])


def test_bench_self_launch_two_ranks_reference_arm():
    """`bench.py --impl reference --gpus 2` with no launcher around it: it starts two ranks
    itself (gloo is not needed: the reference arm runs on rank 0 only), rank 0 prints one JSON
    line with n_gpus 2 and both ranks exit 0."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--workload", "n128_d64_f32", "--steps", "1",
                          "--warmup", "0"], cwd=root, env=env, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
