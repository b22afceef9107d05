"""The multi-GPU path of bench.py on CPU: two gloo ranks run the same max-over-ranks timing and
whole-job throughput code the N>1 benchmark uses (each rank runs an independent replica, so
the only exchange is the timing reduction), and the reference arm prints only on rank 0."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, ms_by_rank, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    ms = bench.max_over_ranks(ms_by_rank[rank], world, "cpu")
    value, ms_step = bench.job_throughput(2048, world, ms, 10)
    out.put((rank, ms, value, ms_step))
    dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ms_by_rank = [20.0, 25.0]
    procs = [ctx.Process(target=_rank, args=(r, 2, port, ms_by_rank, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value, ms_step in res:
        assert ms == 25.0                      # slowest rank
        assert abs(ms_step - 2.5) < 1e-12
        assert abs(value - 2 * 2048 / 2.5e-3) < 1e-6   # all ranks' tokens / max time


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.0, 1, "cpu") == 3.0
    assert bench.job_throughput(100, 1, 10.0, 5) == (100 / 2e-3, 2.0)


def test_reference_arm_silent_on_nonzero_rank():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
