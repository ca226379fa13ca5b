"""The multi-GPU path is N independent replicas (the layer has no exchange
step): ranks meet only for the timing barrier and the max over ranks.  These
run that host logic as world_size-2 gloo process groups on the CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, q):
    import sys
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    dist.barrier()
    mx = bench.max_over_ranks(times[rank], dist, "cpu")
    val = bench.job_throughput(1.0e12, 10, world, mx)
    q.put((rank, mx, val))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    times = [12.0, 15.0]     # per-rank device milliseconds for 10 steps
    procs = [ctx.Process(target=_worker, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, val in out:
        assert mx == 15.0                          # the slowest rank's time
        assert val == pytest.approx(1.0e12 * 10 * 2 / 15e-3)   # work of both ranks / max time


def test_single_rank_helpers():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert bench.job_throughput(2.0, 5, 1, 10.0) == pytest.approx(1000.0)


def _ref_worker(rank, world, port, q):
    """--impl reference under torchrun: rank 0 alone runs and prints; others exit 0."""
    import subprocess
    import sys
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--steps", "2", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    q.put((rank, p.returncode, p.stdout))


def test_reference_arm_prints_on_rank0_only():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ref_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict((r, (rc, so)) for r, rc, so in [q.get(timeout=300) for _ in procs])
    for p in procs:
        p.join(timeout=60)
    import json
    assert out[0][0] == 0 and out[1][0] == 0
    assert out[1][1].strip() == ""
    line = json.loads(out[0][1].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
