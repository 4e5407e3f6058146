"""The multi-GPU path of bench.py on CPU: world_size-2 gloo ranks.

The layer forward has no exchange step on one node's data-parallel path,
so N GPUs run N independent replicas; the only cross-rank steps are the
barrier and the max-over-ranks reduction of the step time, and the job's
throughput counts every rank's tokens over the slowest rank's time.
"""
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [2.0, 3.5][rank]
        dist.barrier()
        ms = bench.max_over_ranks(local_ms, world, "cpu")
        q.put((rank, ms, bench.job_tokens_per_s(4096, world, ms)))
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_max_over_ranks_and_job_throughput_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [3.5, 3.5]            # every rank sees the slowest rank's time
    assert out[0][2] == pytest.approx(2 * 4096 / 3.5e-3)  # all ranks' tokens over that time


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(1.25, 1) == 1.25
    assert bench.job_tokens_per_s(4096, 1, 2.0) == pytest.approx(2048000.0)


def test_reference_arm_exits_quietly_on_nonzero_ranks():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
