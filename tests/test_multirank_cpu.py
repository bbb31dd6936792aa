"""The multi-rank logic of bench.py on CPU with world_size 2 (gloo), no GPU.

Several GPUs run independent replicas of the update (weak scaling); the only
cross-rank steps are a barrier around the timed region and the max over ranks of
the elapsed time, from which rank 0 reports the job's ms per layer.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 30.0][rank]           # the second rank is the slow one
        dist.barrier()
        job = bench.max_over_ranks(local_ms, dist, "cpu")
        q.put((rank, job, bench.job_ms_per_layer(job, steps=10, n_dirs=2, world=world)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [30.0, 30.0]
    # 10 steps x 2 directions x 2 replicas in 30 ms
    assert res[0][2] == pytest.approx(30.0 / 40)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(7.0) == 7.0
    assert bench.job_ms_per_layer(7.0, 7, 1, 1) == 1.0


def test_reference_arm_only_rank_zero_reports():
    """Under torchrun every rank but 0 exits without work or output."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == ""


def test_gpu_count_must_match_world_size():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert out.returncode != 0
