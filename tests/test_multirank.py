"""bench.py's multi-rank plumbing on CPU: two gloo ranks (no GPU).

Every rank runs its own independent batch; the job's time is the slowest
rank's, taken with one all-reduce.  The reference arm prints on rank 0 only.
"""
import io
import os
import contextlib
import socket

import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = bench.max_over_ranks(values[rank])
        assert bench.dist_env() == (rank, world, rank)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    world = 2
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    values = [3.5, 7.25]
    mp.spawn(_worker, args=(world, _free_port(), values, out), nprocs=world, join=True)
    assert dict(out) == {0: 7.25, 1: 7.25}


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks(4.0) == 4.0


def test_reference_arm_prints_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()

    class Args:
        ref_rows = 8
        steps = 1
        warmup = 1
        gpus = 2

    with contextlib.redirect_stdout(buf):
        rc = bench.run_reference(Args(), bench.workloads.CONFIGS["tiny"])
    assert rc == 0 and buf.getvalue() == ""


def test_gpus_must_match_launched_processes():
    """``--gpus N`` with fewer (or more) processes than N is refused, so that
    one process can never be reported as N GPUs."""
    assert bench.check_world(1, 1) is None
    assert bench.check_world(4, 4) is None
    assert "torch.distributed.run" in bench.check_world(8, 1)
    assert bench.check_world(2, 4) is not None


def test_bench_refuses_gpus_without_launcher():
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--steps", "1"],
                       capture_output=True, text=True, cwd=root, env=env)
    assert r.returncode != 0
    assert "--gpus 2 but 1 process" in r.stderr
