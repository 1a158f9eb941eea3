"""Multi-process (world size 2, gloo, CPU) checks of bench.py's replica logic.

Every rank runs an independent replica of the decode step (the path has no
exchange step), so the only cross-rank operations are the barrier around the
timed region and the max-over-ranks reduction of the step time; the whole-job
value counts every replica's verified tokens.  No GPU is used.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        bench.sync_ranks()
        local_ms = 1.5 + rank            # rank 1 is the slow replica
        slowest = bench.max_over_ranks(local_ms)
        value = bench.weak_scaling_value(32, world, slowest)
        out[rank] = (slowest, value)
        bench.sync_ranks()
    finally:
        dist.destroy_process_group()


def test_replicas_take_max_time_and_sum_tokens():
    world = 2
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
        slowest, value = out[r]
        assert slowest == pytest.approx(2.5)
        assert value == pytest.approx(2 * 32 / 2.5e-3)


def test_single_process_helpers_without_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.25) == 3.25
    bench.sync_ranks()
    assert bench.weak_scaling_value(32, 1, 4.0) == pytest.approx(8000.0)


def test_dist_env_parsing(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "4")
    monkeypatch.setenv("RANK", "3")
    monkeypatch.setenv("LOCAL_RANK", "3")
    assert bench.dist_env() == (3, 4, 3)


def test_reference_arm_runs_only_on_rank_zero(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    args = bench.parse_args(["--impl", "reference", "--gpus", "2"])
    assert bench.run_reference(args) is None
