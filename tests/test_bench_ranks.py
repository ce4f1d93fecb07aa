"""Host logic of bench.py's multi-GPU (replica) mode on CPU: two gloo ranks
agree on the max of their per-rank times, the whole-job value counts every
rank's work over that time, and the reference arm does its work on rank 0
only (the other ranks exit at once)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.reduce_max(times[rank])
        value = bench.whole_job_tflops(2.0e12, world, got)
        out[rank] = (got, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_replica_timing_takes_the_max_over_ranks():
    world = 2
    times = [3.5, 5.25]
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), times, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        ms, value = res[r]
        assert ms == max(times)
        assert value == pytest.approx(2.0e12 * world / (max(times) * 1e-3) / 1e12)


def test_single_process_reduce_is_identity():
    import bench
    assert bench.reduce_max(4.0) == 4.0
    assert bench.whole_job_tflops(1e12, 1, 1.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    called = []
    monkeypatch.setattr(bench, "cpu_inputs", lambda *a, **k: called.append(1))
    assert bench.main(["--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3"]) == 0
    assert not called
