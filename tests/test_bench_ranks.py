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


def test_reference_arm_prints_the_contract_line(monkeypatch, capsys):
    """Rank 0 of the reference arm times the oracle and prints one JSON line with
    the contract's keys (shrunken inputs so that it runs in a moment)."""
    import json

    import numpy as np

    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    rng = np.random.default_rng(0)
    small = {"up": (rng.standard_normal((64, 64)), rng.standard_normal((64, 32))),
             "down": (rng.standard_normal((64, 64)), rng.standard_normal((64, 32)))}
    monkeypatch.setattr(bench, "SHAPES", {"up": (64, 32), "down": (64, 32)})
    monkeypatch.setattr(bench, "cpu_inputs", lambda *a, **k: small)
    assert bench.main(["--impl", "reference", "--steps", "2", "--warmup", "1"]) == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    r = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in r, key
    assert r["impl"] == "reference" and r["steps"] == 2 and r["warmup"] == 1
    assert r["value"] > 0 and r["cpu_baseline"]["kind"] == "oracle" and r["cpu_baseline"]["cores"] >= 1
    assert r["cpu_baseline"]["value"] == r["value"]
    assert r["e2e"]["h2d_bytes_per_step"] == 0 and r["e2e"]["d2h_bytes_per_step"] == 0
    assert r["e2e"]["value"] == r["value"] and r["e2e"]["unit"] == r["unit"]


def test_traffic_figure_only_while_the_kernel_is_unchanged(monkeypatch, tmp_path):
    """roofline.traffic comes from the committed ncu summary of the product
    kernel, and only while the kernel source still hashes to the value recorded
    there: a changed kernel reports null."""
    import hashlib
    import re
    import bench
    t = bench.load_traffic()
    recorded = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", open(bench.TRAFFIC_FILE).read()).group(1)
    current = hashlib.sha256(open(bench.GEMM_SOURCE, "rb").read()).hexdigest()
    if recorded == current:
        assert t is not None and t > 0
    else:  # the kernel changed after the capture: no figure until it is recaptured
        assert t is None
    changed = tmp_path / "rmm_gemm.cu"
    changed.write_bytes(open(bench.GEMM_SOURCE, "rb").read() + b"\n// changed\n")
    monkeypatch.setattr(bench, "GEMM_SOURCE", str(changed))
    assert bench.load_traffic() is None


def test_metric_counts_the_methods_k():
    """The useful-FLOP count of every reported point uses k = ceil(rho * d) as
    the oracle states it (pinned to the paper's worked counts)."""
    import bench
    import oracle
    for d in (128, 256, 4096, 8192, 14336, 28672, 32768):
        for rho in (0.25, 0.5, 0.6, 0.7, 0.8, 0.9, 1.0):
            assert bench.retained(rho, d) == oracle.retained_count(rho, d), (rho, d)


def test_cpu_baseline_repeats_the_sample_until_its_time_budget(monkeypatch):
    """The RMM arm's cpu_baseline times the oracle sample repeatedly until the
    requested CPU time is reached (at least once, at most max_reps times), and
    reports the flops and seconds of all repetitions together."""
    import bench
    clock = {"t": 0.0}

    def fake_sample(inputs64, rho, rows):
        clock["t"] += 0.3
        return 0.3, 2.0 * rows

    monkeypatch.setattr(bench, "oracle_sample", fake_sample)
    t, f, reps = bench.oracle_timed(None, 0.8, 64, min_seconds=1.0)
    assert reps == 4 and abs(t - 1.2) < 1e-9 and f == 4 * 128.0
    t, f, reps = bench.oracle_timed(None, 0.8, 64, min_seconds=0.0)
    assert reps == 1 and f == 128.0
    t, f, reps = bench.oracle_timed(None, 0.8, 64, min_seconds=100.0, max_reps=5)
    assert reps == 5
