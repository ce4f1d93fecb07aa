"""Benchmark of Reduced Matrix Multiplication (RMM) on B200.

One step = one pass of the whole RMM hot path (column scores, TopK, staging of
A[:, I], the gathered tensor-core product) over the Llama-3.1-8B-shaped MLP
workload at n = 4096 tokens, rho = 0.8, bf16: the up/gate-projection shape
(A 4096 x 4096, B 4096 x 14336) and the down-projection shape
(A 4096 x 14336, B 14336 x 4096), each with its own index set.

Metric: useful TFLOP/s = sum of 2 n ceil(rho d) m over the step / step time,
with the same kernels at rho = 1 (identity index set) and cuBLAS dense
matmul reported beside it.  Inputs (149 MB and 234 MB per op) exceed the
126 MB L2, so no flush runs between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl rmm|reference]
N > 1 runs one independent replica per GPU (weak scaling, no collective on the
data path; a barrier and a max over ranks bracket the timing).
`--impl reference` times the CPU oracle (a deliberately slow fp64 program) on
a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "RMM op latency and useful TFLOP/s (2·n·⌈ρd⌉·m) vs ρ=1, % of bf16 peak"
WORKLOAD = "llama3.1-8b-mlp-linear-rmm"
SHAPES = {"up": (4096, 14336), "down": (14336, 4096)}
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "pair_gemm_llama8b_mlp_n4096.md")
GEMM_SOURCE = os.path.join(ROOT, "input_adaptive_reduced_b200", "csrc", "rmm_gemm.cu")


def retained(rho: float, d: int) -> int:
    x = rho * d
    r = round(x)
    k = r if abs(x - r) <= 1e-9 * d else math.ceil(x)
    return max(1, min(d, int(k)))


def useful_flops(n: int, rho: float) -> float:
    return float(sum(2.0 * n * retained(rho, d) * m for d, m in SHAPES.values()))


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        return pk["bf16_tflops"], pk.get("bf16_tflops_sustained"), pk["hbm_gbs"], "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


def load_traffic():
    """Per-launch DRAM bytes of the product kernel from the committed ncu summary,
    only if the kernel source has not changed since the counters were taken."""
    try:
        text = open(TRAFFIC_FILE).read()
        want = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", text).group(1)
        have = hashlib.sha256(open(GEMM_SOURCE, "rb").read()).hexdigest()
        if want != have:
            return None
        return float(re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text).group(1))
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sms, maxs, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sms.append(float(parts[0]))
                maxs.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for name, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(name)
        loaded = [s for s, p in zip(sms, power) if p > 250.0] or sms
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(maxs) if maxs else None,
                "reasons": sorted(reasons), "samples": len(sms),
                "power_w_max": max(power) if power else None}


def reduce_max(value: float, device=None) -> float:
    """Max of a per-rank time over all ranks (the replica timing rule); the
    identity when no process group is initialised."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Useful TFLOP/s of the whole job: every rank's work over the slowest rank's time."""
    return flops_per_rank_step * world / (ms_per_step * 1e-3) / 1e12


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample(inputs64, rho: float, rows: int):
    """Time the oracle on full selection of both ops plus `rows` output rows of
    each product.  Returns (seconds, useful flops done)."""
    import oracle
    t0 = time.perf_counter()
    flops = 0.0
    for name, (A64, B64) in inputs64.items():
        d, m = SHAPES[name]
        I, _ = oracle.select(A64, rho=rho)
        oracle.reduced_product(A64, B64, I, rows=list(range(rows)))
        flops += 2.0 * rows * len(I) * m
    return time.perf_counter() - t0, flops


def oracle_timed(inputs64, rho: float, rows: int, min_seconds: float, max_reps: int = 100):
    """Repeat oracle_sample until at least `min_seconds` of CPU work (at least
    once, at most `max_reps` times).  Returns (seconds, useful flops, repetitions)."""
    t, f, reps = 0.0, 0.0, 0
    while reps < max(1, max_reps) and (reps == 0 or t < min_seconds):
        ti, fi = oracle_sample(inputs64, rho, rows)
        t += ti
        f += fi
        reps += 1
    return t, f, reps


def cpu_inputs(n_rows: int, seed: int):
    import workloads as W
    import oracle
    out = {}
    for name, gen in (("up", W.mlp_up), ("down", W.mlp_down)):
        A, B = gen(seed, n=n_rows)
        out[name] = (oracle.as_f64(A), oracle.as_f64(B))
    return out


def cores_used() -> int:
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n and n.isdigit() else (os.cpu_count() or 1)


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    n, rho = args.n, args.rho
    inputs64 = cpu_inputs(n, seed=1)
    # size the per-step sample so that warmup + steps stay within ~3 minutes
    t1, _ = oracle_sample(inputs64, rho, rows=1)
    t5, _ = oracle_sample(inputs64, rho, rows=5)
    per_row = max((t5 - t1) / 4.0, 1e-4)
    budget = 180.0 / max(1, args.steps + args.warmup)
    rows = int(max(1, min(64, (budget - t1) / per_row)))
    for _ in range(args.warmup):
        oracle_sample(inputs64, rho, rows)
    total_t, total_f = 0.0, 0.0
    for _ in range(args.steps):
        t, f = oracle_sample(inputs64, rho, rows)
        total_t += t
        total_f += f
    value = total_f / total_t / 1e12
    ms = total_t / args.steps * 1e3
    sample = (f"full selection (scores + TopK) of both ops and {rows} of {n} output rows of each "
              f"reduced product per step, fp64, OpenMP over rows")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "n": n, "rho": rho, "shapes": SHAPES, "sample_rows": rows},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores_used(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- RMM arm
def run_rmm(args):
    import torch
    import torch.distributed as dist
    import input_adaptive_reduced_b200 as rmm
    import workloads as W

    rank, world, local = dist_env()
    if args.gpus != world:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}; using WORLD_SIZE", file=sys.stderr)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the RMM kernels have no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    n, rho = args.n, args.rho
    stream = torch.cuda.current_stream(dev)
    ops = {}
    for name, gen in (("up", W.mlp_up), ("down", W.mlp_down)):
        d, m = SHAPES[name]
        A, B = gen(1000 * rank + 1, n=n, device=dev)
        entry = {"A": A, "B": B, "d": d, "m": m}
        for tag, r in (("rmm", rho), ("dense", 1.0)):
            p = rmm.rmm_problem_init(rmm.RMM_LINEAR, rmm.RMM_BF16, n, d, m)
            p.rho = r
            plan = rmm.Plan(p)
            ws = rmm.workspace_for(plan, dev, stream)
            entry[tag] = {"plan": plan, "ws": ws, "k": plan.k,
                          "Y": torch.empty((n, m), dtype=torch.bfloat16, device=dev)}
        ops[name] = entry

    def run_op(e, tag):
        c = e[tag]
        rmm.rmm_matmul(c["plan"], e["A"], e["B"], c["Y"], None, c["ws"], stream)

    def step(tag="rmm"):
        for e in ops.values():
            run_op(e, tag)

    # warm-up
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)

    # product-kernel events, one pair per op per timed step
    n_ev = args.steps * len(ops)
    ev_start = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    ev_stop = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    for e in ev_start + ev_stop:
        e.record(stream)
    torch.cuda.synchronize(dev)

    sampler = ClockSampler(local)
    sampler.start()
    barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    i_ev = 0
    for _ in range(args.steps):
        for e in ops.values():
            c = e["rmm"]
            c["plan"].set_product_events(ev_start[i_ev], ev_stop[i_ev])
            run_op(e, "rmm")
            i_ev += 1
    t_stop.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop()
    for e in ops.values():
        e["rmm"]["plan"].set_product_events(None, None)
    rmm.check_workspaces()

    ms_total = reduce_max(t_start.elapsed_time(t_stop), dev)
    ms_step = ms_total / args.steps
    flops_step = useful_flops(n, rho)
    value = whole_job_tflops(flops_step, world, ms_step)

    # product kernel (dominant kernel): algorithmic flops per launch / event time
    gemm_ms = [s.elapsed_time(t) for s, t in zip(ev_start, ev_stop)]
    per_op = list(ops.values())
    gemm_flops = [2.0 * n * per_op[i % len(per_op)]["rmm"]["k"] * per_op[i % len(per_op)]["m"]
                  for i in range(len(gemm_ms))]
    achieved = sum(gemm_flops) / (sum(gemm_ms) * 1e-3) / 1e12
    peak_burst, peak_sust, hbm, peak_src = load_peaks()
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak_burst, "unit": "TFLOP/s",
                "frac": achieved / peak_burst, "traffic": load_traffic(),
                "peak_kind": f"{peak_src} cuBLAS bf16 burst",
                "frac_of_sustained": (achieved / peak_sust) if peak_sust else None,
                "kernel": "pair_gemm_kernel<bf16, kBRows, 256, split> (CTA pair, cta_group::2, 256x256 tiles, split tail)",
                "avg_launch_us": sum(gemm_ms) / len(gemm_ms) * 1e3}

    # per-op latency at rho and at rho = 1 (same kernels, identity I) and cuBLAS dense
    def op_latency(fn, iters=20):
        for _ in range(3):
            fn()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(iters):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / iters

    points = {}
    for name, e in ops.items():
        d, m = e["d"], e["m"]
        t_r = op_latency(lambda: run_op(e, "rmm"))
        t_1 = op_latency(lambda: run_op(e, "dense"))
        t_cb = op_latency(lambda: torch.matmul(e["A"], e["B"]))
        k = e["rmm"]["k"]
        points[name] = {"n": n, "d": d, "m": m, "k": k, "ms": t_r,
                        "useful_tflops": 2.0 * n * k * m / (t_r * 1e-3) / 1e12,
                        "ms_rho1": t_1, "tflops_rho1": 2.0 * n * d * m / (t_1 * 1e-3) / 1e12,
                        "ms_cublas_dense": t_cb, "speedup_vs_rho1": t_1 / t_r,
                        "kernel_launches": e["rmm"]["plan"].kernel_launches}

    # more evidence timed by the same run (outside the headline timed region):
    # the Llama-3-70B MLP ops and the attention forms at n = 4096
    if not args.no_extra_points:
        points.update(extra_points(dev, stream, rho, op_latency))

    # end to end through the public API with host buffers (pinned), copies timed
    e2e = None
    if not args.no_e2e:
        host = {}
        h2d = d2h = 0
        for name, e in ops.items():
            hA = e["A"].cpu().pin_memory()
            hB = e["B"].cpu().pin_memory()
            hY = torch.empty_like(e["rmm"]["Y"], device="cpu").pin_memory()
            dA = torch.empty_like(e["A"])
            dB = torch.empty_like(e["B"])
            host[name] = (hA, hB, hY, dA, dB)
            h2d += hA.numel() * hA.element_size() + hB.numel() * hB.element_size()
            d2h += hY.numel() * hY.element_size()

        # Copies in and out run on their own streams and overlap the products:
        # an op's product waits for its inputs, its copy-out waits for the
        # product, the next step's copy-in of those inputs waits until the
        # product that read them is done, and the next product into Y waits
        # for Y's copy-out.
        h2d_stream = torch.cuda.Stream(dev)
        d2h_stream = torch.cuda.Stream(dev)
        ev = {name: {"in": torch.cuda.Event(), "done": torch.cuda.Event(), "out": torch.cuda.Event()}
              for name in ops}
        for name in ops:
            for x in ev[name].values():
                x.record(stream)

        def e2e_step():
            for name, e in ops.items():
                hA, hB, hY, dA, dB = host[name]
                h2d_stream.wait_event(ev[name]["done"])
                with torch.cuda.stream(h2d_stream):
                    dA.copy_(hA, non_blocking=True)
                    dB.copy_(hB, non_blocking=True)
                ev[name]["in"].record(h2d_stream)
                stream.wait_event(ev[name]["in"])
                stream.wait_event(ev[name]["out"])
                c = e["rmm"]
                rmm.rmm_matmul(c["plan"], dA, dB, c["Y"], None, c["ws"], stream)
                ev[name]["done"].record(stream)
                d2h_stream.wait_event(ev[name]["done"])
                with torch.cuda.stream(d2h_stream):
                    hY.copy_(c["Y"], non_blocking=True)
                ev[name]["out"].record(d2h_stream)

        def join():
            for name in ops:
                stream.wait_event(ev[name]["out"])

        for _ in range(3):
            e2e_step()
        join()
        torch.cuda.synchronize(dev)
        e2e_steps = max(3, min(args.steps, 20))
        barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        h2d_stream.wait_event(a)  # the timed copies start after the start event
        for _ in range(e2e_steps):
            e2e_step()
        join()
        b.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = reduce_max(a.elapsed_time(b) / e2e_steps, dev)
        e2e = {"value": whole_job_tflops(flops_step, world, ms_e2e), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
               "path": "pinned host A, B -> device, rmm_matmul (C ABI), Y -> pinned host; copies in "
                       "and out on their own streams, overlapping the products"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        rows = args.cpu_rows
        inputs64 = cpu_inputs(n, seed=1)
        t, f, reps = oracle_timed(inputs64, rho, rows, args.cpu_seconds)
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": cores_used(), "kind": "oracle",
               "sample": f"{reps} x (full selection of both ops and {rows} of {n} output rows of each "
                         f"product), fp64 C with OpenMP over rows; {t:.1f} s"}

    launches = sum(e["rmm"]["plan"].kernel_launches for e in ops.values()) * args.steps
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Llama-3.1-8B-shaped activations and N(0,0.02) weights)",
            "config": {"workload": WORKLOAD, "n": n, "rho": rho, "shapes": SHAPES,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "inputs larger than L2 (149 MB and 234 MB per op); no flush"},
            "roofline": roofline, "points": points, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def extra_points(dev, stream, rho, op_latency):
    """Per-op latency at rho, at rho = 1 and of the dense torch product for the
    Llama-3-70B up / down projections at n = 4096 and for causal attention
    (32 query heads, 8 KV heads, L = 4096, d_h = 128): QK^T, PV scoring P
    itself, and PV taking the token scores written by the softmax kernel that
    produced P (producer-fused scoring; the softmax timed on its own)."""
    import torch
    import input_adaptive_reduced_b200 as rmm
    import workloads as W
    out = {}
    n = 4096
    for shape in ("up", "down"):
        A, B = W.linear_70b(1, n=n, shape=shape, device=dev)
        d, m = A.shape[1], B.shape[1]
        k = retained(rho, d)
        t_r = op_latency(lambda: rmm.matmul(A, B, rho=rho))
        t_1 = op_latency(lambda: rmm.matmul(A, B, rho=1.0))
        t_cb = op_latency(lambda: torch.matmul(A, B))
        out[f"70b_{shape}"] = {"n": n, "d": d, "m": m, "k": k, "ms": t_r,
                               "useful_tflops": 2.0 * n * k * m / (t_r * 1e-3) / 1e12, "ms_rho1": t_1,
                               "ms_cublas_dense": t_cb, "speedup_vs_rho1": t_1 / t_r}
        del A, B
        torch.cuda.empty_cache()
    H, Hkv, dh = 32, 8, 128
    Q, K = W.attn_qk(1, n=n, device=dev)
    Kt = K.repeat_interleave(H // Hkv, dim=0).transpose(1, 2)
    t_r = op_latency(lambda: rmm.qk(Q, K, rho=rho, causal=True))
    t_1 = op_latency(lambda: rmm.qk(Q, K, rho=1.0, causal=True))
    t_d = op_latency(lambda: torch.matmul(Q, Kt))
    out["qk_causal"] = {"heads": H, "kv_heads": Hkv, "L": n, "d_h": dh, "k": retained(rho, dh), "ms": t_r,
                        "ms_rho1": t_1, "ms_torch_dense": t_d, "speedup_vs_rho1": t_1 / t_r}
    # scores of the causal attention for the softmax (bf16, -inf above the diagonal)
    S = rmm.qk(Q, K, rho=1.0, causal=True)
    del Q, K, Kt
    torch.cuda.empty_cache()
    V = (torch.randn((Hkv, n, 128), generator=W.gen(2, dev), device=dev)).to(torch.bfloat16)
    t_sm = op_latency(lambda: rmm.softmax_scores(S, causal=True))
    P, s2 = rmm.softmax_scores(S, causal=True)
    del S
    torch.cuda.empty_cache()
    Vr = V.repeat_interleave(H // Hkv, dim=0)
    k = retained(rho, n)
    t_r = op_latency(lambda: rmm.pv(P, V, rho=rho, causal=True))
    t_g = op_latency(lambda: rmm.pv(P, V, rho=rho, causal=True, scores=s2))
    t_1 = op_latency(lambda: rmm.pv(P, V, rho=1.0, causal=True))
    t_d = op_latency(lambda: torch.matmul(P, Vr))
    out["pv_causal"] = {"heads": H, "kv_heads": Hkv, "L": n, "d_v": 128, "k": k, "ms": t_r,
                        "ms_given_scores": t_g, "ms_rho1": t_1, "ms_torch_dense": t_d,
                        "ms_softmax_with_scores": t_sm, "speedup_vs_rho1": t_1 / t_r,
                        "speedup_vs_rho1_given_scores": t_1 / t_g}
    del P, V, Vr, s2
    torch.cuda.empty_cache()
    # fused RMM attention (features rho, tokens rho) against the same three steps as
    # separate ops (scores written, softmax with token scores, PV on the given
    # scores) and torch's dense causal attention (scaled_dot_product_attention)
    Q, K = W.attn_qk(1, n=n, device=dev)
    V = (torch.randn((Hkv, n, 128), generator=W.gen(2, dev), device=dev)).to(torch.bfloat16)
    alpha = 1.0 / math.sqrt(dh)
    t_f = op_latency(lambda: rmm.attention(Q, K, V, rho, rho, causal=True, alpha=alpha))
    t_f1 = op_latency(lambda: rmm.attention(Q, K, V, 1.0, 1.0, causal=True, alpha=alpha))

    def unfused():
        S = rmm.qk(Q, K, rho=rho, alpha=alpha, causal=True)
        P, s2 = rmm.softmax_scores(S, causal=True)
        return rmm.pv(P, V, rho=rho, causal=True, scores=s2)
    t_u = op_latency(unfused)
    t_sdpa = None
    try:
        Kr, Vr = K.repeat_interleave(H // Hkv, dim=0), V.repeat_interleave(H // Hkv, dim=0)
        t_sdpa = op_latency(lambda: torch.nn.functional.scaled_dot_product_attention(
            Q[None], Kr[None], Vr[None], is_causal=True))
        del Kr, Vr
    except Exception:
        pass
    flops_qk = 2.0 * H * retained(rho, dh) * n * (n + 1) / 2  # causal half of the scores, per pass
    out["attention_fused_causal"] = {"heads": H, "kv_heads": Hkv, "L": n, "d_h": dh, "rho_d": rho, "rho_t": rho,
                                     "ms": t_f, "ms_rho1": t_f1, "ms_unfused_ops": t_u,
                                     "ms_torch_sdpa_dense": t_sdpa, "passes_over_the_scores": 3,
                                     "score_tflops_per_pass": flops_qk / (t_f * 1e-3) / 1e12}
    del Q, K, V
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- sweep
def write_bandwidth(dev, stream, nbytes=1 << 30, iters=10):
    """Write-only HBM rate (GB/s): a 1 GiB fill, timed with CUDA events.  The
    measured copy peak counts a read and a write per byte; an op whose traffic
    is almost all writes is bound by this lower figure instead."""
    import torch
    buf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    for _ in range(3):
        buf.fill_(1)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(iters):
        buf.fill_(1)
    b.record(stream)
    torch.cuda.synchronize(dev)
    gbs = nbytes * iters / (a.elapsed_time(b) * 1e-3) / 1e9
    del buf
    return gbs


def run_sweep(args):
    """Latency, useful TFLOP/s and roofline fraction at every point of the five
    workloads (RMM at each rho, the same kernels at rho = 1, and the dense
    torch/cuBLAS product), written as JSON lines to --sweep-out."""
    import torch
    import input_adaptive_reduced_b200 as rmm
    import workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peak_tf, _, peak_gbs, _ = load_peaks()
    out = open(args.sweep_out, "w") if args.sweep_out else None
    # --sweep-only "cfg:op:n[:rho],...": run only the matching points
    only = [tuple(x.split(":")) for x in args.sweep_only.split(",")] if args.sweep_only else None

    def want(cfg, op, n, rho=None):
        if only is None:
            return True
        for sel in only:
            if (sel[0] == str(cfg) and (len(sel) < 2 or sel[1] == op) and (len(sel) < 3 or sel[2] == str(n))
                    and (rho is None or len(sel) < 4 or abs(float(sel[3]) - rho) < 1e-9)):
                return True
        return False

    write_gbs = write_bandwidth(dev, stream) if any(want(3, "qk", n) for n in (1024, 2048, 4096)) else None

    def lat(fn, iters=20):
        for _ in range(3):
            fn()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(iters):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / iters

    def emit(rec):
        line = json.dumps(rec)
        print(line, flush=True)
        if out:
            out.write(line + "\n")
            out.flush()

    # GPU time of 20 ops replayed from a CUDA graph, so that the host's launch
    # cost is not what is timed (tiny and decode-sized ops)
    gs = torch.cuda.Stream(dev)

    def graph_lat(fn, reps=20):
        with torch.cuda.stream(gs):
            for _ in range(3):
                fn()
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=gs):
            for _ in range(reps):
                fn()
        best = float("inf")
        for _ in range(5):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(gs)
            with torch.cuda.stream(gs):
                g.replay()
            b.record(gs)
            torch.cuda.synchronize(dev)
            best = min(best, a.elapsed_time(b) / reps)
        del g
        return best

    def linear_points(cfg, name, A, B, rhos):
        n, d = A.shape
        m = B.shape[1]
        t_dense = lat(lambda: torch.matmul(A, B))
        for rho in rhos:
            if not want(cfg, name, n, rho):
                continue
            k = retained(rho, d)
            t = lat(lambda: rmm.matmul(A, B, rho=rho))
            flops = 2.0 * n * k * m
            hbm = 2.0 * (n * d + k * m + n * m)  # A once, retained B rows once, Y
            bound = "tensor" if n >= 512 else "hbm"
            frac = (flops / (t * 1e-3) / 1e12) / peak_tf if bound == "tensor" else (hbm / (t * 1e-3) / 1e9) / peak_gbs
            rec = {}
            if cfg == 1:  # a few microseconds of GPU work: the op and cuBLAS replayed from graphs too
                Y = torch.empty((n, m), dtype=A.dtype, device=dev)
                rec = {"ms_gpu_graph": graph_lat(lambda: rmm.matmul(A, B, rho=rho, out=Y)),
                       "ms_dense_gpu_graph": graph_lat(lambda: torch.matmul(A, B, out=Y))}
            emit({"config": cfg, "op": name, "n": n, "d": d, "m": m, "rho": rho, "k": k, "ms": t,
                  "useful_tflops": flops / (t * 1e-3) / 1e12, "gbs": hbm / (t * 1e-3) / 1e9,
                  "bound": bound, "frac": frac, "ms_dense_cublas": t_dense, **rec})

    # 1: tiny fp32
    if want(1, "fp32", 64):
        A, B = W.linear_small(1, device=dev)
        linear_points(1, "fp32", A, B, [0.25, 0.5, 1.0])
    # 2: Llama-3.1-8B MLP
    for n in (1024, 2048, 4096):
        for name, gen in (("up", W.mlp_up), ("down", W.mlp_down)):
            if not want(2, name, n):
                continue
            A, B = gen(1, n=n, device=dev)
            linear_points(2, name, A, B, [0.5, 0.7, 0.8, 1.0])
            del A, B
    # 3: QK^T, 32 heads / 8 KV heads, d_h = 128, causal
    for n in (1024, 2048, 4096):
        if not want(3, "qk", n):
            continue
        Q, K = W.attn_qk(1, n=n, device=dev)
        Kt = K.repeat_interleave(4, dim=0).transpose(1, 2)
        t_dense = lat(lambda: torch.matmul(Q, Kt))
        for rho in (0.5, 0.8, 1.0):
            if not want(3, "qk", n, rho):
                continue
            k = retained(rho, 128)
            t = lat(lambda: rmm.qk(Q, K, rho=rho, causal=True))
            flops = 2.0 * n * k * n * 32
            hbm = 32 * (2.0 * n * 128 + 2 * 2.0 * n * k + 2.0 * n * n) + 8 * 2.0 * n * 128
            # the op's traffic is the n x n score matrix it writes: judged against the
            # write-only HBM rate measured in this run
            s_bytes = 32 * 2.0 * n * n
            emit({"config": 3, "op": "qk", "n": n, "rho": rho, "k": k, "ms": t,
                  "useful_tflops": flops / (t * 1e-3) / 1e12, "gbs": hbm / (t * 1e-3) / 1e9,
                  "bound": "hbm_write", "write_gbs": s_bytes / (t * 1e-3) / 1e9, "write_peak_gbs": write_gbs,
                  "frac": s_bytes / (t * 1e-3) / 1e9 / write_gbs, "frac_of_copy_peak": hbm / (t * 1e-3) / 1e9 / peak_gbs,
                  "ms_dense_torch": t_dense})
        del Q, K, Kt
    # 4: PV, token selection
    for n in (2048, 4096):
        if not want(4, "pv", n):
            continue
        P, V = W.attn_pv(1, n=n, device=dev)
        Vr = V.repeat_interleave(4, dim=0)
        t_dense = lat(lambda: torch.matmul(P, Vr))
        # P is a causal softmax: "pv" states it (RMM_FLAG_CAUSAL, the blocks above the
        # diagonal are skipped); "pv_nocausal" reads all of P
        for op, causal in (("pv", True), ("pv_nocausal", False)):
            for rho in (0.5, 0.8, 1.0):
                if not want(4, op, n, rho):
                    continue
                k = retained(rho, n)
                t = lat(lambda: rmm.pv(P, V, rho=rho, causal=causal))
                flops = 2.0 * n * k * 128 * 32
                p_bytes = 2.0 * n * (n + 1) / 2 if causal else 2.0 * n * n  # P's nonzero part once
                hbm = 32 * (p_bytes + 2.0 * k * 128 + 2.0 * n * 128)  # P once, V rows, O
                emit({"config": 4, "op": op, "n": n, "rho": rho, "k": k, "ms": t,
                      "useful_tflops": flops / (t * 1e-3) / 1e12, "gbs": hbm / (t * 1e-3) / 1e9,
                      "bound": "hbm", "frac": hbm / (t * 1e-3) / 1e9 / peak_gbs, "ms_dense_torch": t_dense})
        del P, V, Vr
    # decode step: one query row per head against t cached tokens (Llama-3.1-8B
    # attention: 32 / 8 heads, d_h = d_v = 128, `batch` sequences); GPU time of
    # 20 ops replayed from a CUDA graph
    for batch, t in ((1, 4096), (8, 4096), (8, 32768), (16, 32768)):
        key = f"{batch}x{t}"
        if not (want("decode", "qk", key) or want("decode", "pv", key)):
            continue
        q, K, V, P = W.attn_decode(1, t=t, batch=batch, device=dev)
        H, Hkv = q.shape[0], K.shape[0]
        for op, mode, X, Z, m in (("qk", rmm.RMM_QK, q, K, t), ("pv", rmm.RMM_PV, P, V, 128)):
            for rho in (0.5, 0.8, 1.0):
                if not want("decode", op, key, rho):
                    continue
                d = X.shape[2]
                p = rmm.rmm_problem_init(mode, rmm.RMM_BF16, 1, d, m)
                p.rho = rho
                p.heads, p.kv_heads = H, Hkv
                p.lda, p.ldb = d, Z.shape[2]
                p.stride_a, p.stride_b = X.stride(0), Z.stride(0)
                p.ldy, p.stride_y = m, m
                if mode == rmm.RMM_QK:
                    p.alpha = 1.0 / math.sqrt(d)
                plan = rmm.Plan(p)
                ws = rmm.workspace_for(plan, dev, gs)
                Y = torch.empty((H, 1, m), dtype=torch.bfloat16, device=dev)
                I = torch.empty((H, plan.k), dtype=torch.int32, device=dev)
                t_op = graph_lat(lambda: rmm.rmm_matmul_batched(plan, X, Z, Y, I, ws, gs))
                t_sel = graph_lat(lambda: rmm.rmm_select(plan, X, I, None, ws, gs)) if plan.k < d else 0.0
                if mode == rmm.RMM_QK:
                    # K in full (the scores need every key), q, S
                    hbm = 2.0 * Hkv * t * d + 2.0 * H * d + 2.0 * H * t
                    rec = {"kv_bytes_read": 2.0 * Hkv * t * d}
                else:
                    # P, the V rows of the union of each group's token sets, O
                    grp = I.view(Hkv, -1)
                    union = sum(int(torch.unique(grp[j]).numel()) for j in range(Hkv))
                    hbm = 2.0 * H * t + 2.0 * union * m + 2.0 * H * m
                    rec = {"v_rows_read": union, "v_rows_total": Hkv * t}
                emit({"config": "decode", "op": op, "batch": batch, "t": t, "rho": rho, "k": plan.k,
                      "ms": t_op, "ms_select": t_sel, "kernel_launches": plan.kernel_launches,
                      "useful_gflop": 2.0 * H * plan.k * (t if mode == rmm.RMM_QK else m) / 1e9,
                      "gbs": hbm / (t_op * 1e-3) / 1e9, "bound": "hbm",
                      "frac": hbm / (t_op * 1e-3) / 1e9 / peak_gbs, **rec})
        del q, K, V, P
    # fused RMM attention (features and tokens at rho) against the three steps as
    # separate ops, and the softmax that writes P with its token scores
    for n in (1024, 2048, 4096):
        if not (want("attn", "fused", n) or want("attn", "softmax", n)):
            continue
        H, Hkv, dh = 32, 8, 128
        Q, K = W.attn_qk(1, n=n, device=dev)
        V = (torch.randn((Hkv, n, 128), generator=W.gen(2, dev), device=dev)).to(torch.bfloat16)
        alpha = 1.0 / math.sqrt(dh)
        if want("attn", "softmax", n):
            S = rmm.qk(Q, K, rho=1.0, alpha=alpha, causal=True)
            t = lat(lambda: rmm.softmax_scores(S, causal=True))
            moved = 32 * (2.0 * n * (n + 1) / 2 + 2.0 * n * n)  # causal half of S read, P written in full
            emit({"config": "attn", "op": "softmax", "n": n, "ms": t, "gbs": moved / (t * 1e-3) / 1e9,
                  "bound": "hbm", "frac": moved / (t * 1e-3) / 1e9 / peak_gbs})
            del S
        for rho in (0.5, 0.8, 1.0):
            if not want("attn", "fused", n, rho):
                continue
            t = lat(lambda: rmm.attention(Q, K, V, rho, rho, causal=True, alpha=alpha))
            flops = 2.0 * H * retained(rho, dh) * n * (n + 1) / 2  # one causal pass over the reduced scores
            emit({"config": "attn", "op": "fused", "n": n, "rho": rho, "ms": t, "bound": "tensor",
                  "score_tflops_per_pass": flops / (t * 1e-3) / 1e12, "passes": 3})
        del Q, K, V
    # low-bit form: E4M3 operands with per-tensor scales, bf16 output, on the
    # Llama-3.1-8B MLP shapes; dense reference: torch's scaled fp8 matmul
    for n in (2048, 4096):
        for name, gen in (("up", W.mlp_up), ("down", W.mlp_down)):
            if not want("fp8", name, n):
                continue
            A, B = gen(1, n=n, device=dev)
            Aq, sa = W.quantize_e4m3(A)
            Bq, sb = W.quantize_e4m3(B)
            del A, B
            d, m = Aq.shape[1], Bq.shape[1]
            t_dense = None
            try:
                Bcm = Bq.t().contiguous().t()
                one = torch.ones((), device=dev)
                t_dense = lat(lambda: torch._scaled_mm(Aq, Bcm, scale_a=one * sa, scale_b=one * sb,
                                                       out_dtype=torch.bfloat16))
            except Exception:
                pass
            for rho in (0.5, 0.8, 1.0):
                if not want("fp8", name, n, rho):
                    continue
                k = retained(rho, d)
                t = lat(lambda: rmm.matmul(Aq, Bq, rho=rho, alpha=sa * sb))
                flops = 2.0 * n * k * m
                emit({"config": "fp8", "op": name, "n": n, "d": d, "m": m, "rho": rho, "k": k, "ms": t,
                      "useful_tflops": flops / (t * 1e-3) / 1e12, "bound": "tensor",
                      "frac_of_bf16_peak": flops / (t * 1e-3) / 1e12 / peak_tf,
                      "ms_dense_scaled_mm": t_dense})
            del Aq, Bq
    # 5: Llama-3-70B linear
    for shape in ("up", "down", "qkv"):
        for n in (1, 16, 512, 2048, 4096):
            if not want(5, shape, n):
                continue
            A, B = W.linear_70b(1, n=n, shape=shape, device=dev)
            linear_points(5, shape, A, B, [0.5, 0.6, 0.7, 0.8, 1.0])
            del A, B
    if out:
        out.close()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["rmm", "reference"], default="rmm")
    ap.add_argument("--n", type=int, default=4096)
    ap.add_argument("--rho", type=float, default=0.8)
    ap.add_argument("--cpu-rows", type=int, default=64)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="repeat the CPU oracle sample until this much CPU time has been timed")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-extra-points", action="store_true",
                    help="skip the 70B and attention points timed after the headline")
    ap.add_argument("--sweep", action="store_true", help="time every point of the five workloads")
    ap.add_argument("--sweep-out", default=None)
    ap.add_argument("--sweep-only", default=None,
                    help='comma-separated "config:op:n[:rho]" points, e.g. "5:down:16:0.8,3:qk:4096"')
    args = ap.parse_args(argv)
    if args.sweep:
        return run_sweep(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_rmm(args)


if __name__ == "__main__":
    sys.exit(main())
