#!/usr/bin/env python
"""Throughput of exact ring attention on B200: causal-adjusted TFLOP/s, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
                    [--pass fwd|bwd|decode|merge|ring|ring-bwd] [--algo auto|tcgen05|tcgen05_1sm|simt]
                    [--ring-ranks R]

A step is one ring_attn_fwd call over the whole workload (every query shard folds
every KV shard in ring order). Default workload: bf16, B=1, H=8, S=1,048,576,
D=128, P=32, causal striped. Inputs are seeded synthetic tensors resident in HBM
(larger than L2, so no flush is needed between steps). With N>1 every rank runs
its own independent instance (seed + rank): weak scaling, no collective on the data
path; the step time is the max over ranks. `--gpus N` outside torchrun starts the N
ranks itself.

--pass ring spreads one sequence over ranks instead (the pages' ring: KV shards
travel between ranks while each rank folds the one it holds): virtual ranks on one
GPU, or one rank per GPU under torchrun. --pass ring-bwd does the same for the
backward (KV shards and their dK/dV accumulators travel the other way).

--impl reference times the fp64 CPU oracle (the correctness reference) on a
bounded sample of query rows of the same workload; rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

METRIC = "causal-adjusted attention TFLOP/s and % of B200 dense BF16 peak, 1 GPU"
DEFAULT_WORKLOAD = "c5_bf16_s1m_striped"
# the dominant kernel of the D=128 path and the sources that define it; its committed DRAM
# traffic figure is used only while these files are unchanged
KERNEL_NAME = "ring_fwd_sm100_2sm_kernel"
KERNEL_SRCS = [os.path.join(ROOT, "sequence_exact_attention_ring_b200", "csrc", f)
               for f in ("fwd_sm100_2sm.cu", "softmax_rows.cuh", "sm100_ptx.cuh", "ring_schedule.h")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ring_fwd_sm100_2sm_traffic.json")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synthetic.WORKLOADS))
    ap.add_argument("--algo", default="auto", choices=["auto", "tcgen05", "tcgen05_1sm", "simt"],
                    help="forward kernel (auto: the library's choice for the workload)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU time of the oracle sample")
    ap.add_argument("--pass", dest="which", default="fwd", choices=["fwd", "bwd", "decode", "merge", "ring", "ring-bwd"],
                    help="fwd: the forward hot path (the headline line); bwd: ring_attn_bwd on the same workload; "
                         "decode: one decode step against the workload's K/V as the cache; ring: the ring spread "
                         "over ranks (virtual ranks on one GPU, or one rank per GPU under torchrun)")
    ap.add_argument("--ring-ranks", type=int, default=8,
                    help="--pass ring on one GPU: number of virtual ranks the sequence is spread over")
    return ap.parse_args()


def relaunch_under_torchrun(args) -> int:
    """`--gpus N` (N > 1) outside torchrun: start N ranks on this node with torchrun and
    return its exit code (rank 0 prints the line)."""
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.run(cmd).returncode


# ------------------------------------------------------------------ distributed plumbing

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        # a short timeout: ranks that wait for one another end with an error, not a hang
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gather_objects(obj, world):
    if world == 1:
        return [obj]
    import torch.distributed as dist
    out = [None] * world
    dist.all_gather_object(out, obj)
    return out


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of this GPU every 200 ms while the timed region runs."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int):
        self.proc = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, flag in zip(names, parts[3:]):
                if flag.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ peaks / traffic

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_sha256() -> str:
    h = hashlib.sha256()
    for path in KERNEL_SRCS:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def kernel_traffic_per_launch(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it matches the current kernel source."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    if d.get("kernel_source_sha256") != kernel_source_sha256():
        return None
    per = d.get("bytes_per_launch", {}).get(workload)
    return float(per) if per is not None else None


# ------------------------------------------------------------------ CPU oracle sample

def oracle_sample_rate(w, q, k, v, target_seconds: float, seed_offset: int = 0):
    """Time the fp64 oracle on seeded query rows of one head; returns (TFLOP/s, rows, seconds, flops)."""
    import oracle
    from threadpoolctl import threadpool_info
    g = torch.Generator().manual_seed(w.seed + 2000 + seed_offset)
    b = 0
    h = int(torch.randint(0, w.Hq, (1,), generator=g).item())
    n_probe = 8
    ts = torch.randperm(w.S, generator=g)[:4096].tolist()
    picked, flops, elapsed = [], 0.0, 0.0
    qh = q[b:b + 1, h:h + 1].cpu()
    g_kv = h // (w.Hq // w.Hkv)
    kh = k[b:b + 1, g_kv:g_kv + 1].cpu()
    vh = v[b:b + 1, g_kv:g_kv + 1].cpu()
    idx = 0
    while idx < len(ts) and (elapsed < target_seconds):
        batch = ts[idx: idx + n_probe]
        idx += len(batch)
        rows = [(0, 0, t) for t in batch]
        t0 = time.perf_counter()
        oracle.attention_rows(qh, kh, vh, rows, w.causal, w.scale)
        elapsed += time.perf_counter() - t0
        picked += batch
        flops += sum(4.0 * w.D * ((t + 1) if w.causal else w.S) for t in batch)
        n_probe = min(64, n_probe * 2)
    cores = 0
    for info in threadpool_info():
        if info.get("user_api") == "blas":
            cores = max(cores, int(info.get("num_threads", 0)))
    return flops / elapsed / 1e12, len(picked), elapsed, flops, max(cores, 1), h


# ------------------------------------------------------------------ arms

def run_reference(args, world, rank):
    """The correctness reference (fp64 CPU oracle) on bounded samples of the workload."""
    if rank != 0:
        return
    w = synthetic.get(args.workload)
    dev = "cuda" if (w.gen_device == "cuda" and torch.cuda.is_available()) else "cpu"
    if w.gen_device == "cuda" and dev == "cpu":
        print(json.dumps({"impl": "reference", "unavailable": "workload inputs are drawn on a CUDA device"}))
        return
    q, k, v = synthetic.make_inputs(w, dev)
    per_step = max(0.2, min(args.cpu_seconds, 120.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup):
        oracle_sample_rate(w, q, k, v, per_step / 4, seed_offset=i)
    rates, rows, secs, cores = [], 0, 0.0, 1
    for i in range(args.steps):
        r, n, s, _, cores, _ = oracle_sample_rate(w, q, k, v, per_step, seed_offset=100 + i)
        rates.append(r)
        rows += n
        secs += s
    value = statistics.median(rates)
    total = w.causal_flops()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total / (value * 1e12) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{rows} query rows of one head per step (fp64 oracle, full score rows), "
                                   f"{secs:.1f} s total; ms_per_step extrapolates to the whole workload"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def workload_config(w):
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "S": w.S, "D": w.D, "P": w.P,
            "causal": w.causal, "layout": w.layout, "heavy_keys": w.heavy_keys,
            "l2": "inputs larger than L2 (no flush)" if w.qkvo_bytes() > 126e6 else "L2 flushed between steps",
            "flops_per_step": w.causal_flops()}


def flush_l2(buf):
    if buf is not None:
        buf.add_(1)


def run_ours(args, world, rank, local):
    from sequence_exact_attention_ring_b200 import HostRunner, binding, ring_attention, status
    w = synthetic.get(args.workload)
    binding.load()
    dev = torch.device("cuda", local if world > 1 else 0)
    w_rank = synthetic.custom(w.name, w.dtype, w.B, w.Hq, w.Hkv, w.S, w.D, w.P, w.causal, w.layout,
                              w.seed + rank, w.heavy_keys, "cuda")
    q, k, v = synthetic.make_inputs(w_rank, dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.S), dtype=torch.float32, device=dev)
    from sequence_exact_attention_ring_b200 import workspace_bytes
    ws = torch.empty(workspace_bytes(q, k, w.P, w.causal, w.layout), dtype=torch.uint8, device=dev)
    l2buf = None if w.qkvo_bytes() > 126e6 else torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ring_attention(q, k, v, w.P, w.causal, w.layout, w.scale, out=out, lse=lse, workspace=ws, stream=stream,
                       algo=args.algo)

    for _ in range(args.warmup):
        flush_l2(l2buf)
        step()
    torch.cuda.synchronize(dev)
    if status(ws) != 0:
        raise RuntimeError("kernel watchdog tripped during warm-up")

    barrier(world)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev.index)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start.record(stream)
    for i in range(args.steps):
        flush_l2(l2buf)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    barrier(world)
    st = status(ws)
    elapsed_ms = t_start.elapsed_time(t_end)
    launch_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    elapsed_ms = max_over_ranks(elapsed_ms, world)
    launch_ms_max = max_over_ranks(launch_ms, world)

    flops = w.causal_flops()
    value = flops * world * args.steps / (elapsed_ms * 1e-3) / 1e12
    peaks, peak_src = measured_peaks()
    peak = float(peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"])
    achieved = w.algorithmic_flops() / (launch_ms_max * 1e-3) / 1e12

    # ---- end to end: pinned host buffers, H2D + kernel + D2H inside the timed region
    e2e = None
    if not args.no_e2e:
        # Host-resident inputs through the public HostRunner: every step copies its q, k, v
        # in from pinned memory and its out, lse back; two device buffer sets and a copy
        # stream let one step's copies overlap another step's kernel.
        qh, kh, vh = q.cpu().pin_memory(), k.cpu().pin_memory(), v.cpu().pin_memory()
        del out
        runner = HostRunner(q.shape, k.shape, q.dtype, w.P, w.causal, w.layout, w.scale, device=dev, buffers=2)
        copy_stream = torch.cuda.Stream(dev)
        runner.run_steps([(qh, kh, vh)], copy_stream, stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e_steps = max(2, min(args.steps, 4))
        e0.record(copy_stream)
        runner.run_steps([(qh, kh, vh)] * e_steps, copy_stream, stream)
        e1.record(copy_stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        e2e = {"value": flops * world * e_steps / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": runner.h2d_bytes() * world, "d2h_bytes_per_step": runner.d2h_bytes() * world,
               "steps": e_steps, "pipelined": "2 device buffer sets, copies on their own stream"}

    clocks_all = gather_objects(clocks, world)
    statuses = gather_objects(st, world)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n, secs, fl, cores, h = oracle_sample_rate(w, q, k, v, args.cpu_seconds)
        cpu = {"value": rate, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} seeded query rows of head {h} ({fl / 1e9:.1f} GFLOP causal-adjusted, "
                         f"{secs:.1f} s), fp64, full score rows"}
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "fp32",
        "data": "synthetic", "config": workload_config(w),
        "pct_of_peak": 100.0 * value / world / peak,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": kernel_traffic_per_launch(w.name),
                     "peak_source": f"{peak_src} bf16_tflops_sustained (seconds-long kernel under the power cap)",
                     "kernel": KERNEL_NAME},
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clocks_all[0] if world == 1 else {"per_rank": clocks_all},
        "cpu_baseline": cpu,
        "status": statuses,
    }
    print(json.dumps(line))


BWD_METRIC = "causal-adjusted attention backward TFLOP/s (10*D FLOPs per allowed pair), 1 GPU"


def run_backward(args, world, rank, local):
    """Times ring_attn_bwd (prep + dK/dV + dQ kernels) on the workload; out/lse from one
    untimed forward. Algorithmic work: 5 matrix products per allowed (query, key) pair,
    10*D FLOPs (the kernels recompute S and dP once more, which is not counted)."""
    from sequence_exact_attention_ring_b200 import binding, ring_attention, ring_attention_backward
    w = synthetic.get(args.workload)
    binding.load()
    dev = torch.device("cuda", local if world > 1 else 0)
    w_rank = synthetic.custom(w.name, w.dtype, w.B, w.Hq, w.Hkv, w.S, w.D, w.P, w.causal, w.layout,
                              w.seed + rank, w.heavy_keys, "cuda")
    q, k, v = synthetic.make_inputs(w_rank, dev)
    dout = synthetic.make_dout(w_rank, dev)
    out, lse = ring_attention(q, k, v, w.P, w.causal, w.layout, w.scale)
    wsb = binding.ring_attn_bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.S, w.D, w.P, int(w.causal),
                                                {"contiguous": 0, "striped": 1, "zigzag": 2}[w.layout], 1)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        return ring_attention_backward(q, k, v, out, lse, dout, w.P, w.causal, w.layout, w.scale, workspace=ws,
                                       stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    barrier(world)
    sampler = ClockSampler(dev.index)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    st = binding.ring_attn_status(ws.data_ptr(), stream.cuda_stream)
    elapsed = max_over_ranks(t0.elapsed_time(t1), world)
    launch_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in ev), world)
    flops = 2.5 * w.causal_flops()
    alg = 2.5 * w.algorithmic_flops()
    peaks, peak_src = measured_peaks()
    peak = float(peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"])
    achieved = alg / (launch_ms * 1e-3) / 1e12
    clocks_all = gather_objects(clocks, world)
    if rank != 0:
        return
    print(json.dumps({
        "metric": BWD_METRIC, "value": flops * world * args.steps / (elapsed * 1e-3) / 1e12, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(w), **{"pass": "bwd", "flops_per_step": flops}),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None,
                     "peak_source": f"{peak_src} bf16_tflops_sustained",
                     "kernel": "bwd_prep_kernel + bwd_dkdv_kernel + bwd_dq_kernel (one ring_attn_bwd call)"},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks_all[0] if world == 1 else {"per_rank": clocks_all},
        "status": st,
    }))


DECODE_METRIC = "decode step against a sharded KV cache: cache GB/s read, 1 GPU"


def run_decode(args, world, rank, local):
    """Times ring_attn_decode (split-KV kernel + merge) with the workload's K/V as the cache.
    Algorithmic bytes per step: K and V read once, q read, out and lse written."""
    from sequence_exact_attention_ring_b200 import binding, ring_attention_decode
    w = synthetic.get(args.workload)
    binding.load()
    dev = torch.device("cuda", local if world > 1 else 0)
    w_rank = synthetic.custom(w.name, w.dtype, w.B, w.Hq, w.Hkv, w.S, w.D, w.P, False, w.layout, w.seed + rank,
                              w.heavy_keys, "cuda")
    _, k, v = synthetic.make_inputs(w_rank, dev)
    q1 = synthetic.make_decode_query(w_rank, dev)
    lay = {"contiguous": 0, "striped": 1, "zigzag": 2}[w.layout]
    ws = torch.zeros(binding.ring_attn_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.S, w.D, w.P, lay, 1),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    esz = 2
    nbytes = 2 * w.B * w.Hkv * w.S * w.D * esz + 2 * w.B * w.Hq * w.D * esz + w.B * w.Hq * 4

    def step():
        return ring_attention_decode(q1, k, v, w.P, w.layout, w.scale, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    barrier(world)
    sampler = ClockSampler(dev.index)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    st = binding.ring_attn_status(ws.data_ptr(), stream.cuda_stream)
    ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in ev), world)
    peaks, peak_src = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    achieved = nbytes / (ms * 1e-3) / 1e9
    clocks_all = gather_objects(clocks, world)
    if rank != 0:
        return
    print(json.dumps({
        "metric": DECODE_METRIC, "value": achieved * world, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": dict({k_: v_ for k_, v_ in workload_config(w).items() if k_ != "flops_per_step"},
                       **{"pass": "decode", "causal": False, "cache_bytes": nbytes,
                          "l2": "cache larger than L2 (no flush)"}),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "peak_source": f"{peak_src} hbm_gbs",
                     "kernel": "decode_kernel + merge_kernel (one ring_attn_decode call)"},
        "gpu_launches": 2 * args.steps,
        "clocks": clocks_all[0] if world == 1 else {"per_rank": clocks_all},
        "status": st,
    }))


MERGE_METRIC = "merge of per-step partials (ring_attn_merge): HBM GB/s, 1 GPU"


def run_merge(args, world, rank, local):
    """Times ring_attn_merge on the workload's per-step partials: P parts of fp32 O rows
    (B*Hq*Sq rows of one query shard's worth, D wide) and their lse, merged to bf16 O and
    fp32 lse. Algorithmic bytes: every part read once, the result written once."""
    from sequence_exact_attention_ring_b200 import binding, merge
    w = synthetic.get(args.workload)
    binding.load()
    dev = torch.device("cuda", local if world > 1 else 0)
    rows = w.B * w.Hq * w.Sq
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed + 900 + rank)
    o_parts = torch.randn((w.P, rows, w.D), generator=gen, device=dev, dtype=torch.float32)
    l_parts = torch.randn((w.P, rows), generator=gen, device=dev, dtype=torch.float32) * 4
    nbytes = w.P * rows * (w.D + 1) * 4 + rows * (w.D * 2 + 4)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        merge(o_parts, l_parts, torch.bfloat16, stream=stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    sampler = ClockSampler(dev.index)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        ev[i][0].record(stream)
        merge(o_parts, l_parts, torch.bfloat16, stream=stream)
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in ev), world)
    peaks, peak_src = measured_peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    clocks_all = gather_objects(clocks, world)
    if rank != 0:
        return
    print(json.dumps({
        "metric": MERGE_METRIC, "value": achieved * world, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "parts": w.P, "rows": rows, "D": w.D, "bytes": nbytes,
                   "l2": "parts larger than L2 (no flush)" if nbytes > 126e6 else "parts fit in L2"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                     "frac": achieved / float(peaks["hbm_gbs"]), "traffic": None,
                     "peak_source": f"{peak_src} hbm_gbs", "kernel": "merge_kernel"},
        "gpu_launches": args.steps,
        "clocks": clocks_all[0] if world == 1 else {"per_rank": clocks_all},
    }))


RING_METRIC = "ring spread over ranks (forward): causal-adjusted attention TFLOP/s"


def run_ring(args, world, rank, local):
    """The forward ring with the sequence spread over ranks (RingAttention deep-architecture
    article, sections 2, 4, 5): every rank keeps one query shard, the KV shards travel the
    ring, each step is one ring_attn_fwd_ring_step launch whose epilogue folds the block
    into the rank's running state.
      one GPU: --ring-ranks virtual ranks, each with its own buffers and streams; the KV
               shards move by device-to-device copies on copy streams while steps run;
      N GPUs (torchrun): one rank per GPU, KV shards over NCCL point-to-point into the
               GPU's own buffers.
    The whole job is one sequence (strong scaling). Also reports the per-step copy and
    compute durations (the zero-bubble condition of section 4) and, on one GPU, the
    single-launch ring_attn_fwd time of the same workload."""
    from sequence_exact_attention_ring_b200 import binding, ring, ring_attention
    w = synthetic.get(args.workload)
    binding.load()
    dev = torch.device("cuda", local if world > 1 else 0)
    R = world if world > 1 else args.ring_ranks
    if w.S % R or (w.layout == "zigzag" and w.S % (2 * R)):
        raise SystemExit(f"S={w.S} does not split into {R} ring shards")
    q, k, v = synthetic.make_inputs(w, dev)
    stream = torch.cuda.current_stream(dev)
    fused_ms = None
    if world == 1:
        # the single-launch forward of the same workload, for comparison
        out = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, w.S), dtype=torch.float32, device=dev)
        ring_attention(q, k, v, w.P, w.causal, w.layout, w.scale, out=out, lse=lse, stream=stream)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(2):
            ring_attention(q, k, v, w.P, w.causal, w.layout, w.scale, out=out, lse=lse, stream=stream)
        f1.record(stream)
        torch.cuda.synchronize(dev)
        fused_ms = f0.elapsed_time(f1) / 2
        del out, lse
    qs, ks, vs = (ring.split_shards(t, R, w.layout) for t in (q, k, v))
    del q, k, v
    if world > 1:
        qs, ks, vs = [qs[rank]], [ks[rank]], [vs[rank]]
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    if world == 1:
        vr = ring.VirtualRing(qs, ks, vs, w.causal, w.layout, w.scale)

        def step(timing=False):
            return vr.run(timing=timing)
    else:
        comm = torch.cuda.Stream(dev)

        def step(timing=False):
            ring.ring_attention_distributed(qs[0], ks[0], vs[0], w.causal, w.layout, w.scale, stream=stream,
                                            comm_stream=comm)
            return None

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    barrier(world)
    sampler = ClockSampler(dev.index)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    barrier(world)
    elapsed = max_over_ranks(t0.elapsed_time(t1), world)
    overlap = None
    if world == 1:
        # one more, instrumented pass: per rank and step, the copy and the compute durations
        tm = step(timing=True)
        torch.cuda.synchronize(dev)
        comp = [[a.elapsed_time(b) for a, b in per] for per in tm["compute"]]
        cop = [[a.elapsed_time(b) for a, b in per] for per in tm["copy"]]
        overlap = {"virtual_ranks": R, "step_ms_wall": elapsed / args.steps,
                   "fused_single_launch_ms": fused_ms,
                   "compute_ms_per_rank_max": max(sum(c) for c in comp),
                   "copy_ms_per_rank_max": max(sum(c) for c in cop) if R > 1 else 0.0,
                   "copy_ms_per_step_max": max(max(c) for c in cop) if R > 1 else 0.0,
                   "kv_bytes_per_step_per_rank": 2 * ks[0].numel() * ks[0].element_size()}
    flops = w.causal_flops()
    value = flops * args.steps / (elapsed * 1e-3) / 1e12
    peaks, peak_src = measured_peaks()
    peak = float(peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"])
    skipped = 0
    if w.causal and w.layout == "contiguous":
        skipped = R * (R - 1) // 2  # fully masked blocks: no launch unless first or last
    launches_per_step = R * R - skipped + (R - 1 if skipped else 0)
    clocks_all = gather_objects(clocks, world)
    if rank != 0:
        return
    print(json.dumps({
        "metric": RING_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed / args.steps, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": dict(workload_config(w), **{"pass": "ring", "ring_ranks": R,
                                              "transport": "device-to-device copies between virtual ranks"
                                              if world == 1 else "NCCL point-to-point between GPUs"}),
        "roofline": {"bound": "tensor", "achieved": value / world, "peak": peak, "unit": "TFLOP/s",
                     "frac": value / world / peak, "traffic": None,
                     "peak_source": f"{peak_src} bf16_tflops_sustained",
                     "kernel": "ring_fwd_sm100_2sm_kernel (one launch per ring step, fold epilogue)"},
        "overlap": overlap,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks_all[0] if world == 1 else {"per_rank": clocks_all},
    }))


RING_BWD_METRIC = "ring spread over ranks (backward): attention backward TFLOP/s (10*D FLOPs per allowed pair)"


def run_ring_backward(args, world, rank, local):
    """The backward ring with the sequence spread over ranks (RingAttention deep-architecture
    article, section "activation checkpointing and memory recomputation"): every rank keeps
    its query shard, dO and row statistics; the KV shards travel the other way carrying
    their dK/dV accumulators; each step is the dK/dV part then the dQ part of
    ring_attn_bwd_ring_step.
      one GPU: --ring-ranks virtual ranks (device-to-device copies between their buffers);
      N GPUs (torchrun): one rank per GPU, NCCL point-to-point.
    out and lse come from one untimed single-launch forward. Strong scaling: one sequence.
    Also reports the per-step copy and compute durations and, on one GPU, the single-launch
    ring_attn_bwd time of the same workload."""
    from sequence_exact_attention_ring_b200 import binding, ring, ring_attention, ring_attention_backward
    w = synthetic.get(args.workload)
    binding.load()
    dev = torch.device("cuda", local if world > 1 else 0)
    R = world if world > 1 else args.ring_ranks
    if w.S % R or (w.layout == "zigzag" and w.S % (2 * R)):
        raise SystemExit(f"S={w.S} does not split into {R} ring shards")
    q, k, v = synthetic.make_inputs(w, dev)
    dout = synthetic.make_dout(w, dev)
    stream = torch.cuda.current_stream(dev)
    out, lse = ring_attention(q, k, v, w.P, w.causal, w.layout, w.scale, stream=stream)
    fused_ms = None
    if world == 1:
        ring_attention_backward(q, k, v, out, lse, dout, w.P, w.causal, w.layout, w.scale, stream=stream)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        ring_attention_backward(q, k, v, out, lse, dout, w.P, w.causal, w.layout, w.scale, stream=stream)
        f1.record(stream)
        torch.cuda.synchronize(dev)
        fused_ms = f0.elapsed_time(f1)
    shards = [ring.split_shards(t, R, w.layout) for t in (q, k, v, out, dout)]
    lses = [x.squeeze(-1).contiguous() for x in ring.split_shards(lse.unsqueeze(-1), R, w.layout)]
    del q, k, v, out, dout, lse
    qs, ks, vs, outs, douts = shards
    if world > 1:
        qs, ks, vs, outs, douts, lses = ([x[rank]] for x in (qs, ks, vs, outs, douts, lses))
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    if world == 1:
        vr = ring.VirtualBackwardRing(qs, ks, vs, outs, lses, douts, w.causal, w.layout, w.scale)

        def step(timing=False):
            return vr.run(timing=timing)
    else:
        comm = torch.cuda.Stream(dev)

        def step(timing=False):
            ring.ring_attention_backward_distributed(qs[0], ks[0], vs[0], outs[0], lses[0], douts[0], w.causal,
                                                     w.layout, w.scale, stream=stream, comm_stream=comm)
            return None

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    barrier(world)
    sampler = ClockSampler(dev.index)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    barrier(world)
    elapsed = max_over_ranks(t0.elapsed_time(t1), world)
    overlap = None
    if world == 1:
        tm = step(timing=True)
        torch.cuda.synchronize(dev)
        comp = [[a.elapsed_time(b) for a, b in per] for per in tm["compute"]]
        cop = [[a.elapsed_time(b) for a, b in per] for per in tm["copy"]]
        overlap = {"virtual_ranks": R, "step_ms_wall": elapsed / args.steps,
                   "fused_single_launch_ms": fused_ms,
                   "compute_ms_per_rank_max": max(sum(c) for c in comp),
                   "copy_ms_per_rank_max": max(sum(c) for c in cop) if R > 1 else 0.0,
                   "copy_ms_per_step_max": max(max(c) for c in cop) if R > 1 else 0.0,
                   "bytes_per_step_per_rank": (2 * ks[0].numel() * ks[0].element_size()
                                               + 2 * ks[0].numel() * 4) if R > 1 else 0}
    flops = 2.5 * w.causal_flops()
    value = flops * args.steps / (elapsed * 1e-3) / 1e12
    peaks, peak_src = measured_peaks()
    peak = float(peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"])
    clocks_all = gather_objects(clocks, world)
    if rank != 0:
        return
    print(json.dumps({
        "metric": RING_BWD_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed / args.steps, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": dict(workload_config(w), **{"pass": "ring-bwd", "ring_ranks": R,
                                              "transport": "device-to-device copies between virtual ranks"
                                              if world == 1 else "NCCL point-to-point between GPUs"}),
        "roofline": {"bound": "tensor", "achieved": value / world, "peak": peak, "unit": "TFLOP/s",
                     "frac": value / world / peak, "traffic": None,
                     "peak_source": f"{peak_src} bf16_tflops_sustained",
                     "kernel": "bwd_prep_kernel, then per ring step bwd_dkdv_kernel and bwd_dq_kernel"},
        "overlap": overlap,
        "gpu_launches": (R + 2 * R * R) * args.steps,
        "clocks": clocks_all[0] if world == 1 else {"per_rank": clocks_all},
    }))


def dispatch(args, world, rank, local):
    """Runs the arm and pass the arguments select."""
    if args.impl == "reference":
        run_reference(args, world, rank)
    elif args.which == "bwd":
        run_backward(args, world, rank, local)
    elif args.which == "decode":
        run_decode(args, world, rank, local)
    elif args.which == "merge":
        run_merge(args, world, rank, local)
    elif args.which == "ring-bwd":
        run_ring_backward(args, world, rank, local)
    elif args.which == "ring":
        run_ring(args, world, rank, local)
    else:
        run_ours(args, world, rank, local)


def main():
    args = parse()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch_under_torchrun(args))
    world, rank, local = dist_setup(args)
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but {world} ranks were launched")
    try:
        dispatch(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
