"""bench.py host logic on CPU: world-size-2 gloo ranks (max over ranks, gathers),
the reference arm's JSON line, and the clock-sample parser."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.max_over_ranks(1.5 + rank, world)
        objs = bench.gather_objects({"rank": rank}, world)
        bench.barrier(world)
        q.put((rank, m, objs))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_gather_with_two_gloo_ranks():
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
    for rank, m, objs in res:
        assert m == 2.5
        assert objs == [{"rank": 0}, {"rank": 1}]


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "c1_fp32_s1k", "--steps", "2", "--warmup", "1", "--cpu-seconds", "0.5"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["config"]["workload"] == "c1_fp32_s1k"


def test_reference_arm_nonzero_rank_is_silent(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class A:
        workload, steps, warmup, cpu_seconds = "c1_fp32_s1k", 1, 0, 0.2
    bench.run_reference(A, 2, 1)
    assert capsys.readouterr().out == ""


def test_clock_sampler_parses_reasons():
    sys.path.insert(0, ROOT)
    import bench
    s = bench.ClockSampler.__new__(bench.ClockSampler)

    class FakeProc:
        def terminate(self):
            pass

        def communicate(self, timeout=None):
            return ("1800, 1965, 900.1, Not Active, Not Active, Not Active, Active\n"
                    "1750, 1965, 950.3, Not Active, Not Active, Not Active, Not Active\n"
                    "1900, 1965, 700.0, Not Active, Not Active, Not Active, Not Active\n", "")
    s.proc = FakeProc()
    d = s.stop()
    assert d["sm_mhz"] == 1800 and d["sm_max_mhz"] == 1965 and d["reasons"] == ["sw_power_cap"]


def test_traffic_figure_only_for_the_measured_kernel_source(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed ncu figure only while the kernel sources
    hash to the value recorded with it; any source change makes it null."""
    sys.path.insert(0, ROOT)
    import bench
    f = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    f.write_text(json.dumps({"kernel_source_sha256": bench.kernel_source_sha256(),
                             "bytes_per_launch": {"c5_bf16_s1m_striped": 123.0}}))
    assert bench.kernel_traffic_per_launch("c5_bf16_s1m_striped") == 123.0
    assert bench.kernel_traffic_per_launch("c4_bf16_gqa_s128k") is None
    f.write_text(json.dumps({"kernel_source_sha256": "0" * 64, "bytes_per_launch": {"c5_bf16_s1m_striped": 123.0}}))
    assert bench.kernel_traffic_per_launch("c5_bf16_s1m_striped") is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.json"))
    assert bench.kernel_traffic_per_launch("c5_bf16_s1m_striped") is None



def test_gpus_flag_starts_that_many_ranks():
    """`bench.py --gpus 2` outside torchrun launches two ranks itself (gloo here); rank 0
    prints one line that reports both."""
    env = dict(os.environ)
    for key in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(key, None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                        "--workload", "c1_fp32_s1k", "--steps", "1", "--warmup", "1", "--cpu-seconds", "0.3"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["impl"] == "reference"


def test_rank_count_must_match_the_gpus_flag():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                        "--workload", "c1_fp32_s1k", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert r.returncode != 0 and "2 but 1 ranks" in (r.stderr + r.stdout)


def test_every_pass_is_accepted_and_dispatched(monkeypatch):
    """Each --pass value parses and reaches its own runner (the runners themselves need a GPU)."""
    sys.path.insert(0, ROOT)
    import bench
    called = []
    for name in ("run_ours", "run_backward", "run_decode", "run_merge", "run_ring", "run_ring_backward"):
        monkeypatch.setattr(bench, name, lambda *a, _n=name, **k: called.append(_n))
    for which, runner in (("fwd", "run_ours"), ("bwd", "run_backward"), ("decode", "run_decode"),
                          ("merge", "run_merge"), ("ring", "run_ring"), ("ring-bwd", "run_ring_backward")):
        monkeypatch.setattr(sys, "argv", ["bench.py", "--pass", which, "--ring-ranks", "4"])
        args = bench.parse()
        assert args.which == which and args.ring_ranks == 4
        called.clear()
        bench.dispatch(args, 1, 0, 0)
        assert called == [runner]
