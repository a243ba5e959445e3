"""Host logic of bench.py, on the CPU: the max-over-ranks timing across two gloo ranks,
per-rank replica inputs, the recorded-traffic lookup, and the oracle arm's JSON line."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import torch
        ms = [0.5, 2.25][rank]
        e2e = [7.0, 3.0][rank]
        out = (bench.max_over_ranks(ms, dist, torch.device("cpu")),
               bench.max_over_ranks(e2e, dist, torch.device("cpu")))
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_max_over_ranks_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank reports the slowest rank's time, for each timed region separately
    assert res[0] == res[1] == (2.25, 7.0)


def test_replicas_draw_distinct_inputs_per_rank():
    import torch
    cpu = torch.device("cpu")
    _, w0, n0 = bench.make_workload("tiny", cpu, 0)
    _, w1, n1 = bench.make_workload("tiny", cpu, 1)
    _, w0b, _ = bench.make_workload("tiny", cpu, 0)
    assert n0 == n1 == 256  # weak scaling: the same work on every rank
    assert not np.array_equal(w0.k_bits, w1.k_bits) and not np.array_equal(w0.q_bits, w1.q_bits)
    assert np.array_equal(w0.k_bits, w0b.k_bits)  # and reproducible per rank


def test_recorded_traffic_follows_the_kernel_sources(monkeypatch, tmp_path):
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    assert rows, "no traffic recorded"
    t = bench.recorded_traffic(rows[0][0], rows[0][1])
    if t is not None:  # sources unchanged since the capture: read + write bytes
        assert t == int(rows[0][3]) + int(rows[0][4])
    assert bench.recorded_traffic(rows[0][0], "no_such_kernel") is None
    # any change to the kernel sources invalidates every record
    changed = tmp_path / "attend_mma.cu"
    changed.write_text(open(os.path.join(ROOT, bench.KERNEL_SOURCES[0])).read() + "\n// edited\n")
    monkeypatch.setattr(bench, "KERNEL_SOURCES", (str(changed),) + tuple(bench.KERNEL_SOURCES[1:]))
    assert bench.recorded_traffic(rows[0][0], rows[0][1]) is None


def _run_bench(args, env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=300)


def test_reference_arm_line_and_nonzero_ranks_exit_quietly():
    r = _run_bench(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1"], {})
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "config", "cpu_baseline", "e2e"):
        assert key in line
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0
    r1 = _run_bench(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1"],
                    {"RANK": "1", "WORLD_SIZE": "2"})
    assert r1.returncode == 0 and r1.stdout.strip() == ""


def test_staging_trade_arithmetic():
    """The staged-hybrid line's trade: PCIe bytes kept off the link against GPU time added,
    from the two staged entries of one run."""
    bf16 = {"h2d_bytes_per_step": 8_000_000_000, "roofline": {"peak": 50.0}, "attention_gpu_ms_per_step": 7.5,
            "ms_per_step": 160.0}
    hyb = {"h2d_bytes_per_step": 2_000_000_000, "roofline": {"peak": 48.0}, "attention_gpu_ms_per_step": 11.0,
           "ms_per_step": 40.0}
    t = bench.staging_trade(bf16, hyb)
    assert t["pcie_bytes_saved_per_step"] == 6_000_000_000
    assert t["pcie_bytes_ratio"] == 4.0
    assert t["pcie_ms_saved_per_step"] == pytest.approx(120.0)  # 6 GB at the BF16 run's 50 GB/s ceiling
    assert t["gpu_ms_added_per_step"] == pytest.approx(3.5)
    assert t["step_speedup"] == pytest.approx(4.0)
