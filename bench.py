#!/usr/bin/env python
"""Decode-attention throughput: history tokens/s and achieved HBM GB/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload ragged|exact|hybrid|staged|staged-hybrid|aging|tiny]
                    [--variant auto|simt|mma] [--impl ours|reference] [--no-per-config]

A step is one decode step of the whole hot path over one batch: split attention over
every tier (exact BF16 and, for hybrid workloads, the compact tier) followed by the exact
log-sum-exp merge.  The default workload, the headline, is the ragged paged hybrid batch:
64 sequences with lengths uniform on [1024, 65536], 16-token pages, the newest 1024 tokens
of each exact BF16 and the rest 4-bit codes, 32 query / 8 KV heads, d 128, 512-token
splits (about 2.4 GB of history per step, larger than the 126 MB L2, so no flush is needed
between steps).  The same run measures the other workloads (exact GQA, hybrid, staged 128k
BF16 and staged 128k hybrid) and reports them under ``per_config``; the staged hybrid entry
carries the staging trade (PCIe bytes saved against GPU time added).

Timing: whole steps are timed by CUDA events at the two ends of the timed loop; the
dominant kernel is timed separately, its launches back to back with events only at the
ends, so it keeps the launch overlap it has inside a step.  Staged workloads are
PCIe-bound and are timed by host wall clock with timing-disabled fences.

One process per GPU (torchrun for N > 1): every rank runs an independent replica on its
own batch (the batch partitions with no exchange), so scaling is weak and the reported
value is the tokens of all ranks over the slowest rank's time.  Rank 0 prints one JSON
line.  ``--impl reference`` times the float64 CPU oracle on this host's cores instead.
"""
from __future__ import annotations

import argparse
import gc
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attention history tokens/s/GPU & achieved HBM GB/s vs B200 peak"
UNIT = "history tokens/s"
FALLBACK_HBM_GBS = 6650.0
WORKLOADS = ["ragged", "exact", "hybrid", "tiny", "staged", "staged-hybrid", "aging"]
PER_CONFIG = ("exact", "hybrid", "staged", "staged-hybrid", "aging")
STAGED = ("staged", "staged-hybrid")


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="ragged", choices=WORKLOADS)
    ap.add_argument("--layers", type=int, default=None, help="staged workloads: layers (default 16)")
    ap.add_argument("--variant", default="auto", choices=["auto", "simt", "mma"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--soak-seconds", type=float, default=1.5,
                    help="untimed steady-state run before the timed region (clocks settle, samples taken)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="budget of the oracle's timed sample (per-config entries get a third of it)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="the headline workload only (per-config entries are measured only for the default "
                         "ragged workload)")
    ap.add_argument("--staged-steps", type=int, default=20, help="timed steps of the per-config staged entries")
    ap.add_argument("--fuse", action="store_true",
                    help="time the one-call akv_decode (the library plans the slots and enqueues the attention "
                         "and merge launches) instead of akv_decode_attend and akv_merge_lse calls")
    return ap.parse_args(argv)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


KERNEL_SOURCES = ("kv_cache_tiering_b200/csrc/attend_mma.cu", "kv_cache_tiering_b200/csrc/akv_internal.cuh")


def recorded_traffic(workload: str, kernel: str):
    """DRAM bytes (read + write) per launch of `kernel` on `workload`, as one ncu capture
    recorded them in profiles/dram_traffic.txt; None when nothing is recorded or the
    kernel sources have changed since (their hash no longer matches the record)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    key = h.hexdigest()[:16]
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) == 5 and not line.startswith("#") and parts[:3] == [workload, kernel, key]:
                return int(parts[3]) + int(parts[4])
    return None


# ----------------------------------------------------------------------------------
# clocks sampled during the run
# ----------------------------------------------------------------------------------


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None
        self.marks = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def mark(self, name):
        self.marks.append((name, time.monotonic()))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)

    def summary(self, t0: float, t1: float):
        rows = []
        for t, line in self.lines:
            if t0 <= t <= t1:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[4:8]) if v.lower() == "active"})
        pw = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "power_w_max": max(pw) if pw else None}


# ----------------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------------


def make_workload(name: str, device, rank: int):
    from kv_cache_tiering_b200 import synth, workloads
    base = synth.WORKLOADS[name]
    wl = synth.Workload(base.name, base.B, base.Hq, base.Hkv, base.d, base.split_tokens, seed=base.seed + rank,
                        extra=dict(base.extra))
    if name in ("exact", "tiny"):
        w = workloads.ExactResident(wl, device)
        tokens = w.B * w.T
    elif name == "hybrid":
        w = workloads.HybridResident(wl, device)
        tokens = w.B * w.T
    else:
        w = workloads.RaggedPaged(wl, device, generator="torch")
        tokens = int(w.lens.sum())
    return wl, w, tokens


def tier_bytes(name: str, wl) -> list:
    """Algorithmic bytes each tier's attention launch reads per step (K and V, all KV heads):
    4096 B per exact token and 1056 B per compact token at d 128 (64 B of codes and a 2-byte
    norm per head per tensor).  Host-only: both arms describe the same workload."""
    from kv_cache_tiering_b200 import synth
    H, d = wl.Hkv, wl.d
    exact_tok, compact_tok = 2 * H * d * 2, 2 * H * (d // 2 + 2)
    if name in ("exact", "tiny"):
        return [wl.B * wl.extra["T"] * exact_tok]
    if name == "hybrid":
        T, W = wl.extra["T"], wl.extra["window"]
        return [wl.B * (T - W) * compact_tok, wl.B * W * exact_tok]
    lens = synth.ragged_lengths(wl).astype(int)
    ex = [min(int(L), wl.extra["window"]) for L in lens]
    return [sum(int(L) - e for L, e in zip(lens, ex)) * compact_tok, sum(ex) * exact_tok]


DESCRIPTIONS = {
    "exact": "exact-tier GQA decode: batch 8, 32 q / 8 KV heads, d 128, 8192 BF16 tokens, contiguous, 512-token splits",
    "tiny": "tiny exact decode: batch 1, 1 q / 1 KV head, d 64, 256 BF16 tokens, 4 splits of 64",
    "hybrid": "hybrid tier: batch 4, 32 q / 8 KV heads, d 128, 32768 tokens (newest 2048 BF16, 30720 4-bit codes)",
    "ragged": "ragged paged hybrid: batch 64, lengths U[1024, 65536], 16-token pages through seeded permutations, "
              "newest 1024 BF16, the rest 4-bit codes, Student-t(3) keys, 32 q / 8 KV heads, d 128, 512-token splits",
    "staged-hybrid": "staged 128k hybrid history: batch 1, {L} layers, 32 q / 8 KV heads, d 128, 131072 tokens per "
                     "layer: newest 2048 BF16 on the device, 129024 as 4-bit codes in pinned host memory, 4096-token "
                     "chunks through a 2-buffer device region, one token appended per step",
    "staged": "staged 128k history: batch 1, {L} layers, 32 q / 8 KV heads, d 128, 131072 BF16 tokens per layer in "
              "pinned host memory, 4096-token chunks through a 2-buffer device region, one token appended per step",
}


def config_of(name: str, wl, args, world: int, layers=None) -> dict:
    """The config of a bench line; the same dict for both arms."""
    desc = DESCRIPTIONS[name].format(L=layers or wl.extra.get("layers", 16))
    d = {"workload": desc, "batch": wl.B, "q_heads": wl.Hq, "kv_heads": wl.Hkv, "head_dim": wl.d,
         "split_tokens": wl.split_tokens, "parallelism": f"independent replicas x{world}", "accumulate": "f32",
         "variant": args.variant}
    if name in STAGED:
        d["timing"] = "host wall clock, timing-disabled fences"
        return d
    kv = sum(tier_bytes(name, wl))
    d["kv_bytes_per_step"] = kv
    d["l2"] = ("inputs larger than the 126 MB L2, no flush" if kv > 126e6
               else "L2 flushed (256 MB write) before every step; each step timed by its own events, the flush not "
                    "timed")
    d["step"] = ("one akv_decode call (attention launches + merge launch)" if args.fuse
                 else "attention launches + merge launch")
    return d


# ----------------------------------------------------------------------------------
# reference arm: the float64 CPU oracle
# ----------------------------------------------------------------------------------


def _codes(enc):
    return enc.codes, enc.scale_bits


def oracle_sequence_fn(name, wl, seed_rank=0):
    """Return (fn(i) -> tokens processed, n_units, description) running the oracle on unit i."""
    import numpy as np
    from kv_cache_tiering_b200 import synth
    from oracle import akv_oracle as ora
    f64 = ora.bf16_bits_to_f64
    if name in ("exact", "tiny"):
        T = wl.extra["T"]
        q = synth.queries(wl)

        def fn(i):
            b = i % wl.B
            k, v = synth.history_head_major(wl, b, T)
            ora.decode_sequence(f64(q[b]), [(f64(k), f64(v))], wl.scale, wl.split_tokens)
            return T
        return fn, wl.B, "one sequence (all heads, all splits, merge) per unit"
    if name == "hybrid":
        T, W = wl.extra["T"], wl.extra["window"]
        q = synth.queries(wl)

        def fn(i):
            b = i % wl.B
            k, v = synth.history_head_major(wl, b, T)
            h = i % wl.Hkv
            G = wl.Hq // wl.Hkv
            ek, ev = ora.encode(k[h, :T - W]), ora.encode(v[h, :T - W])
            kh, vh = ora.dequantize(ek.codes, ek.scale_bits)[None], ora.dequantize(ev.codes, ev.scale_bits)[None]
            tiers = [(kh, vh), (f64(k[h:h + 1, T - W:]), f64(v[h:h + 1, T - W:]))]
            ora.decode_sequence(f64(q[b, h * G:(h + 1) * G]), tiers, wl.scale, wl.split_tokens)
            return T / wl.Hkv
        return fn, wl.B * wl.Hkv, "one (sequence, KV head) with its 4 query heads per unit, encode included"
    if name == "staged-hybrid":
        n, W = 16384, wl.extra["window"]  # one layer's decode over a 16384-token sample per unit
        gen = synth.stream(wl.seed, "oracle-sample-hybrid")

        def fn(i):
            k = synth.normal_bf16(gen, (wl.Hkv, n, wl.d))
            v = synth.normal_bf16(gen, (wl.Hkv, n, wl.d))
            q = synth.normal_bf16(gen, (wl.Hq, wl.d))
            kh = np.stack([ora.dequantize(*_codes(ora.encode(k[h, :n - W]))) for h in range(wl.Hkv)])
            vh = np.stack([ora.dequantize(*_codes(ora.encode(v[h, :n - W]))) for h in range(wl.Hkv)])
            ora.decode_sequence(f64(q), [(kh, vh), (f64(k[:, n - W:]), f64(v[:, n - W:]))], wl.scale,
                                wl.split_tokens)
            return n
        return fn, 4, "one layer's decode over a 16384-token sample (14336 compact, encode included) per unit"
    if name == "staged":
        n = 16384  # tokens of one layer per unit (a bounded sample of the 131072-token layer)
        gen = synth.stream(wl.seed, "oracle-sample")

        def fn(i):
            k = synth.normal_bf16(gen, (wl.Hkv, n, wl.d))
            v = synth.normal_bf16(gen, (wl.Hkv, n, wl.d))
            q = synth.normal_bf16(gen, (wl.Hq, wl.d))
            ora.decode_sequence(f64(q), [(f64(k), f64(v))], wl.scale, wl.split_tokens)
            return n
        return fn, 4, "one layer's decode over a 16384-token sample of its history per unit"
    lens = synth.ragged_lengths(wl)
    q = synth.queries(wl)

    def fn(i):
        b = int(np.argsort(lens)[i * (wl.B - 1) // 7]) if i < 8 else i % wl.B
        L = int(lens[b])
        Wn = min(L, wl.extra["window"])
        k, v = synth.history_head_major(wl, b, L, key_dist="student_t")
        h = 0
        ek, ev = ora.encode(k[h, :L - Wn]), ora.encode(v[h, :L - Wn])
        kh, vh = ora.dequantize(ek.codes, ek.scale_bits)[None], ora.dequantize(ev.codes, ev.scale_bits)[None]
        tiers = [(kh, vh), (f64(k[h:h + 1, L - Wn:]), f64(v[h:h + 1, L - Wn:]))]
        ora.decode_sequence(f64(q[b, :4]), tiers, wl.scale, wl.split_tokens)
        return L / wl.Hkv
    return fn, 8, "one KV head of one sequence per unit, 8 sequences spread over the length range"


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        return os.cpu_count() or 1


def time_oracle(name, wl, budget_s: float = 15.0, max_units=None):
    """The oracle on a bounded sample: units of the workload (cycling through them) until
    budget_s seconds or max_units units (default: 8 passes over the workload's units)."""
    fn, n_units, desc = oracle_sequence_fn(name, wl)
    tokens, units = 0.0, 0
    t0 = time.perf_counter()
    while units < (max_units or 8 * n_units):
        tokens += fn(units)
        units += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return tokens / dt, units, desc, dt


def cpu_baseline(name, wl, budget_s: float):
    cv, units, desc, dt = time_oracle(name, wl, budget_s)
    return {"value": cv, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{units} units ({desc}), {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from kv_cache_tiering_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    fn, n_units, desc = oracle_sequence_fn(args.workload, wl)
    for i in range(args.warmup):
        fn(i)
    times, tokens = [], 0.0
    for i in range(args.steps):
        t0 = time.perf_counter()
        tokens += fn(i)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = tokens / total
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(args.workload, wl, args, args.gpus, args.layers),
            "reference": "float64 numpy oracle on the host CPU; each step is one unit: " + desc,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{args.steps} units: {desc}"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------------


def max_over_ranks(x: float, dist, device) -> float:
    """The largest of every rank's x (every rank calls this, in the same order)."""
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class Ctx:
    """One process per GPU: rank, device and (for N > 1) the NCCL group for barriers and the
    max over ranks.  Every rank takes the same collective steps in the same order."""

    def __init__(self, timeout_s: int = 600):
        import datetime
        import torch
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(self.local)
        self.dev = torch.device("cuda", self.local)
        self.dist = None
        if self.world > 1:
            import torch.distributed as dist
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=timeout_s), device_id=self.dev)
            self.dist = dist

    def max(self, x: float) -> float:
        return max_over_ranks(x, self.dist, self.dev) if self.dist else float(x)

    def barrier(self):
        if self.dist:
            self.dist.barrier()

    def close(self):
        if self.dist:
            self.dist.barrier()
            self.dist.destroy_process_group()


def variant_of(name: str):
    from kv_cache_tiering_b200 import akv
    return {"auto": akv.AKV_VARIANT_AUTO, "simt": akv.AKV_VARIANT_SIMT, "mma": akv.AKV_VARIANT_MMA}[name]


def free_device_memory():
    import torch
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def run_resident(name, ctx, args, steps, warmup, cpu_s):
    """One resident workload: whole steps, the attention kernels back to back, and the
    end-to-end leg through akv_decode_host.  Returns the bench line (every rank)."""
    import torch
    from kv_cache_tiering_b200 import akv
    from kv_cache_tiering_b200 import workloads as wlmod

    dev = ctx.dev
    variant = variant_of(args.variant)
    wl, w, tokens = make_workload(name, dev, ctx.rank)
    step = w.step
    stream = torch.cuda.current_stream()
    flush = None
    if w.kv_bytes() <= 126e6:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    fuse = args.fuse and variant != akv.AKV_VARIANT_SIMT
    live = [i for i, t in enumerate(step.tiers) if int(sum(t.lens)) > 0]

    def run_step(q):
        if fuse:
            step.decode(q, variant, stream)
        else:
            step.step(q, variant, stream)

    def one_step():
        if flush is not None:
            flush.fill_(1)
        run_step(w.q)

    # attention launches (one per non-empty tier, B <= 256), plus the merge
    launches_per_step = len(live) + 1
    sampler = ClockSampler(ctx.local)
    sampler.start()
    for _ in range(max(3, warmup)):
        one_step()
    torch.cuda.synchronize()
    t_soak = time.monotonic()
    while time.monotonic() - t_soak < args.soak_seconds:
        for _ in range(20):
            one_step()
        torch.cuda.synchronize()

    # ---- whole steps: events at the two ends of the timed loop only (with an L2 flush
    # between steps, each step is bracketed by its own events after the flush instead)
    ctx.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step_ev = ([(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(steps)] if flush is not None else None)
    start.record(stream)
    for i in range(steps):
        if flush is not None:
            flush.fill_(1)
            step_ev[i][0].record(stream)
        run_step(w.q)
        if flush is not None:
            step_ev[i][1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.monotonic()
    ms = start.elapsed_time(end) if flush is None else sum(a.elapsed_time(b) for a, b in step_ev)
    ms = ctx.max(ms)

    # ---- each tier's attention kernel alone, its launches back to back (events only at the
    # ends, so a launch overlaps the previous one's tail as it does inside a step)
    n_k = max(steps, 20)
    tier_ms = []
    for j in live:
        if flush is None:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n_k):
                step.attend_tier(j, w.q, variant, stream)
            b.record(stream)
            torch.cuda.synchronize()
            t = a.elapsed_time(b) / n_k
        else:
            evs = []
            for _ in range(n_k):
                flush.fill_(1)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                step.attend_tier(j, w.q, variant, stream)
                b.record(stream)
                evs.append((a, b))
            torch.cuda.synchronize()
            t = sum(a.elapsed_time(b) for a, b in evs) / n_k
        tier_ms.append(ctx.max(t))
    t_post = time.monotonic()
    while time.monotonic() - t_post < 0.3:  # samples inside the loaded window
        for _ in range(20):
            one_step()
        torch.cuda.synchronize()
    err = int(step.err.item())

    # ---- end to end through the public API: every step takes its query from pinned host
    # memory and leaves O and LSE in pinned host memory.  Unfused, that is one akv_decode_host
    # call per step on the compute stream (the GPU reads the query and writes the results over
    # PCIe itself, alternating two output buffers).  Fused (akv_decode has no host form), the
    # copies run on streams of their own with two buffers each, events ordering every reuse.
    q_host = torch.from_numpy(w.q_bits.view("int16")).pin_memory()
    pair = [step, wlmod.DecodeStep(step.B, step.Hq, step.Hkv, step.d, step.split_tokens, step.scale, step.tiers, dev)]
    q_dev = [torch.empty_like(w.q) for _ in range(2)]
    o_host = [torch.empty(step.o.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    lse_host = [torch.empty(step.lse.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_used = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    e2e_ev = None

    def e2e_host_step(i):
        j = i % 2
        if flush is not None:
            flush.fill_(1)
            if e2e_ev is not None:
                e2e_ev[i][0].record(stream)
        step.decode_host(q_host, o_host[j], lse_host[j], 0, variant, stream)
        if flush is not None and e2e_ev is not None:
            e2e_ev[i][1].record(stream)

    def e2e_copy_step(i):
        j, st_j = i % 2, pair[i % 2]
        up.wait_event(ev_used[j])
        with torch.cuda.stream(up):
            q_dev[j].copy_(q_host, non_blocking=True)
            ev_in[j].record(up)
        stream.wait_event(ev_in[j])
        stream.wait_event(ev_out[j])
        if flush is not None:
            flush.fill_(1)
        if fuse:
            st_j.decode(q_dev[j], variant, stream)
        else:
            st_j.step(q_dev[j], variant, stream)
        ev_used[j].record(stream)
        down.wait_event(ev_used[j])
        with torch.cuda.stream(down):
            o_host[j].copy_(st_j.o, non_blocking=True)
            lse_host[j].copy_(st_j.lse, non_blocking=True)
            ev_out[j].record(down)

    e2e_step = e2e_copy_step if fuse else e2e_host_step
    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if flush is not None and not fuse:
        e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(steps)]
    ctx.barrier()
    e0.record(stream)
    up.wait_event(e0)
    for i in range(steps):
        e2e_step(i)
    if fuse:
        stream.wait_event(ev_out[(steps - 1) % 2])
        stream.wait_event(ev_out[steps % 2])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) if e2e_ev is None else sum(a.elapsed_time(b) for a, b in e2e_ev)
    e2e_ms = ctx.max(e2e_ms)
    sampler.stop()

    total_tokens = tokens * ctx.world * steps
    value = total_tokens / (ms * 1e-3)
    e2e_value = total_tokens / (e2e_ms * 1e-3)
    peak, peak_kind = peaks()
    tb = w.tier_bytes()
    assert sum(tb) == sum(tier_bytes(name, wl)), "host and device byte counts disagree"
    kernel_names = ["attend_codes_mma" if step.tiers[i].kind == akv.AKV_TIER_CODES4 else "attend_bf16_mma"
                    for i in live]
    if variant == akv.AKV_VARIANT_SIMT:
        kernel_names = [k.replace("_mma", "_simt") for k in kernel_names]
    j = max(range(len(live)), key=lambda k: tier_ms[k])  # the dominant kernel: the longest launch
    dom_ms, dom_bytes, dom_kernel = tier_ms[j], tb[live[j]], kernel_names[j]
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ctx.world, "steps": steps,
            "warmup": warmup, "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(name, wl, args, ctx.world),
            "hbm_gbs": w.kv_bytes() * ctx.world * steps / (ms * 1e-3) / 1e9,
            "hbm_frac_step": w.kv_bytes() * steps / (ms * 1e-3) / 1e9 / peak,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": recorded_traffic(name, dom_kernel),
                         "kernel": dom_kernel, "algorithmic_bytes": dom_bytes, "kernel_ms_avg": dom_ms,
                         "kernel_timing": f"{n_k} launches of the tier's attention back to back, CUDA events at the "
                                          "ends" + ("" if flush is None else ", each launch after an L2 flush"),
                         "peak_source": f"{peak_kind} hbm_gbs (copy bandwidth)",
                         "tiers_ms_avg": dict(zip(kernel_names, tier_ms)),
                         "tiers_bytes": dict(zip(kernel_names, [tb[i] for i in live])),
                         "tiers_frac": {k: tb[i] / (t * 1e-3) / 1e9 / peak
                                        for k, i, t in zip(kernel_names, live, tier_ms)}},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(q_host.numel() * 2),
                    "d2h_bytes_per_step": int(o_host[0].numel() * 4 + lse_host[0].numel() * 4),
                    "transfers": ("copies on their own streams, two buffers each" if fuse else
                                  "akv_decode_host: the GPU reads the pinned query and writes O and LSE "
                                  "into pinned host memory, one stream")},
            "gpu_launches": launches_per_step * steps,
            "clocks": sampler.summary(t_soak, t_wall1 + 0.3), "device_error_word": err}
    if ctx.rank == 0 and ctx.world == 1 and cpu_s > 0:
        line["cpu_baseline"] = cpu_baseline(name, wl, cpu_s)
    return line


def pcie_ceiling(chunk_bytes: int, device, sources, rounds: int = 5, copies: int = 32) -> float:
    """Pinned host-to-device bandwidth (GB/s) with the copies the stager issues: chunk_bytes
    spans of the staged run's own pinned history (`sources`, its per-layer host tensors, so
    the same pages and NUMA placement) into two alternating device buffers, back to back on
    one stream; host wall clock between timing-disabled fences, best of `rounds`."""
    import torch
    spans = []
    for h in sources:
        flat = h.view(torch.uint8).reshape(-1)
        for c in range(flat.numel() // chunk_bytes):
            if len(spans) < copies:
                spans.append(flat[c * chunk_bytes:(c + 1) * chunk_bytes])
    if not spans:
        return 0.0
    dst = [torch.empty(chunk_bytes, dtype=torch.uint8, device=device) for _ in range(2)]
    s = torch.cuda.Stream(device)
    fence = torch.cuda.Event()  # timing disabled: it does not serialise the copies it follows
    best = 0.0
    for r in range(rounds + 1):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        with torch.cuda.stream(s):
            for c, src in enumerate(spans):
                dst[c % 2].copy_(src, non_blocking=True)
            fence.record(s)
        fence.synchronize()
        dt = time.perf_counter() - t0
        if r > 0:  # the first round warms the path
            best = max(best, len(spans) * chunk_bytes / dt / 1e9)
    del dst
    return best


def chunk_attention_ms(st, hybrid: bool, variant, n: int = 20):
    """GPU time of one step's attention launches with the history already in device memory:
    one full chunk's launch timed back to back (events at the ends), times the chunks of a
    step, plus (hybrid) the window's launch.  Returns (ms per step, per-launch detail)."""
    import torch
    from kv_cache_tiering_b200 import akv, synth
    wl, H, d, dev = st.wl, st.wl.Hkv, st.wl.d, st.device
    q = st.inputs(0)[0][0]
    s = torch.cuda.current_stream()

    def timed(tier):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        akv.akv_decode_attend(q, 1, wl.Hq, H, d, wl.scale, [tier], wl.split_tokens, st.o_part, st.lse_part,
                              st.o_part.shape[0], variant, st.err, s)
        a.record(s)
        for _ in range(n):
            akv.akv_decode_attend(q, 1, wl.Hq, H, d, wl.scale, [tier], wl.split_tokens, st.o_part, st.lse_part,
                                  st.o_part.shape[0], variant, st.err, s)
        b.record(s)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    if hybrid:
        rows = st.chunk // 16
        buf = torch.empty(rows * st.crow, dtype=torch.uint8, device=dev)
        buf.copy_(st.host[0][:rows * st.crow])
        base = buf.data_ptr()
        tier = akv.Tier(akv.AKV_TIER_CODES4, base, base + H * st.bb, lens=[st.chunk], slot_base=[0], stride_seq=0,
                        stride_head=1, stride_token=2 * H)
        t_chunk = timed(tier)
        wb = st.win[0].data_ptr()
        wtier = akv.Tier(akv.AKV_TIER_BF16, wb, wb + H * d * 2, lens=[st.W], slot_base=[st.n_cslots], stride_seq=0,
                         stride_head=d, stride_token=2 * H * d)
        t_win = timed(wtier)
        per_step = st.L * (st.Tc / st.chunk * t_chunk + t_win)
        return per_step, {"compact_chunk_ms": t_chunk, "window_ms": t_win}
    g = synth.torch_generator(wl.seed, wl.name, "bench-chunk", device=dev)
    rows = torch.empty((st.chunk, 2, H, d), dtype=torch.int16, device=dev)
    rows[:, 0] = synth.torch_normal_bf16(g, (st.chunk, H, d), dev)
    rows[:, 1] = synth.torch_normal_bf16(g, (st.chunk, H, d), dev)
    base = rows.data_ptr()
    tier = akv.Tier(akv.AKV_TIER_BF16, base, base + H * d * 2, lens=[st.chunk], slot_base=[0], stride_seq=0,
                    stride_head=d, stride_token=2 * H * d)
    t_chunk = timed(tier)
    return st.L * st.T / st.chunk * t_chunk, {"bf16_chunk_ms": t_chunk}


def run_staged(name, ctx, args, steps, warmup, cpu_s):
    """Staged 128k decode: PCIe-bound, timed by host wall clock around an uninstrumented loop
    (timing-enabled events serialise the copies they observe); one replica per rank."""
    import torch
    from kv_cache_tiering_b200 import synth, workloads

    dev = ctx.dev
    hybrid = name == "staged-hybrid"
    base = synth.WORKLOADS[name]
    wl = synth.Workload(base.name, base.B, base.Hq, base.Hkv, base.d, base.split_tokens, seed=base.seed + ctx.rank,
                        extra=dict(base.extra))
    layers = args.layers or wl.extra["layers"]
    n_warm = max(3, warmup)
    n_steps = n_warm + steps
    variant = variant_of(args.variant)
    if hybrid:
        st = workloads.StagedHybridDecode(wl, dev, layers=layers, T=wl.extra["T"], W=wl.extra["window"],
                                          chunk=wl.extra["chunk"], max_steps=n_steps + 1)
        chunk_bytes = (st.chunk // 16) * st.crow
    else:
        st = workloads.StagedDecode(wl, dev, layers=layers, max_steps=n_steps + 1, source="torch")
        chunk_bytes = st.chunk * st.row_bytes
    o_host = torch.empty(st.o.shape, dtype=torch.float32).pin_memory()
    lse_host = torch.empty(st.lse.shape, dtype=torch.float32).pin_memory()
    inputs = [st.inputs(i) for i in range(n_steps)]

    def one_step(i):
        st.step(*inputs[i], variant)
        with torch.cuda.stream(st.compute_stream):  # the step's result, read back every step
            o_host.copy_(st.o, non_blocking=True)
            lse_host.copy_(st.lse, non_blocking=True)

    pcie_peak = pcie_ceiling(chunk_bytes, dev, st.host)
    sampler = ClockSampler(ctx.local)
    sampler.start()
    for i in range(n_warm):
        one_step(i)
    torch.cuda.synchronize()
    ctx.barrier()
    h2d0 = st.h2d_bytes
    tw0 = time.monotonic()
    t0 = time.perf_counter()
    for i in range(n_warm, n_steps):
        one_step(i)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    tw1 = time.monotonic()
    dt = ctx.max(dt)
    sampler.stop()
    h2d = st.h2d_bytes - h2d0
    n_tok = sum(layers * (wl.extra["T"] + i + 1) for i in range(n_warm, n_steps))
    value = n_tok * ctx.world / dt
    attn_ms, attn_detail = chunk_attention_ms(st, hybrid, variant)
    err = int(st.err.item())
    st.close()
    pcie = h2d / dt / 1e9
    launches = layers * ((-(-st.Tc // st.chunk) + 2) if hybrid else (-(-(wl.extra["T"] + 1) // st.chunk) + 1))
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ctx.world, "steps": steps,
            "warmup": warmup, "ms_per_step": 1e3 * dt / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(name, wl, args, ctx.world, layers),
            "roofline": {"bound": "pcie", "achieved": pcie, "peak": pcie_peak, "unit": "GB/s",
                         "frac": pcie / pcie_peak, "traffic": None,
                         "peak_source": f"pinned host-to-device copies of {chunk_bytes} B (one staged chunk) back to "
                                        "back, host wall clock with timing-disabled fences, best of 5 rounds of 32"},
            "pcie_h2d_gbs": pcie, "h2d_bytes_per_step": h2d // steps,
            "attention_gpu_ms_per_step": attn_ms, "attention_gpu_detail": attn_detail,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": h2d // steps,
                    "d2h_bytes_per_step": (0 if hybrid else layers * st.row_bytes)
                    + 4 * (o_host.numel() + lse_host.numel())},
            "gpu_launches": steps * launches,
            "clocks": sampler.summary(tw0, tw1), "device_error_word": err}
    if ctx.rank == 0 and ctx.world == 1 and cpu_s > 0:
        line["cpu_baseline"] = cpu_baseline(name, wl, cpu_s)
    return line


def staging_trade(bf16: dict, hyb: dict) -> dict:
    """The hybrid tier judged by the bytes it keeps off PCIe against the GPU time it adds,
    from the two staged entries of one run."""
    saved = bf16["h2d_bytes_per_step"] - hyb["h2d_bytes_per_step"]
    return {"pcie_bytes_per_step_bf16": bf16["h2d_bytes_per_step"],
            "pcie_bytes_per_step_hybrid": hyb["h2d_bytes_per_step"],
            "pcie_bytes_saved_per_step": saved,
            "pcie_bytes_ratio": bf16["h2d_bytes_per_step"] / max(1, hyb["h2d_bytes_per_step"]),
            "pcie_ms_saved_per_step": saved / (bf16["roofline"]["peak"] * 1e9) * 1e3,
            "attention_gpu_ms_per_step_bf16": bf16["attention_gpu_ms_per_step"],
            "attention_gpu_ms_per_step_hybrid": hyb["attention_gpu_ms_per_step"],
            "gpu_ms_added_per_step": hyb["attention_gpu_ms_per_step"] - bf16["attention_gpu_ms_per_step"],
            "step_ms_bf16": bf16["ms_per_step"], "step_ms_hybrid": hyb["ms_per_step"],
            "step_speedup": bf16["ms_per_step"] / hyb["ms_per_step"]}


def run_aging(name, ctx, args, steps, warmup, cpu_s):
    """Live hybrid decode with window aging on the hybrid shape: every step appends a token
    per sequence; every 16 steps each window hands its oldest page to the compact tier.
    Timed with CUDA events on the step's stream, whole steps and the parts."""
    import torch
    from kv_cache_tiering_b200 import synth, workloads

    dev = ctx.dev
    base = synth.WORKLOADS["hybrid"]
    wl = synth.Workload("aging", base.B, base.Hq, base.Hkv, base.d, base.split_tokens, seed=base.seed + ctx.rank,
                        extra=dict(base.extra))
    T, W = wl.extra["T"], wl.extra["window"]
    n_warm = max(3, warmup)
    n_steps = n_warm + steps
    sampler = ClockSampler(ctx.local)  # started early: its first sample takes a moment
    sampler.start()
    st = workloads.AgingHybrid(wl, dev, [T] * wl.B, W, max_steps=n_steps + 1, source="torch")
    variant = variant_of(args.variant)
    inputs = [st.inputs(i) for i in range(n_steps)]
    stream = torch.cuda.current_stream()
    for i in range(n_warm):
        st.step(*inputs[i], variant, stream)
    torch.cuda.synchronize()
    aged0 = st.aged_blocks
    tok0 = int(st.c.sum() + st.win.sum())  # history tokens before the first timed step
    ctx.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tw0 = time.monotonic()
    e0.record(stream)
    for i in range(n_warm, n_steps):
        st.step(*inputs[i], variant, stream, sync_state=False)
    e1.record(stream)
    torch.cuda.synchronize()
    tw1 = time.monotonic()
    sampler.stop()
    ms = ctx.max(e0.elapsed_time(e1))
    # bytes one step's attention reads at the start of the timed steps: per KV head, K and V,
    # a compact token is d/2 code bytes + a 2-byte norm, a window token 2d bytes
    step_bytes = int(st.c.sum()) * wl.Hkv * 2 * (wl.d // 2 + 2) + int(st.win.sum()) * wl.Hkv * 2 * wl.d * 2
    st._state()
    aged = st.aged_blocks - aged0
    # step j attends every earlier token plus the B it appends
    tok = sum(tok0 + wl.B * (j + 1) for j in range(steps))
    value = tok * ctx.world / (ms * 1e-3)
    err = int(st.err.item())
    peak, peak_kind = peaks()
    achieved = step_bytes / (ms / steps * 1e-3) / 1e9
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ctx.world, "steps": steps,
            "warmup": warmup, "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "window aging on the hybrid shape: batch 4, 32 q / 8 KV heads, d 128, "
                                   "32768 tokens, newest 2048-2063 BF16 in 16-token ring pages, the rest 4-bit "
                                   "code pages; one token appended per step, full window pages encoded into "
                                   "the compact tier", "parallelism": f"independent replicas x{ctx.world}",
                       "variant": args.variant, "timing": "CUDA events around whole steps",
                       "step": "one akv_aging_step call (append, aging encode, attention launches, merge)"},
            "aged_pages_in_timed_steps": int(aged),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": None, "kernel": "whole step (append, aging, both tiers, merge)",
                         "algorithmic_bytes": step_bytes, "peak_source": f"{peak_kind} hbm_gbs (copy bandwidth)"},
            "e2e": None, "gpu_launches": steps * 4 + 2 * int(aged > 0) * (aged // wl.B),
            # the timed steps take milliseconds: the samples within 0.25 s of them
            "clocks": sampler.summary(tw0 - 0.25, tw1 + 0.25), "device_error_word": err}
    if ctx.rank == 0 and ctx.world == 1 and cpu_s > 0:
        # the oracle of the hybrid shape: the aging step attends the same two tiers (its encode of
        # one page per 16 steps is a small part of the work)
        line["cpu_baseline"] = cpu_baseline("hybrid", base, cpu_s)
    return line


def run_workload(name, ctx, args, steps, warmup, cpu_s):
    if name in STAGED:
        return run_staged(name, ctx, args, steps, warmup, cpu_s)
    if name == "aging":
        return run_aging(name, ctx, args, steps, warmup, cpu_s)
    return run_resident(name, ctx, args, steps, warmup, cpu_s)


def main(argv=None):
    args = parse(argv)
    if args.impl == "reference":
        return run_reference(args)
    ctx = Ctx()
    cpu_s = 0.0 if args.no_cpu_baseline else args.cpu_seconds
    try:
        line = run_workload(args.workload, ctx, args, args.steps, args.warmup, cpu_s)
        # the other workloads ride along on one GPU; a multi-GPU run times the headline only
        # (every rank would otherwise pin its own 10 GB of staged history)
        if args.workload == "ragged" and not args.no_per_config and ctx.world == 1:
            per = {}
            for name in PER_CONFIG:
                free_device_memory()
                steps = min(args.steps, args.staged_steps) if name in STAGED else args.steps
                per[name] = run_workload(name, ctx, args, steps, args.warmup, cpu_s / 3)
            per["staged-hybrid"]["staging_trade"] = staging_trade(per["staged"], per["staged-hybrid"])
            line["per_config"] = per
        if ctx.rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        ctx.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
