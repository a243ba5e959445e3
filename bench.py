#!/usr/bin/env python
"""Decode-attention throughput: history tokens/s and achieved HBM GB/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload exact|hybrid|ragged|tiny]
                    [--variant auto|simt|mma] [--impl ours|reference]

A step is one decode step of the whole hot path over one batch: split attention over
every tier (exact BF16 and, for hybrid workloads, the compact tier) followed by the exact
log-sum-exp merge.  The default workload is the exact-tier GQA decode: batch 8, 32 query
/ 8 KV heads, d 128, 8192 BF16 tokens per sequence, 512-token splits (268 MB of K/V per
step, larger than the 126 MB L2, so no flush is needed between steps).

One process per GPU (torchrun for N > 1): every rank runs an independent replica on its
own batch (the batch partitions with no exchange), so scaling is weak and the reported
value is the tokens of all ranks over the slowest rank's time.  Rank 0 prints one JSON
line.  ``--impl reference`` times the float64 CPU oracle on this host's cores instead.
"""
from __future__ import annotations

import argparse
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


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="exact", choices=["exact", "hybrid", "ragged", "tiny", "staged", "staged-hybrid", "aging"])
    ap.add_argument("--layers", type=int, default=None, help="staged workload: layers (default 16)")
    ap.add_argument("--variant", default="auto", choices=["auto", "simt", "mma"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--soak-seconds", type=float, default=1.5,
                    help="untimed steady-state run before the timed region (clocks settle, samples taken)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fuse", action="store_true",
                    help="time the one-call akv_decode (the library plans the slots and enqueues the attention "
                         "and merge launches) instead of akv_decode_attend and akv_merge_lse calls")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


SAMPLE = 8  # timed steps between two steps whose launches are bracketed by events

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


def describe(name, wl, w=None):
    """The config of a bench line; w (the device workload) adds its bytes per step."""
    d = {"workload": {
        "exact": "exact-tier GQA decode: batch 8, 32 q / 8 KV heads, d 128, 8192 BF16 tokens, contiguous, 512-token splits",
        "tiny": "tiny exact decode: batch 1, 1 q / 1 KV head, d 64, 256 BF16 tokens, 4 splits of 64",
        "hybrid": "hybrid tier: batch 4, 32 q / 8 KV heads, d 128, 32768 tokens (newest 2048 BF16, 30720 4-bit codes)",
        "ragged": "ragged paged hybrid: batch 64, lengths U[1024, 65536], 16-token pages, newest 1024 BF16",
        "staged-hybrid": "staged 128k hybrid history: batch 1, 16 layers, 32 q / 8 KV heads, d 128, newest 2048 "
                         "tokens BF16 on the device, 129024 compact in pinned host memory, 4096-token chunks",
        "staged": "staged 128k history: batch 1, 16 layers, 32 q / 8 KV heads, d 128, 131072 BF16 tokens per layer "
                  "in pinned host memory, 4096-token chunks through a 2-buffer device region, one token appended "
                  "per step",
    }[name], "batch": wl.B, "q_heads": wl.Hq, "kv_heads": wl.Hkv, "head_dim": wl.d, "split_tokens": wl.split_tokens}
    if w is not None:
        d["kv_bytes_per_step"] = w.kv_bytes()
        d["l2"] = ("inputs larger than the 126 MB L2, no flush" if w.kv_bytes() > 126e6
                   else "L2 flushed (256 MB write) before every step; each step timed by its own events, the flush not timed")
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
            "config": {**describe(args.workload, wl), "reference": "float64 numpy oracle on the host CPU",
                       "step": desc},
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


def run_ours(args):
    import torch
    from kv_cache_tiering_b200 import akv

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    variant = {"auto": akv.AKV_VARIANT_AUTO, "simt": akv.AKV_VARIANT_SIMT, "mma": akv.AKV_VARIANT_MMA}[args.variant]
    wl, w, tokens = make_workload(args.workload, dev, rank)
    step = w.step
    stream = torch.cuda.current_stream()
    flush = None
    if w.kv_bytes() <= 126e6:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    fuse = args.fuse and variant != akv.AKV_VARIANT_SIMT

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
    launches_per_step = sum(1 for t in step.tiers if int(sum(t.lens)) > 0) + 1

    sampler = ClockSampler(local)
    sampler.start()
    for _ in range(max(3, args.warmup)):
        one_step()
    torch.cuda.synchronize()
    # soak: steady-state steps before the timed region
    t_soak = time.monotonic()
    while time.monotonic() - t_soak < args.soak_seconds:
        for _ in range(20):
            one_step()
        torch.cuda.synchronize()

    # events around every tier's launch on every SAMPLE-th step, so the dominant kernel is
    # timed on its own; the other steps run without events between their launches (an event
    # between two kernels would stop the next one from overlapping the previous one's tail)
    live = [i for i, t in enumerate(step.tiers) if int(sum(t.lens)) > 0]
    per_tier = not fuse and len(live) > 1
    n_b = len(live) + 1 if per_tier else 2
    sampled = list(range(0, args.steps, SAMPLE))
    bounds = [[torch.cuda.Event(enable_timing=True) for _ in sampled] for _ in range(n_b)]
    a0, a1 = bounds[0], bounds[-1]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.monotonic()
    # with an L2 flush between steps (inputs smaller than L2), each step is bracketed by its own
    # events after the flush, and the time is the sum of the steps: the flush is not timed
    step_ev = ([(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)] if flush is not None else None)
    start.record(stream)
    for i in range(args.steps):
        if flush is not None:
            flush.fill_(1)
            step_ev[i][0].record(stream)
        k = i // SAMPLE if i % SAMPLE == 0 else -1
        if k >= 0:
            a0[k].record(stream)
        if fuse:
            step.decode(w.q, variant, stream)
        elif per_tier and k >= 0:
            for j, ti in enumerate(live):
                step.attend_tier(ti, w.q, variant, stream)
                bounds[j + 1][k].record(stream)
        else:
            step.attend(w.q, variant, stream)
        if k >= 0:
            a1[k].record(stream)
        if not fuse:
            step.merge(stream)
        if flush is not None:
            step_ev[i][1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.monotonic()
    if dist:
        dist.barrier()
    ms = start.elapsed_time(end) if flush is None else sum(a.elapsed_time(b) for a, b in step_ev)
    attend_ms = [a0[k].elapsed_time(a1[k]) for k in range(len(sampled))]
    tier_ms = ([statistics.fmean(bounds[j][k].elapsed_time(bounds[j + 1][k]) for k in range(len(sampled)))
                for j in range(len(live))] if per_tier else None)
    if dist:
        ms = max_over_ranks(ms, dist, dev)
    # post-timed soak so the sampler has points inside the loaded window
    t_post = time.monotonic()
    while time.monotonic() - t_post < 0.3:
        for _ in range(20):
            one_step()
        torch.cuda.synchronize()
    err = int(step.err.item())

    # ---- end to end through the public API: every step takes its query from pinned host memory
    # and leaves O and LSE in pinned host memory.  Unfused, that is one akv_decode_host call
    # per step on the compute stream (the GPU reads the query and writes the results over PCIe
    # itself, alternating two output buffers).  Fused (akv_decode has no host form), the copies
    # run on streams of their own with two buffers each, events ordering every reuse.
    from kv_cache_tiering_b200 import workloads as wlmod
    q_host = torch.from_numpy(w.q_bits.view("int16")).pin_memory()
    pair = [step, wlmod.DecodeStep(step.B, step.Hq, step.Hkv, step.d, step.split_tokens, step.scale, step.tiers, dev)]
    q_dev = [torch.empty_like(w.q) for _ in range(2)]
    o_host = [torch.empty(step.o.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    lse_host = [torch.empty(step.lse.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # upload j landed
    ev_used = [torch.cuda.Event() for _ in range(2)]  # step j's compute is done with its buffers
    ev_out = [torch.cuda.Event() for _ in range(2)]   # download j landed

    e2e_ev = None  # per-step events when the L2 flush sits between steps (set for the timed run)

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
                  for _ in range(args.steps)]
    if dist:
        dist.barrier()
    e0.record(stream)
    up.wait_event(e0)
    for i in range(args.steps):
        e2e_step(i)
    if fuse:
        stream.wait_event(ev_out[(args.steps - 1) % 2])
        stream.wait_event(ev_out[args.steps % 2])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) if e2e_ev is None else sum(a.elapsed_time(b) for a, b in e2e_ev)
    if dist:
        e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    sampler.stop()

    total_tokens = tokens * world * args.steps
    value = total_tokens / (ms * 1e-3)
    e2e_value = total_tokens / (e2e_ms * 1e-3)
    peak, peak_kind = peaks()
    attend_avg_ms = sum(attend_ms) / len(attend_ms)
    kv_bytes = w.kv_bytes()
    tb = w.tier_bytes()
    kernel_names = ["attend_codes_mma" if step.tiers[i].kind == akv.AKV_TIER_CODES4 else "attend_bf16_mma"
                    for i in live]
    if variant == akv.AKV_VARIANT_SIMT:
        kernel_names = [k.replace("_mma", "_simt") for k in kernel_names]
    if per_tier:
        # the dominant kernel: the tier launch with the largest share of the step
        j = max(range(len(live)), key=lambda k: tier_ms[k])
        dom_ms, dom_bytes, dom_kernel = tier_ms[j], tb[live[j]], kernel_names[j]
    else:
        dom_ms, dom_bytes = attend_avg_ms, kv_bytes
        dom_kernel = kernel_names[0] if len(live) == 1 else "attention launches"
        if fuse:
            dom_kernel += " + merge (one akv_decode call)"
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    traffic = None if fuse else recorded_traffic(args.workload, dom_kernel)
    clocks = sampler.summary(t_soak, t_wall1 + 0.3)
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": dict(describe(args.workload, wl, w), parallelism=f"independent replicas x{world}",
                               accumulate="f32", variant=args.variant,
                               step="one akv_decode call (attention launches + merge launch)" if fuse
                               else "attention launches + merge launch"),
                "hbm_gbs": kv_bytes * world * args.steps / (ms * 1e-3) / 1e9,
                "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                             "frac": achieved / peak, "traffic": traffic, "kernel": dom_kernel,
                             "algorithmic_bytes": dom_bytes, "kernel_ms_avg": dom_ms,
                             "peak_source": f"{peak_kind} hbm_gbs (copy bandwidth)",
                             "attend_ms_avg": attend_avg_ms,
                             "tiers_ms_avg": dict(zip(kernel_names, tier_ms)) if per_tier else None},
                "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(q_host.numel() * 2),
                        "d2h_bytes_per_step": int(o_host[0].numel() * 4 + lse_host[0].numel() * 4),
                        "transfers": ("copies on their own streams, two buffers each" if fuse else
                                      "akv_decode_host: the GPU reads the pinned query and writes O and LSE "
                                      "into pinned host memory, one stream")},
                "gpu_launches": launches_per_step * args.steps,
                "clocks": clocks, "device_error_word": err}
        if world == 1 and not args.no_cpu_baseline:
            cv, units, desc, dt = time_oracle(args.workload, wl)
            line["cpu_baseline"] = {"value": cv, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                                    "sample": f"{units} units ({desc}), {dt:.1f} s"}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_staged(args):
    """Staged 128k decode: PCIe-bound, timed by host wall clock around an uninstrumented loop
    (timing-enabled events serialise the copies they observe); one replica per rank."""
    import torch
    from kv_cache_tiering_b200 import akv, synth, workloads

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=dev)
    hybrid = args.workload == "staged-hybrid"
    base = synth.WORKLOADS[args.workload]
    wl = synth.Workload(base.name, base.B, base.Hq, base.Hkv, base.d, base.split_tokens, seed=base.seed + rank,
                        extra=dict(base.extra))
    layers = args.layers or wl.extra["layers"]
    n_steps = max(3, args.warmup) + args.steps
    if hybrid:
        st = workloads.StagedHybridDecode(wl, dev, layers=layers, T=wl.extra["T"], W=wl.extra["window"],
                                          chunk=wl.extra["chunk"], max_steps=n_steps + 1)
    else:
        st = workloads.StagedDecode(wl, dev, layers=layers, max_steps=n_steps + 1)
    o_host = torch.empty(st.o.shape, dtype=torch.float32).pin_memory()
    lse_host = torch.empty(st.lse.shape, dtype=torch.float32).pin_memory()

    def one_step(i):
        st.step(*inputs[i], variant)
        with torch.cuda.stream(st.compute_stream):  # the step's result, read back every step
            o_host.copy_(st.o, non_blocking=True)
            lse_host.copy_(st.lse, non_blocking=True)
    variant = {"auto": akv.AKV_VARIANT_AUTO, "simt": akv.AKV_VARIANT_SIMT, "mma": akv.AKV_VARIANT_MMA}[args.variant]
    inputs = [st.inputs(i) for i in range(n_steps)]
    # pinned host -> device copy bandwidth of this machine (the PCIe roofline): the best of three
    # rounds of four 256 MiB copies, timed with events on the copying stream
    probe_h = torch.empty(256 << 20, dtype=torch.uint8).pin_memory()
    probe_d = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(3):
        probe_d.copy_(probe_h, non_blocking=True)
    torch.cuda.synchronize()
    pcie_peak = 0.0
    for _ in range(3):
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record()
        for _ in range(4):
            probe_d.copy_(probe_h, non_blocking=True)
        p1.record()
        torch.cuda.synchronize()
        pcie_peak = max(pcie_peak, 4 * probe_h.numel() / (p0.elapsed_time(p1) * 1e-3) / 1e9)
    del probe_h, probe_d
    sampler = ClockSampler(local)
    sampler.start()
    for i in range(max(3, args.warmup)):
        one_step(i)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    h2d0 = st.h2d_bytes
    tw0 = time.monotonic()
    t0 = time.perf_counter()
    for i in range(max(3, args.warmup), n_steps):
        one_step(i)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    tw1 = time.monotonic()
    if dist:
        t = torch.tensor([dt], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dt = float(t.item())
    sampler.stop()
    h2d = st.h2d_bytes - h2d0
    n_tok = sum(layers * (wl.extra["T"] + i + 1) for i in range(max(3, args.warmup), n_steps))
    value = n_tok * world / dt
    err = int(st.err.item())
    st.close()
    if rank == 0:
        pcie = h2d / dt / 1e9
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": ("staged 128k hybrid history: batch 1, %d layers, 32 q / 8 KV heads, d 128, "
                                        "131072 tokens per layer: newest 2048 BF16 on the device, 129024 as 4-bit "
                                        "codes in pinned host memory, 4096-token chunks through a 2-buffer device "
                                        "region, one token appended per step" if hybrid else
                                        "staged 128k history: batch 1, %d layers, 32 q / 8 KV heads, d 128, "
                                        "131072 BF16 tokens per layer in pinned host memory, 4096-token chunks "
                                        "through a 2-buffer device region, one token appended per step") % layers,
                           "timing": "host wall clock, timing-disabled fences", "parallelism":
                           f"independent replicas x{world}", "variant": args.variant},
                "roofline": {"bound": "pcie", "achieved": pcie, "peak": pcie_peak, "unit": "GB/s",
                             "frac": pcie / pcie_peak, "traffic": None,
                             "peak_source": "pinned 256 MiB host-to-device copies measured in this run (best of 3 rounds of 4)"},
                "pcie_h2d_gbs": pcie, "h2d_bytes_per_step": h2d // args.steps,
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": h2d // args.steps,
                        "d2h_bytes_per_step": (0 if hybrid else layers * st.row_bytes)
                        + 4 * (o_host.numel() + lse_host.numel())},
                # attention launches per layer (one per staged chunk, plus the window for the
                # hybrid) and the merge
                "gpu_launches": args.steps * layers * (
                    (-(-st.Tc // st.chunk) + 2) if hybrid else (-(-(wl.extra["T"] + 1) // st.chunk) + 1)),
                "clocks": sampler.summary(tw0, tw1), "device_error_word": err}
        if world == 1 and not args.no_cpu_baseline:
            cv, units, desc, odt = time_oracle(args.workload, wl)
            line["cpu_baseline"] = {"value": cv, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                                    "sample": f"{units} units ({desc}), {odt:.1f} s"}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_aging(args):
    """Live hybrid decode with window aging on the hybrid shape: every step appends a token
    per sequence; every 16 steps each window hands its oldest page to the compact tier.
    Timed with CUDA events on the step's stream, whole steps and the parts."""
    import torch
    from kv_cache_tiering_b200 import akv, synth, workloads

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    base = synth.WORKLOADS["hybrid"]
    wl = synth.Workload("aging", base.B, base.Hq, base.Hkv, base.d, base.split_tokens, seed=base.seed + rank,
                        extra=dict(base.extra))
    T, W = wl.extra["T"], wl.extra["window"]
    n_warm = max(3, args.warmup)
    n_steps = n_warm + args.steps
    st = workloads.AgingHybrid(wl, dev, [T] * wl.B, W, max_steps=n_steps + 1, source="torch")
    variant = {"auto": akv.AKV_VARIANT_AUTO, "simt": akv.AKV_VARIANT_SIMT, "mma": akv.AKV_VARIANT_MMA}[args.variant]
    inputs = [st.inputs(i) for i in range(n_steps)]
    stream = torch.cuda.current_stream()
    for i in range(n_warm):
        st.step(*inputs[i], variant, stream)
    torch.cuda.synchronize()
    aged0, tok = st.aged_blocks, 0
    st.encode_events = []
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n_warm, n_steps):
        tok += int(st.c.sum() + st.win.sum()) + wl.B
        st.step(*inputs[i], variant, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if dist:
        ms = max_over_ranks(ms, dist, dev)
    aged = st.aged_blocks - aged0
    enc_us = [a.elapsed_time(b) * 1e3 for a, b in st.encode_events]
    value = tok * world / (ms * 1e-3)
    err = int(st.err.item())
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": "window aging on the hybrid shape: batch 4, 32 q / 8 KV heads, d 128, "
                                       "32768 tokens, newest 2048-2063 BF16 in 16-token ring pages, the rest 4-bit "
                                       "code pages; one token appended per step, full window pages encoded into "
                                       "the compact tier", "parallelism": f"independent replicas x{world}",
                           "variant": args.variant, "timing": "CUDA events around whole steps"},
                "aged_blocks_in_timed_steps": int(aged) * wl.Hkv, "aging_events": len(enc_us),
                "aging_encode_us_avg": sum(enc_us) / max(1, len(enc_us)),
                "e2e": None, "gpu_launches": args.steps * 3 + int(aged > 0) * (aged // wl.B),
                "device_error_word": err}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload in ("staged", "staged-hybrid"):
        return run_staged(args)
    if args.workload == "aging":
        return run_aging(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
