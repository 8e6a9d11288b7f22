"""Benchmark: steady-state chunk step of the 832x464 single-layer rollout.

One step = one 4-latent-frame chunk of the rollout at steady state: the chunk's
queries attend 6 anchor + 8 window frames + the chunk itself (27144 keys,
12 heads, head_dim 128, bf16) through ``chunk_attention_fwd`` (RoPE staging of
Q and the current K, then tensor-core attention), then the chunk's K/V are
appended to the cache through ``kv_cache_append_rope`` (RoPE of K, oldest
non-anchor frames evicted).  The metric is useful attention TFLOP/s
(4 * Lq * Lk * H * D per step), with ms/step, the attention kernel's share of
the dense bf16 roofline and the append kernel's GB/s reported beside it.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                [--shard heads|layers]
Multi-GPU (one process per GPU; ``--gpus N`` without torchrun starts the N ranks
through torch.distributed.run): with ``--shard heads`` (the default) rank r owns
a contiguous range of the 12 heads of the layer cache, so the ranks split one
chunk step (strong scaling); with ``--shard layers`` every rank runs a layer
cache of its own (weak scaling).  Neither has a collective on the data path;
the timed region is bracketed by barriers and the max elapsed time over ranks
is reported.  At one GPU the line also carries the 30-layer x 4-step chunk
(120 attention calls and one batched append of 30 layer caches) as extra keys.
``--impl reference`` times the CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from kv_cache_chunk_ring_b200 import shard as sh  # noqa: E402
from kv_cache_chunk_ring_b200 import workloads as wl  # noqa: E402

SPEC = wl.VIDEO_832x464
METRIC = "chunk-attention useful TFLOP/s & % of B200 bf16 peak; ms/chunk; append GB/s"
UNIT = "TFLOP/s"
STEADY_CHUNK = 4          # chunks 0-3 fill the cache; from chunk 4 on it holds 14 frames
POOL = 3                  # distinct input chunks cycled through the timed steps
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def step_flops(spec=SPEC, heads=None) -> float:
    lq = spec.chunk_tokens
    lk = (spec.sinks + spec.window + spec.chunk_frames) * spec.tokens_per_frame
    return 4.0 * lq * lk * (spec.heads if heads is None else heads) * spec.head_dim


def append_bytes(spec=SPEC, heads=None) -> float:
    # read K and V, write rotated K and V: 4 * F * T * H * D * 2 bytes
    return 4.0 * spec.chunk_tokens * (spec.heads if heads is None else heads) * spec.head_dim * 2


def config_dict(spec=SPEC, shard="heads", world=1) -> dict:
    lk = (spec.sinks + spec.window + spec.chunk_frames) * spec.tokens_per_frame
    return {
        "workload": spec.name,
        "heads": spec.heads, "head_dim": spec.head_dim,
        "tokens_per_frame": spec.tokens_per_frame, "grid": [spec.grid_h, spec.grid_w],
        "chunk_frames": spec.chunk_frames, "sinks": spec.sinks, "window": spec.window,
        "q_tokens": spec.chunk_tokens, "keys": lk,
        "step": "chunk_attention_fwd (RoPE stage + attention) + kv_cache_append_rope, steady state",
        "l2": "inputs larger than L2: each step reads 130 MB of cached K/V + 55.6 MB chunk inputs",
        "parallelism": ("single GPU" if world == 1 else
                        f"{world} ranks, {'heads of one layer cache split' if shard == 'heads' else 'one layer cache each'}; no collective"),
    }


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


ATTN_SOURCES = ("attn_sm100.cu", "sm100_ptx.cuh", "kvcr_internal.h")


def kernel_source_hash(names=ATTN_SOURCES) -> str:
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "kv_cache_chunk_ring_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(record="chunk_attn_832x464.json", names=ATTN_SOURCES):
    """DRAM bytes per launch of a kernel from its committed ncu record (JSON: source
    hash and dram bytes per launch), or None when the record is missing or was taken
    on different kernel source."""
    p = os.path.join(ROOT, "profiles", record)
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    if rec.get("source_hash") != kernel_source_hash(names):
        return None
    return float(rec["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        self.dev = ids[device_index] if device_index < len(ids) else str(device_index)
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"kvcr_clocks_{os.getpid()}.csv")
        self.t0 = self.t1 = None

    def window(self, t0: float, t1: float):
        """Wall-clock bounds (time.time()) of the timed region: only samples taken
        inside it are summarised."""
        self.t0, self.t1 = t0, t1

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "25"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            cols = [c.strip() for c in line.split(",")]
            if len(cols) < 10:
                continue
            try:
                stamp, frac = (cols[0].split(".") + ["0"])[:2]
                t = time.mktime(time.strptime(stamp, "%Y/%m/%d %H:%M:%S")) + float("0." + frac)
                clk = float(cols[2])
                top = float(cols[3])
            except ValueError:
                continue
            if self.t0 is not None and not (self.t0 <= t <= self.t1):
                continue                      # outside the timed region
            sm.append(clk)
            mx = top
            for n, c in zip(names, cols[6:10]):
                if c.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------- multi-process --

def free_port() -> int:
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def max_over_ranks(value: float, dist, device) -> float:
    """The largest of every rank's value (the whole job ends when the slowest rank does)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_throughput(world: int, steps: int, flops_per_step: float, elapsed_ms: float) -> float:
    """TFLOP/s of all ranks together: every rank runs `steps` steps of its own work."""
    return world * steps * flops_per_step / (elapsed_ms * 1e-3) / 1e12


# --------------------------------------------------------------------- ours --

def run_ours(args, rank: int, world: int, dist) -> dict:
    import torch
    from kv_cache_chunk_ring_b200 import build as _build
    from kv_cache_chunk_ring_b200 import kvcr

    if rank == 0 or not os.path.exists(os.path.join(ROOT, "kv_cache_chunk_ring_b200", "libkvcr.so")):
        _build.build()
    if dist is not None:
        dist.barrier()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    spec = SPEC
    shard = args.shard if world > 1 else "heads"
    if shard == "heads":                    # this rank's heads of the one layer cache
        h0, h1 = sh.head_range(spec.heads, world, rank)
        layer = 0
    else:                                   # a layer cache of its own, all heads
        h0, h1 = 0, spec.heads
        layer = rank
    T, H, D, F = spec.tokens_per_frame, h1 - h0, spec.head_dim, spec.chunk_frames
    stream = torch.cuda.current_stream()

    cache = kvcr.Cache(spec.sinks, spec.window, T, H, D, F, rope=spec.rope(), fused_finalize=True)
    # seeded synthetic chunks: fill chunks + a pool for timing, this rank's heads
    gen = wl.rollout_chunks(wl.shrink(spec, n_chunks=STEADY_CHUNK + POOL), layer=layer)
    chunks = []
    for item in gen:
        chunks.append(tuple(sh.slice_heads(torch.from_numpy(item[x]), h0, h1).to(dev, torch.bfloat16)
                            for x in ("q", "k", "v")))
    o = torch.empty_like(chunks[0][0])
    frame = [0]

    def step(i):
        q, k, v = chunks[STEADY_CHUNK + (i % POOL)] if i >= 0 else chunks[i + STEADY_CHUNK]
        frames = list(range(frame[0], frame[0] + F))
        cache.attention(q, k, v, frames, out=o)
        cache.append(k, v, frames)
        frame[0] += F

    # fill the cache to steady state (chunks 0-3), then warm up
    for i in range(-STEADY_CHUNK, 0):
        step(i)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert cache.num_cached() == spec.sinks + spec.window

    # ---------------- timed region (device events, no tracing) ----------------
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.5)                                   # nvidia-smi up and sampling
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = kvcr.kvcr_launch_count()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    ev0.record(stream)
    for i in range(args.steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    w1 = time.time()
    if dist is not None:
        dist.barrier()
    launches = kvcr.kvcr_launch_count() - launches0
    sampler.window(w0, w1)
    clocks = sampler.stop()
    elapsed_ms = max_over_ranks(ev0.elapsed_time(ev1), dist, dev)

    # ---------------- per-kernel times (traced pass, same steps) ----------------
    kvcr.kvcr_trace_reset()
    kvcr.kvcr_trace_enable(True)
    for i in range(args.steps):
        step(i)
    torch.cuda.synchronize()
    kvcr.kvcr_trace_enable(False)
    kt = {}
    for kid, name in kvcr.KERNEL_NAMES.items():
        n, ms = kvcr.kvcr_trace_read(kid)
        if n:
            kt[name] = {"launches": n, "avg_ms": ms / n}
    kvcr.kvcr_trace_reset()

    # ---------------- the same step as one fused call (attention + append) ----------------
    def step_fused(i):
        q, k, v = chunks[STEADY_CHUNK + (i % POOL)]
        frames = list(range(frame[0], frame[0] + F))
        cache.attention_finalize(q, k, v, frames, out=o)
        frame[0] += F

    for i in range(args.warmup):
        step_fused(i)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for i in range(args.steps):
        step_fused(i)
    f1.record(stream)
    torch.cuda.synchronize()
    fused_ms = max_over_ranks(f0.elapsed_time(f1), dist, dev)

    # ---------------- end to end through the public API with host buffers ----------------
    # Every step uploads its Q, K, V from pinned host memory and downloads its O.  Two
    # device buffer sets are used in turn: the upload of step i+1 (copy stream) and the
    # download of step i-1 (second copy stream) overlap the compute of step i.
    host = [tuple(t.cpu().pin_memory() for t in chunks[STEADY_CHUNK + j]) for j in range(POOL)]
    dbuf = [tuple(torch.empty_like(chunks[0][x]) for x in range(3)) for _ in range(2)]
    obuf = [torch.empty_like(o) for _ in range(2)]
    o_host = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for _ in range(2)]
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("uploaded", "computed", "downloaded")}
    started = {k: [False, False] for k in ("computed", "downloaded")}

    def e2e_step(i):
        b = i % 2
        hq, hk, hv = host[i % POOL]
        dq, dk, dvv = dbuf[b]
        with torch.cuda.stream(up):
            if started["computed"][b]:
                up.wait_event(ev["computed"][b])       # step i-2 has consumed this buffer set
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dvv.copy_(hv, non_blocking=True)
            ev["uploaded"][b].record(up)
        stream.wait_event(ev["uploaded"][b])
        if started["downloaded"][b]:
            stream.wait_event(ev["downloaded"][b])     # O of step i-2 has left the device
        frames = list(range(frame[0], frame[0] + F))
        cache.attention(dq, dk, dvv, frames, out=obuf[b], stream=stream)
        cache.append(dk, dvv, frames, stream=stream)
        frame[0] += F
        ev["computed"][b].record(stream)
        started["computed"][b] = True
        with torch.cuda.stream(down):
            down.wait_event(ev["computed"][b])
            o_host[b].copy_(obuf[b], non_blocking=True)
            ev["downloaded"][b].record(down)
        started["downloaded"][b] = True

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_event(e0)
    for i in range(args.steps):
        e2e_step(i)
    for b in range(2):
        stream.wait_event(ev["downloaded"][b])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    kvcr.kvcr_check_status()

    flops = step_flops(spec, H)                     # this rank's work per step
    # the whole job per step: one 12-head layer split by head, or one layer per rank
    job_ranks = 1 if shard == "heads" else world
    value = whole_job_throughput(job_ranks, args.steps, step_flops(spec), elapsed_ms)
    e2e_value = whole_job_throughput(job_ranks, args.steps, step_flops(spec), e2e_ms)
    peaks, peak_kind = load_peaks()
    attn = kt.get("chunk_attn", {})
    attn_ms = attn.get("avg_ms", float("nan"))
    achieved = flops / (attn_ms * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    app = kt.get("append_rope", {})
    app_gbs = append_bytes(spec, H) / (app.get("avg_ms", float("nan")) * 1e-3) / 1e9
    chunk_bytes = job_ranks * spec.chunk_tokens * spec.heads * D * 2   # whole job
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "strong" if (shard == "heads" and world > 1) else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict(spec, shard, world),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": recorded_traffic(),
                     "kernel": "chunk_attn (tcgen05 attention, one launch per step)",
                     "peak_source": f"{peak_kind} bf16_tflops (burst)",
                     # the timed loop runs long enough to meet the 1 kW power cap; the
                     # same achieved rate against the sustained (power-capped) figure:
                     "frac_sustained": round(achieved / float(
                         peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])), 4)},
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT,
                "h2d_bytes_per_step": 3 * chunk_bytes, "d2h_bytes_per_step": chunk_bytes,
                "ms_per_step": round(e2e_ms / args.steps, 4),
                "note": "uploads / downloads on two copy streams, double-buffered against compute"},
        "gpu_launches": int(launches),
        "kernels": {k: {"launches": v["launches"], "avg_ms": round(v["avg_ms"], 5)}
                    for k, v in kt.items()},
        "attn_ms_per_call": round(attn_ms + kt.get("rope_stage", {}).get("avg_ms", 0.0), 5),
        "ms_per_step_fused_call": round(fused_ms / args.steps, 4),
        "value_fused_call": round(whole_job_throughput(job_ranks, args.steps, step_flops(spec),
                                                       fused_ms), 2),
        "attn_kernel_pct_of_peak": round(100 * achieved / peak, 2),
        "append_gb_s": round(app_gbs, 1),
        "append_hbm_frac": round(app_gbs / float(peaks["hbm_gbs"]), 4),
        "clocks": clocks,
    }
    # the same kernel against the tensor cores' issue rate at the SM clock seen during the
    # timed region: 148 SMs x 8192 dense bf16 FLOP per SM clock (one 128 x 128 x 16 MMA
    # per 32 clocks, measured full-rate in a standalone tcgen05 loop)
    if clocks and clocks.get("sm_mhz"):
        n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
        clock_peak = n_sm * 8192 * clocks["sm_mhz"] * 1e6 / 1e12
        out["attn_kernel_frac_of_clock_peak"] = round(achieved / clock_peak, 4)
        out["clock_peak_tflops"] = round(clock_peak, 1)
    return out


# ---------------------------------------------------------------- oracle ----

def oracle_sample(rows: int, seed_chunk=STEADY_CHUNK):
    """Build a bounded oracle sample of one steady-state chunk step and return a
    callable that runs it plus the useful FLOPs it covers."""
    from oracle.rollout import rollout  # noqa: F401  (oracle package)
    from oracle.attn import attention
    from oracle.rope import rope3d, rope_positions

    spec = wl.shrink(SPEC, n_chunks=seed_chunk + 1)
    items = list(wl.rollout_chunks(spec))
    pairs = (spec.rope().pairs_t, spec.rope().pairs_h, spec.rope().pairs_w)
    T = spec.tokens_per_frame
    # the steady-state cache content: anchors 0-5 and window frames 8-15 (rotated K, V)
    cached_k, cached_v = [], []
    keep = list(range(spec.sinks)) + list(range(seed_chunk * spec.chunk_frames - spec.window,
                                               seed_chunk * spec.chunk_frames))
    for it in items[:-1]:
        t, h, w = rope_positions(it["frames"], spec.grid_h, spec.grid_w)
        kr = rope3d(it["k"], t, h, w, pairs)
        for n, f in enumerate(it["frames"]):
            if f in keep:
                cached_k.append(kr[n * T:(n + 1) * T])
                cached_v.append(it["v"][n * T:(n + 1) * T].astype(np.float64))
    cur = items[-1]
    sel = wl.sample_rows(spec.chunk_tokens, rows, 2024)
    lk = (len(keep) + spec.chunk_frames) * T
    flops = 4.0 * len(sel) * lk * spec.heads * spec.head_dim
    scale = 1.0 / math.sqrt(spec.head_dim)

    def run():
        t, h, w = rope_positions(cur["frames"], spec.grid_h, spec.grid_w)
        qr = rope3d(cur["q"][sel], t[sel], h[sel], w[sel], pairs)
        kc = rope3d(cur["k"], t, h, w, pairs)
        k_all = np.concatenate(cached_k + [kc])
        v_all = np.concatenate(cached_v + [cur["v"].astype(np.float64)])
        return attention(qr, k_all, v_all, scale)

    return run, flops, len(sel)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(budget_s: float = 15.0) -> dict:
    # two probe sizes separate the fixed cost (RoPE of the chunk's keys) from the per-row cost
    times = []
    for n_probe in (32, 128):
        run, flops, n = oracle_sample(n_probe)
        t0 = time.perf_counter()
        run()
        times.append((n, time.perf_counter() - t0))
    per_row = max((times[1][1] - times[0][1]) / (times[1][0] - times[0][0]), 1e-6)
    fixed = max(times[0][1] - per_row * times[0][0], 0.0)
    rows = int(max(32, min(SPEC.chunk_tokens, (budget_s - fixed) / per_row)))
    run, flops, n = oracle_sample(rows)
    t0 = time.perf_counter()
    run()
    dt = time.perf_counter() - t0
    return {"value": round(flops / dt / 1e12, 6), "unit": UNIT, "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"one steady-state chunk step of {SPEC.name} restricted to {n} of "
                      f"{SPEC.chunk_tokens} query rows (all 12 heads, RoPE of the rows' Q and "
                      f"the chunk's K, attention over 27144 keys), numpy fp64; "
                      f"{dt:.1f} s"}


def run_reference(args) -> dict:
    """The oracle as the reference arm: each step = the bounded oracle sample."""
    per_step_budget = max(0.2, 150.0 / max(1, args.steps + args.warmup))  # ~150 s in all
    run, flops, n = oracle_sample(32)
    t0 = time.perf_counter()
    run()
    per_row = (time.perf_counter() - t0) / n
    rows = int(max(16, min(2048, per_step_budget / max(per_row, 1e-6))))
    run, flops, n = oracle_sample(rows)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    value = args.steps * flops / dt / 1e12
    sample = (f"per step: one steady-state chunk step of {SPEC.name} restricted to {n} query rows"
              f" (all heads, 27144 keys), numpy fp64 on host cores")
    return {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(), "impl": "reference",
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": blas_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------- other workloads ----
# Single-GPU timings of the other workloads; inputs are seeded N(0,1) bf16 drawn on the
# device with torch (same distribution as the parity inputs, generated faster).

def _randn(shape, gen):
    import torch
    return torch.randn(shape, generator=gen, device="cuda", dtype=torch.float32).to(torch.bfloat16)


def _timed(fn, steps, warmup):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def run_layers30(args, clocks=False) -> dict:
    """30 layers x 4 denoising steps per chunk (120 attention calls + 30 appends), timed
    with one append per layer and with one batched append of the 30 caches."""
    import torch
    from kv_cache_chunk_ring_b200 import build as _build
    from kv_cache_chunk_ring_b200 import kvcr
    _build.build()
    spec = wl.VIDEO_832x464_30L
    if getattr(args, "layers", 0):                    # fewer layers (a profiler-sized case)
        spec = dataclasses.replace(spec, name=f"chunk_attn_832x464_{args.layers}layers_4steps",
                                   layers=args.layers)
    T, H, D, F = spec.tokens_per_frame, spec.heads, spec.head_dim, spec.chunk_frames
    # spare slots for the fused last step (chunk_attention_fwd_finalize); the other
    # paths use these caches like plain ones
    caches = [kvcr.Cache(spec.sinks, spec.window, T, H, D, F, rope=spec.rope(),
                         fused_finalize=True) for _ in range(spec.layers)]
    gen = torch.Generator(device="cuda").manual_seed(spec.seed)
    pool = [tuple(_randn((spec.chunk_tokens, H, D), gen) for _ in range(3)) for _ in range(6)]
    o = torch.empty_like(pool[0][0])
    frame = [0]
    n_call = [0]

    def chunk():
        frames = list(range(frame[0], frame[0] + F))
        for li, c in enumerate(caches):
            for s in range(spec.steps):
                q, k, v = pool[n_call[0] % len(pool)]
                n_call[0] += 1
                c.attention(q, k, v, frames, out=o)
            c.append(k, v, frames)
        frame[0] += F

    def chunk_batched():
        # the same chunk with the 30 appends done by one batched launch at its end
        frames = list(range(frame[0], frame[0] + F))
        ks, vs = [], []
        for li, c in enumerate(caches):
            for s in range(spec.steps):
                q, k, v = pool[n_call[0] % len(pool)]
                n_call[0] += 1
                c.attention(q, k, v, frames, out=o)
            ks.append(k)
            vs.append(v)
        kvcr.append_batch(caches, ks, vs, frames)
        frame[0] += F

    def chunk_fused():
        # the same chunk with each layer's last step attending and appending in one call
        frames = list(range(frame[0], frame[0] + F))
        for li, c in enumerate(caches):
            for s in range(spec.steps):
                q, k, v = pool[n_call[0] % len(pool)]
                n_call[0] += 1
                if s == spec.steps - 1:
                    c.attention_finalize(q, k, v, frames, out=o)
                else:
                    c.attention(q, k, v, frames, out=o)
        frame[0] += F

    for _ in range(STEADY_CHUNK):
        chunk()
    kvcr.kvcr_trace_reset()
    sampler = ClockSampler(torch.cuda.current_device()) if clocks else None
    if sampler:
        sampler.start()
        time.sleep(0.5)                               # nvidia-smi up and sampling
    w0 = time.time()
    ms = _timed(chunk, args.steps, args.warmup)
    ms_batched = _timed(chunk_batched, args.steps, args.warmup)
    ms_fused = _timed(chunk_fused, args.steps, args.warmup)
    w1 = time.time()
    if sampler:
        sampler.window(w0, w1)
    clk = sampler.stop() if sampler else None
    kvcr.kvcr_trace_enable(True)
    chunk()
    chunk_batched()
    torch.cuda.synchronize()
    kvcr.kvcr_trace_enable(False)
    kt = {name: kvcr.kvcr_trace_read(kid) for kid, name in kvcr.KERNEL_NAMES.items()}
    kvcr.kvcr_trace_reset()
    flops = spec.layers * spec.steps * step_flops(spec)
    bat_n, bat_ms = kt["append_batch"]
    app_n, app_ms = kt["append_rope"]
    peaks, _ = load_peaks()
    attn_call_ms = kt["chunk_attn"][1] / max(1, kt["chunk_attn"][0])
    bat_gbs = spec.layers * append_bytes(spec) / (bat_ms / max(1, bat_n) * 1e-3) / 1e9
    return {"workload": spec.name, "ms_per_chunk": round(ms, 3),
            "attn_kernel_frac": round(step_flops(spec) / (attn_call_ms * 1e-3) / 1e12 /
                                      float(peaks["bf16_tflops"]), 4),
            # the chunk runs for seconds under the power cap: the sustained peak applies
            "attn_kernel_frac_sustained": round(
                step_flops(spec) / (attn_call_ms * 1e-3) / 1e12 /
                float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])), 4),
            "append_batch_hbm_frac": round(bat_gbs / float(peaks["hbm_gbs"]), 4),
            "clocks": clk,
            "attention_tflops_per_chunk": round(flops / 1e12, 2),
            "value": round(flops / (ms * 1e-3) / 1e12, 2), "unit": UNIT,
            "attn_kernel_ms": round(kt["chunk_attn"][1] / max(1, kt["chunk_attn"][0]), 4),
            "append_kernel_us": round(1e3 * app_ms / max(1, app_n), 2),
            "append_gb_s": round(append_bytes(spec) / (app_ms / max(1, app_n) * 1e-3) / 1e9, 1),
            "ms_per_chunk_batched_append": round(ms_batched, 3),
            "ms_per_chunk_fused_last_step": round(ms_fused, 3),
            "append_batch_kernel_us": round(1e3 * bat_ms / max(1, bat_n), 2),
            "append_batch_gb_s": round(spec.layers * append_bytes(spec) /
                                       (bat_ms / max(1, bat_n) * 1e-3) / 1e9, 1),
            "steps": args.steps, "warmup": args.warmup,
            "note": "steady-state chunks (cache full); 30 independent layer caches, 5.0 GB"}


def moba_useful_flops(spec) -> float:
    n, m, c = spec.n_chunks, spec.n_bidir_chunks, spec.chunk_tokens
    pairs = (n * (n + 1) // 2 + n * (n - 1) // 2 + n + m * m) * c * c
    return 4.0 * pairs * spec.heads * spec.head_dim


def run_moba(args) -> dict:
    import torch
    from kv_cache_chunk_ring_b200 import build as _build
    from kv_cache_chunk_ring_b200 import kvcr
    _build.build()
    spec = wl.MOBA_8x6032
    if args.moba_chunk_tokens:                        # a smaller sequence of the same shape
        spec = dataclasses.replace(spec, name=f"moba_8chunks_x{args.moba_chunk_tokens}",
                                   chunk_tokens=args.moba_chunk_tokens)
    gen = torch.Generator(device="cuda").manual_seed(spec.seed)
    shape = (spec.seq_len, spec.heads, spec.head_dim)
    q, k, v = (_randn(shape, gen) for _ in range(3))
    o = torch.empty_like(q)

    def call():
        kvcr.moba_attention_fwd(q, k, v, spec.n_chunks, spec.chunk_tokens, spec.n_bidir_chunks, o)

    ms = _timed(call, args.steps, args.warmup)
    kvcr.kvcr_check_status()
    flops = moba_useful_flops(spec)
    peaks, kind = load_peaks()
    tf = flops / (ms * 1e-3) / 1e12
    return {"workload": spec.name, "ms_per_call": round(ms, 3), "useful_tflop": round(flops / 1e12, 3),
            "value": round(tf, 2), "unit": UNIT, "frac_of_peak": round(tf / peaks["bf16_tflops"], 4),
            "steps": args.steps, "warmup": args.warmup}


def run_moba_bwd(args) -> dict:
    """MoBA backward (dQ, dK, dV) over the 144768-token training sequence, from the
    forward's O and LSE; also the forward + backward step."""
    import torch
    from kv_cache_chunk_ring_b200 import build as _build
    from kv_cache_chunk_ring_b200 import kvcr
    _build.build()
    spec = wl.MOBA_8x6032
    if args.moba_chunk_tokens:                        # a smaller sequence of the same shape
        spec = dataclasses.replace(spec, name=f"moba_8chunks_x{args.moba_chunk_tokens}",
                                   chunk_tokens=args.moba_chunk_tokens)
    lay = (spec.n_chunks, spec.chunk_tokens, spec.n_bidir_chunks)
    gen = torch.Generator(device="cuda").manual_seed(spec.seed)
    shape = (spec.seq_len, spec.heads, spec.head_dim)
    q, k, v, do = (_randn(shape, gen) for _ in range(4))
    o = torch.empty_like(q)
    lse = torch.empty((spec.heads, spec.seq_len), dtype=torch.float32, device="cuda")
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = torch.empty(kvcr.moba_attention_bwd_workspace_bytes(*lay, spec.heads), dtype=torch.uint8,
                     device="cuda")
    kvcr.moba_attention_fwd(q, k, v, *lay, o, lse)

    def bwd():
        kvcr.moba_attention_bwd(q, k, v, o, do, lse, *lay, dq, dk, dv, workspace=ws)

    def fwd_bwd():
        kvcr.moba_attention_fwd(q, k, v, *lay, o, lse)
        bwd()

    ms = _timed(bwd, args.steps, args.warmup)
    ms_step = _timed(fwd_bwd, max(2, args.steps // 2), 1)
    kvcr.kvcr_check_status()
    kvcr.kvcr_trace_reset()
    kvcr.kvcr_trace_enable(True)
    bwd()
    torch.cuda.synchronize()
    kvcr.kvcr_trace_enable(False)
    kt = {name: kvcr.kvcr_trace_read(kid) for kid, name in kvcr.KERNEL_NAMES.items()}
    kvcr.kvcr_trace_reset()
    fwd_flops = moba_useful_flops(spec)
    flops = 2.5 * fwd_flops          # dV, dP, dQ, dK and the recomputed S: five products
    peaks, kind = load_peaks()
    tf = flops / (ms * 1e-3) / 1e12

    def kms(name):
        n, t = kt[name]
        return t / max(1, n)
    dkdv_ms, dq_ms = kms("moba_bwd_dkdv"), kms("moba_bwd_dq")
    return {"workload": spec.name + "_backward", "ms_per_call": round(ms, 3),
            "useful_tflop": round(flops / 1e12, 3), "value": round(tf, 2), "unit": UNIT,
            "frac_of_peak": round(tf / peaks["bf16_tflops"], 4),
            "kernels_ms": {"prep": round(kms("moba_bwd_prep"), 4), "dkdv": round(dkdv_ms, 3),
                           "dq": round(dq_ms, 3)},
            # executed tensor work: dK/dV kernel 4 products, dQ kernel 3 (S and dP recomputed)
            "executed_tflops": {"dkdv": round(2.0 * fwd_flops / (dkdv_ms * 1e-3) / 1e12, 1),
                                "dq": round(1.5 * fwd_flops / (dq_ms * 1e-3) / 1e12, 1)},
            "fwd_bwd_ms": round(ms_step, 3),
            "fwd_bwd_tflops": round(3.5 * fwd_flops / (ms_step * 1e-3) / 1e12, 2),
            "steps": args.steps, "warmup": args.warmup}


def run_dynwin(args) -> dict:
    """720p rollout, 6 anchors, window drawn per chunk from U{2..8}, plus cross-attention."""
    import torch
    from kv_cache_chunk_ring_b200 import build as _build
    from kv_cache_chunk_ring_b200 import kvcr
    _build.build()
    spec = wl.VIDEO_720P_DYN
    T, H, D, F = spec.tokens_per_frame, spec.heads, spec.head_dim, spec.chunk_frames
    sched = spec.window_schedule()
    self_c = kvcr.Cache(spec.sinks, spec.window, T, H, D, F, rope=spec.rope())
    cross_c = kvcr.Cache(1, 0, spec.text_env, H, D, 1, rope=None)
    gen = torch.Generator(device="cuda").manual_seed(spec.seed)
    pool = [tuple(_randn((spec.chunk_tokens, H, D), gen) for _ in range(3)) for _ in range(3)]
    env_k, env_v = _randn((spec.text_env, H, D), gen), _randn((spec.text_env, H, D), gen)
    loc = [(_randn((spec.text_local, H, D), gen), _randn((spec.text_local, H, D), gen))
           for _ in range(3)]
    cross_c.append(env_k, env_v, [0])
    o = torch.empty_like(pool[0][0])
    ox = torch.empty_like(pool[0][0])
    state = {"c": 0, "flops": 0.0}

    def chunk():
        c = state["c"]
        w = sched[c % len(sched)]
        self_c.evict(w)
        frames = list(range(c * F, (c + 1) * F))
        q, k, v = pool[c % 3]
        lk = (self_c.num_cached() + F) * T
        self_c.attention(q, k, v, frames, out=o)
        lq, lv = loc[c % 3]
        cross_c.attention(q, lq, lv, [c + 1], out=ox)
        self_c.append(k, v, frames)
        state["flops"] += 4.0 * spec.chunk_tokens * (lk + spec.text_env + spec.text_local) * H * D
        state["c"] = c + 1

    for _ in range(STEADY_CHUNK):
        chunk()
    for _ in range(args.warmup):
        chunk()
    torch.cuda.synchronize()
    state["flops"] = 0.0
    n = max(args.steps, len(sched) - state["c"])
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        chunk()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    return {"workload": spec.name, "ms_per_chunk": round(ms, 3), "chunks_timed": n,
            "value": round(state["flops"] / n / (ms * 1e-3) / 1e12, 2), "unit": UNIT,
            "note": "per chunk: evict(W_t), self-attention, cross-attention (512 text keys), append"}


def run_aux(args) -> dict:
    """832x464 steady-state chunk step with 4 auxiliary evidence frames: per chunk,
    kv_cache_set_aux (4 frames, K rotated at their positions), 4 denoising-step
    attention calls over 6 + 8 cached + 4 auxiliary + 4 current frames (33176 keys),
    append (which drops the auxiliary frames)."""
    import torch
    from kv_cache_chunk_ring_b200 import build as _build
    from kv_cache_chunk_ring_b200 import kvcr
    _build.build()
    spec, n_aux, steps = SPEC, 4, 4
    T, H, D, F = spec.tokens_per_frame, spec.heads, spec.head_dim, spec.chunk_frames
    cache = kvcr.Cache(spec.sinks, spec.window, T, H, D, F, rope=spec.rope(), aux_frames=n_aux)
    gen = torch.Generator(device="cuda").manual_seed(spec.seed)
    pool = [tuple(_randn((spec.chunk_tokens, H, D), gen) for _ in range(3)) for _ in range(3)]
    aux_k, aux_v = _randn((n_aux * T, H, D), gen), _randn((n_aux * T, H, D), gen)
    o = torch.empty_like(pool[0][0])
    state = {"c": 0}

    def chunk():
        c = state["c"]
        frames = list(range(c * F, (c + 1) * F))
        if c >= STEADY_CHUNK:
            cache.set_aux(aux_k, aux_v, [max(0, c * F - 8 + i) for i in range(n_aux)])
        for s in range(steps):
            q, k, v = pool[(c + s) % 3]
            cache.attention(q, k, v, frames, out=o)
        cache.append(k, v, frames)
        state["c"] = c + 1

    for _ in range(STEADY_CHUNK):
        chunk()
    ms = _timed(chunk, args.steps, args.warmup)
    kvcr.kvcr_trace_reset()
    kvcr.kvcr_trace_enable(True)
    chunk()
    torch.cuda.synchronize()
    kvcr.kvcr_trace_enable(False)
    kt = {name: kvcr.kvcr_trace_read(kid) for kid, name in kvcr.KERNEL_NAMES.items()}
    kvcr.kvcr_trace_reset()
    kvcr.kvcr_check_status()
    lk = (spec.sinks + spec.window + n_aux + F) * T
    call_flops = 4.0 * spec.chunk_tokens * lk * H * D
    attn_n, attn_ms = kt["chunk_attn"]
    aux_n, aux_ms = kt["set_aux"]
    peaks, kind = load_peaks()
    attn_call = attn_ms / max(1, attn_n)
    aux_bytes = 4.0 * n_aux * T * H * D * 2          # read and write K and V
    return {"workload": spec.name + "_aux4", "keys_per_call": lk,
            "ms_per_chunk": round(ms, 3), "calls_per_chunk": steps,
            "value": round(steps * call_flops / (ms * 1e-3) / 1e12, 2), "unit": UNIT,
            "attn_kernel_ms": round(attn_call, 4),
            "attn_tflops": round(call_flops / (attn_call * 1e-3) / 1e12, 1),
            "attn_frac_of_peak": round(call_flops / (attn_call * 1e-3) / 1e12 /
                                       peaks["bf16_tflops"], 4),
            "set_aux_us": round(1e3 * aux_ms / max(1, aux_n), 2),
            "set_aux_gb_s": round(aux_bytes / (aux_ms / max(1, aux_n) * 1e-3) / 1e9, 1),
            "steps": args.steps, "warmup": args.warmup}


def fp8_mixed_peak(bf16_peak: float) -> float:
    """Peak of the e4m3-QK^T attention's tensor work: half of the useful FLOPs (Q K^T)
    run at the e4m3 rate, nominally twice the bf16 rate, the other half (P V) at the
    bf16 rate, so 4 / (2 / 2 + 2 / 1) = 4/3 of the bf16 peak."""
    return bf16_peak * 4.0 / 3.0


def run_fp8(args) -> dict:
    """832x464 steady-state chunk step with the QK^T product in e4m3: stage (RoPE of Q
    and the chunk's K), e4m3 quantization of both, attention over 6 + 8 cached + 4
    current frames (27144 keys) reading the cache's e4m3 K copies, append (bf16 K/V
    and their e4m3 K copy)."""
    import torch
    from kv_cache_chunk_ring_b200 import build as _build
    from kv_cache_chunk_ring_b200 import kvcr
    _build.build()
    spec = SPEC
    T, H, D, F = spec.tokens_per_frame, spec.heads, spec.head_dim, spec.chunk_frames
    cache = kvcr.Cache(spec.sinks, spec.window, T, H, D, F, rope=spec.rope(), fp8_k=True)
    gen = torch.Generator(device="cuda").manual_seed(spec.seed)
    pool = [tuple(_randn((spec.chunk_tokens, H, D), gen) for _ in range(3)) for _ in range(3)]
    o = torch.empty_like(pool[0][0])
    state = {"c": 0}

    def step():
        c = state["c"]
        frames = list(range(c * F, (c + 1) * F))
        q, k, v = pool[c % 3]
        cache.attention(q, k, v, frames, out=o, fp8=True)
        cache.append(k, v, frames)
        state["c"] = c + 1

    for _ in range(STEADY_CHUNK):
        step()
    ms = _timed(step, args.steps, args.warmup)
    kvcr.kvcr_trace_reset()
    kvcr.kvcr_trace_enable(True)
    for _ in range(max(3, min(args.steps, 20))):
        step()
    torch.cuda.synchronize()
    kvcr.kvcr_trace_enable(False)
    kt = {name: kvcr.kvcr_trace_read(kid) for kid, name in kvcr.KERNEL_NAMES.items()}
    kvcr.kvcr_trace_reset()
    kvcr.kvcr_check_status()
    peaks, kind = load_peaks()
    flops = step_flops(spec)

    def avg(name):
        n, t = kt[name]
        return t / max(1, n)
    attn_ms = avg("chunk_attn_fp8")
    tf = flops / (attn_ms * 1e-3) / 1e12
    peak = fp8_mixed_peak(float(peaks["bf16_tflops"]))
    return {"workload": spec.name + "_qk_e4m3", "ms_per_step": round(ms, 4),
            "value": round(flops / (ms * 1e-3) / 1e12, 2), "unit": UNIT,
            "dtype": "e4m3 QK^T, bf16 P V, fp32 accumulate",
            "attn_kernel_ms": round(attn_ms, 4), "attn_tflops": round(tf, 1),
            "attn_frac_of_mixed_peak": round(tf / peak, 4), "mixed_peak_tflops": round(peak, 1),
            "attn_frac_of_bf16_peak": round(tf / float(peaks["bf16_tflops"]), 4),
            "peak_source": f"{kind} bf16_tflops x 4/3 (Q K^T at the nominal e4m3 rate, 2x bf16)",
            "kernels_ms": {k: round(avg(k), 5) for k, (n, _) in kt.items() if n},
            "steps": args.steps, "warmup": args.warmup}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-layers30", action="store_true",
                    help="leave out the 30-layer chunk figures of the default line")
    ap.add_argument("--shard", default="heads", choices=["heads", "layers"],
                    help="multi-GPU partition: heads of one layer cache per rank (strong "
                         "scaling) or one layer cache per rank (weak scaling)")
    ap.add_argument("--layers", type=int, default=0,
                    help="layers30: number of layer caches (default 30); fewer give a case "
                         "small enough for a full profiler capture")
    ap.add_argument("--moba-chunk-tokens", type=int, default=0,
                    help="moba, moba_bwd: tokens per chunk (default: the workload's 6032); a smaller "
                         "value gives a case small enough for a full profiler capture")
    ap.add_argument("--workload", default="chunk",
                    choices=["chunk", "layers30", "moba", "moba_bwd", "dynwin", "aux", "fp8"],
                    help="chunk: the 832x464 steady-state step (the bench line); the others "
                         "print single-GPU timings of the other workloads")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # start one rank per GPU through torch.distributed.run, with the same arguments
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
               f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1",
               f"--master-port={free_port()}", os.path.abspath(__file__)] + sys.argv[1:]
        sys.exit(subprocess.call(cmd))
    if world > 1 and args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but {world} ranks were started")

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)))
        return
    if args.workload != "chunk":
        fn = {"layers30": run_layers30, "moba": run_moba, "moba_bwd": run_moba_bwd,
              "dynwin": run_dynwin, "aux": run_aux, "fp8": run_fp8}[args.workload]
        if rank == 0:
            print(json.dumps(fn(args)))
        return

    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        out = run_ours(args, rank, world, dist)
        if rank == 0:
            if world == 1 and not args.no_layers30:
                # the 30-layer x 4-step chunk (each layer its own cache, 5 GB: no reuse of
                # one call's K/V by the next in L2), measured after the timed region
                l30 = run_layers30(argparse.Namespace(steps=max(3, min(args.steps, 10)),
                                                      warmup=3, layers=0), clocks=True)
                out.update({
                    "layers30_ms_per_chunk": l30["ms_per_chunk_batched_append"],
                    "layers30_ms_per_chunk_separate_appends": l30["ms_per_chunk"],
                    "layers30_ms_per_chunk_fused_last_step": l30["ms_per_chunk_fused_last_step"],
                    "layers30_attn_kernel_ms": l30["attn_kernel_ms"],
                    "layers30_attn_kernel_frac": l30["attn_kernel_frac"],
                    "layers30_attn_kernel_frac_sustained": l30["attn_kernel_frac_sustained"],
                    "layers30_append_gb_s": l30["append_batch_gb_s"],
                    "layers30_append_hbm_frac": l30["append_batch_hbm_frac"],
                    "layers30_append_separate_gb_s": l30["append_gb_s"],
                    "layers30_clocks": l30["clocks"],
                    "layers30_note": "30 layer caches x 4 denoising steps per chunk: 120 "
                                     "attention calls + one batched append of 30 caches "
                                     "(separate appends timed too); steady-state chunks",
                })
            if world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline()
            print(json.dumps(out))
    finally:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
