"""Helpers shared by the GPU parity tests: device transfer, error metrics, and
running a rollout through the C ABI in the same order as the oracle rollout."""
from __future__ import annotations

import math
from typing import Callable, List, Optional

import numpy as np

# Tolerances on attention outputs against the fp64 oracle, per call:
# max |O - O*| <= 2e-2 and ||O - O*||_2 / ||O*||_2 <= 5e-3 (bf16 inputs, fp32 accumulation).
TOL_MAX_ABS = 2e-2
TOL_REL_RMS = 5e-3
# LSE is an fp32 log-sum-exp of bf16-rounded scores: an absolute bound.
TOL_LSE = 2e-2


def torch_dtype(dtype: str):
    import torch
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def to_dev(x: np.ndarray, dtype: str):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        device="cuda", dtype=torch_dtype(dtype))


def to_np(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def errors(got: np.ndarray, ref: np.ndarray):
    d = got - ref
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    nrm = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(d) / nrm) if nrm > 0 else float(np.linalg.norm(d))
    return max_abs, rel


def assert_close(got, ref, what: str = "", max_abs=TOL_MAX_ABS, rel_rms=TOL_REL_RMS):
    ma, rr = errors(got, ref)
    assert ma <= max_abs and rr <= rel_rms, f"{what}: max_abs={ma:.3e} rel_rms={rr:.3e}"
    return ma, rr


def tee(items, maxsize: int = 2):
    """Two iterators over one pass of ``items`` (each item produced once), for an oracle
    rollout running in a thread beside the GPU rollout; at most ``maxsize`` items wait
    in either queue, so memory stays bounded."""
    import queue
    import threading
    end = object()
    qs = (queue.Queue(maxsize), queue.Queue(maxsize))

    def produce():
        for x in items:
            for q in qs:
                q.put(x)
        for q in qs:
            q.put(end)

    threading.Thread(target=produce, daemon=True).start()

    def drain(q):
        while True:
            x = q.get()
            if x is end:
                return
            yield x
    return drain(qs[0]), drain(qs[1])


def oracle_and_gpu(items, oracle_fn, gpu_fn):
    """Run ``oracle_fn(iterator)`` in a thread and ``gpu_fn(iterator)`` here over one pass of
    ``items``; returns (oracle result, gpu result)."""
    import threading
    a, b = tee(items)
    box = {}

    def run():
        try:
            box["ref"] = oracle_fn(a)
        except BaseException as e:  # re-raised below
            box["err"] = e
            for _ in a:             # keep the producer from blocking
                pass
    th = threading.Thread(target=run)
    th.start()
    try:
        got = gpu_fn(b)
    finally:
        for _ in b:
            pass
        th.join()
    if "err" in box:
        raise box["err"]
    return box["ref"], got


def rope_of(spec):
    return spec.rope()


def gpu_rollout(spec, chunks, rows_for: Optional[Callable] = None, use_rope: bool = True,
                window_schedule: Optional[List[int]] = None, aux_for: Optional[Callable] = None,
                aux_frames: int = 0, finalize: bool = False):
    """Run the rollout through the C ABI.  Returns dict of per-call outputs (rows
    selected by rows_for, numpy fp64), LSEs, slot maps after each append, and the
    Cache (for read-back).  ``aux_for(chunk)`` -> None or (k, v, positions) sets the
    chunk's auxiliary frames before its first step (cache built with
    ``aux_frames`` auxiliary slots).  ``finalize``: each chunk's last step is one
    chunk_attention_fwd_finalize call (attention and append in one pass)."""
    import torch
    from kv_cache_chunk_ring_b200.kvcr import Cache, kv_cache_last_append
    cap = spec.window if window_schedule is None else max(spec.window, max(window_schedule))
    cache = Cache(spec.sinks, cap, spec.tokens_per_frame, spec.heads, spec.head_dim,
                  spec.chunk_frames, rope=spec.rope() if use_rope else None, dtype=spec.dtype,
                  aux_frames=aux_frames, fused_finalize=finalize)
    out = dict(outputs=[], lses=[], slot_maps=[], appended=[], cache=cache)
    for item in chunks:
        c, s, frames = item["chunk"], item["step"], item["frames"]
        if s == 0 and window_schedule is not None:
            cache.evict(window_schedule[c])
        if s == 0 and aux_for is not None:
            aux = aux_for(c)
            if aux is not None:
                cache.set_aux(to_dev(aux[0], spec.dtype), to_dev(aux[1], spec.dtype), aux[2])
        q = to_dev(item["q"], spec.dtype)
        k = to_dev(item["k"], spec.dtype)
        v = to_dev(item["v"], spec.dtype)
        last = s == spec.steps - 1
        if finalize and last:
            o, lse = cache.attention_finalize(q, k, v, frames, want_lse=True)
        else:
            o, lse = cache.attention(q, k, v, frames, want_lse=True)
        rows = np.arange(q.shape[0]) if rows_for is None else np.asarray(rows_for(c, s))
        idx = torch.from_numpy(rows).cuda()
        out["outputs"].append(to_np(o.index_select(0, idx)))
        out["lses"].append(lse.index_select(1, idx).cpu().numpy().astype(np.float64))
        if last:
            if finalize:
                out["appended"].append(kv_cache_last_append(cache.handle, len(frames)))
            else:
                out["appended"].append(cache.append(k, v, frames))
            out["slot_maps"].append(cache.slot_map())
    torch.cuda.synchronize()
    return out


def scale_of(spec) -> float:
    return 1.0 / math.sqrt(spec.head_dim)
