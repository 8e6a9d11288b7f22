"""GPU parity of the cache write (RoPE3D append) and chunk attention against the
fp64 oracle, through the C ABI."""
import math

import numpy as np
import pytest

from kv_cache_chunk_ring_b200 import workloads as wl
from oracle.attn import attention
from oracle.rollout import rollout
from oracle.rope import rope3d, rope_positions
from tests.gpu_helpers import (TOL_LSE, assert_close, gpu_rollout, oracle_and_gpu, to_dev, to_np,
                               errors)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_chunk_ring_b200 import build
    build.build()


def _compare_rollouts(spec, chunks, rows_for=None, use_rope=True, sched=None, tight=None):
    ref = rollout(spec, chunks, rows_for=rows_for, use_rope=use_rope, window_schedule=sched)
    got = gpu_rollout(spec, chunks, rows_for=rows_for, use_rope=use_rope, window_schedule=sched)
    worst = (0.0, 0.0)
    for n, (o, o_ref, l, l_ref) in enumerate(zip(got["outputs"], ref.outputs, got["lses"],
                                                 ref.lses)):
        ma, rr = assert_close(o, o_ref, f"call {n}")
        if tight is not None:
            assert ma <= tight, f"call {n}: max_abs {ma} > {tight}"
        assert np.abs(l - l_ref).max() <= TOL_LSE, f"call {n}: lse"
        worst = (max(worst[0], ma), max(worst[1], rr))
    assert got["slot_maps"] == ref.slot_maps
    assert [a[0] for a in got["appended"]] == ref.appended_slots
    return worst, got


def test_tiny_rollout_f32():
    """2 anchors + 2 window slots, 16 tokens per frame, fp32 end to end."""
    spec = wl.TINY_F32
    worst, _ = _compare_rollouts(spec, list(wl.rollout_chunks(spec)), tight=1e-4)
    assert worst[1] < 1e-5


@pytest.mark.parametrize("kw", [
    dict(grid_h=4, grid_w=4, heads=2, head_dim=128, chunk_frames=2, sinks=2, window=2, n_chunks=6),
    dict(grid_h=5, grid_w=7, heads=3, head_dim=64, chunk_frames=2, sinks=1, window=3, n_chunks=7),
    dict(grid_h=12, grid_w=11, heads=2, head_dim=128, chunk_frames=3, sinks=1, window=3, n_chunks=5),
    dict(grid_h=16, grid_w=8, heads=1, head_dim=128, chunk_frames=1, sinks=0, window=3, n_chunks=6),
    dict(grid_h=3, grid_w=5, heads=2, head_dim=128, chunk_frames=4, sinks=2, window=0, n_chunks=4),
    dict(grid_h=8, grid_w=16, heads=2, head_dim=64, chunk_frames=2, sinks=3, window=5, n_chunks=8),
], ids=["4x4-d128", "5x7-d64", "12x11-d128", "16x8-nosink", "3x5-nowindow", "8x16-d64"])
def test_bf16_rollouts_small(kw):
    spec = wl.shrink(wl.VIDEO_832x464, dtype="bf16", seed=7, **kw)
    _compare_rollouts(spec, list(wl.rollout_chunks(spec)))


@pytest.mark.parametrize("kw", [
    dict(grid_h=5, grid_w=7, heads=2, head_dim=64, chunk_frames=2, sinks=1, window=3, n_chunks=5),
    dict(grid_h=12, grid_w=11, heads=1, head_dim=128, chunk_frames=2, sinks=2, window=2, n_chunks=5),
])
def test_f32_rollouts_small(kw):
    spec = wl.shrink(wl.TINY_F32, seed=8, **kw)
    _compare_rollouts(spec, list(wl.rollout_chunks(spec)), tight=1e-4)


def test_multi_step_cache_read_unchanged():
    """Several denoising steps read the same cache; the last step's K/V are appended."""
    spec = wl.shrink(wl.VIDEO_832x464_30L, grid_h=6, grid_w=10, heads=2, n_chunks=5, layers=1,
                     steps=4, sinks=2, window=3)
    _compare_rollouts(spec, list(wl.rollout_chunks(spec)))


def test_832x464_rollout_40_chunks():
    """The whole 40-chunk 832x464 rollout (12 heads, d128, 1508 tokens/frame, 6 + 8 slots,
    4-frame chunks; frames up to 159, the window wrapping ~19 times): every row of the
    fill-up chunks 0-4 and of the last chunk 39; 1024 random rows plus the first 128 and
    last 16 rows of every other chunk.  Slot maps after every append, bit-exact."""
    spec = wl.VIDEO_832x464
    L = spec.chunk_tokens
    every_row = {0, 1, 2, 3, 4, spec.n_chunks - 1}

    def rows_for(c, s):
        if c in every_row:
            return np.arange(L)
        return wl.sample_rows(L, 1024, 1000 + c, list(range(128)) + list(range(L - 16, L)))

    ref, got = oracle_and_gpu(wl.rollout_chunks(spec),
                              lambda it: rollout(spec, it, rows_for=rows_for),
                              lambda it: gpu_rollout(spec, it, rows_for=rows_for))
    assert len(got["outputs"]) == spec.n_chunks
    worst = (0.0, 0.0)
    for n, (o, o_ref, l, l_ref) in enumerate(zip(got["outputs"], ref.outputs, got["lses"],
                                                 ref.lses)):
        ma, rr = assert_close(o, o_ref, f"chunk {n}")
        assert np.abs(l - l_ref).max() <= TOL_LSE, f"chunk {n}: lse"
        worst = (max(worst[0], ma), max(worst[1], rr))
    assert got["slot_maps"] == ref.slot_maps
    assert [a[0] for a in got["appended"]] == ref.appended_slots
    assert ref.n_keys[-1] == 27144
    print(f"832x464 40-chunk rollout: worst max_abs={worst[0]:.3e} rel_rms={worst[1]:.3e}")


def test_append_writes_rotated_k_and_exact_v():
    import torch
    from kv_cache_chunk_ring_b200.kvcr import Cache
    for dtype, D in (("bf16", 128), ("bf16", 64), ("f32", 64)):
        spec = wl.shrink(wl.VIDEO_832x464, grid_h=7, grid_w=9, heads=3, head_dim=D, dtype=dtype,
                         chunk_frames=3, sinks=2, window=3, n_chunks=4, seed=11)
        cache = Cache(spec.sinks, spec.window, spec.tokens_per_frame, spec.heads, D,
                      spec.chunk_frames, rope=spec.rope(), dtype=dtype)
        pairs = (spec.rope().pairs_t, spec.rope().pairs_h, spec.rope().pairs_w)
        T = spec.tokens_per_frame
        for item in wl.rollout_chunks(spec):
            frames = [f + 1000 for f in item["frames"]]     # large absolute frame index
            k, v = to_dev(item["k"], dtype), to_dev(item["v"], dtype)
            slots, _ = cache.append(k, v, frames)
            torch.cuda.synchronize()
            t, h, w = rope_positions(frames, spec.grid_h, spec.grid_w)
            k_ref = rope3d(item["k"], t, h, w, pairs)
            for n, s in enumerate(slots):
                if s < 0:
                    continue
                kg, vg = cache.slot_tensors(s)
                assert np.array_equal(to_np(vg), item["v"][n * T:(n + 1) * T].astype(np.float64))
                kr = k_ref[n * T:(n + 1) * T]
                diff = np.abs(to_np(kg) - kr)
                if dtype == "bf16":
                    # within one bf16 ulp of the exact rotation (8 significant bits)
                    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(kr), 1e-30))) - 7)
                    assert np.all(diff <= ulp + 1e-30), float((diff / ulp).max())
                else:
                    assert diff.max() <= 1e-5 * max(1.0, np.abs(kr).max())


def test_zero_queries_closed_form():
    """Q = 0: O is the mean of the visible V rows and LSE = ln(number of keys)."""
    import torch
    from kv_cache_chunk_ring_b200.kvcr import Cache
    spec = wl.shrink(wl.VIDEO_832x464, grid_h=10, grid_w=13, heads=2, n_chunks=4, sinks=1,
                     window=2, chunk_frames=2, seed=12)
    cache = Cache(spec.sinks, spec.window, spec.tokens_per_frame, spec.heads, spec.head_dim,
                  spec.chunk_frames, rope=spec.rope())
    vs = {}
    for item in wl.rollout_chunks(spec):
        q = torch.zeros(item["q"].shape, dtype=torch.bfloat16, device="cuda")
        k, v = to_dev(item["k"], "bf16"), to_dev(item["v"], "bf16")
        vis = [f for f in sorted(vs)]
        o, lse = cache.attention(q, k, v, item["frames"], want_lse=True)
        all_v = np.concatenate([vs[f] for f in vis] + [item["v"]]).astype(np.float64)
        mean = all_v.mean(axis=0)
        assert_close(to_np(o), np.broadcast_to(mean, o.shape), "mean of V")
        np.testing.assert_allclose(lse.cpu().numpy(), math.log(all_v.shape[0]), atol=1e-3)
        slots, ev = cache.append(k, v, item["frames"])
        T = spec.tokens_per_frame
        for n, f in enumerate(item["frames"]):
            vs[f] = item["v"][n * T:(n + 1) * T]
        for f in ev:
            vs.pop(f, None)


def test_deterministic_and_future_independent():
    """Two identical calls give bit-identical outputs; appending later chunks never
    changes an earlier chunk's output (it was computed before)."""
    import torch
    from kv_cache_chunk_ring_b200.kvcr import Cache
    spec = wl.shrink(wl.VIDEO_832x464, grid_h=9, grid_w=17, heads=2, n_chunks=3, seed=13)
    items = list(wl.rollout_chunks(spec))
    cache = Cache(spec.sinks, spec.window, spec.tokens_per_frame, spec.heads, spec.head_dim,
                  spec.chunk_frames, rope=spec.rope())
    for item in items[:2]:
        q, k, v = (to_dev(item[x], "bf16") for x in ("q", "k", "v"))
        o1, l1 = cache.attention(q, k, v, item["frames"], want_lse=True)
        o2, l2 = cache.attention(q, k, v, item["frames"], want_lse=True)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        cache.append(k, v, item["frames"])


def test_cross_attention_no_rope():
    """Causal chunk-wise cross-attention: the chunk's queries read the shared env
    prompt (an anchor slot of a RoPE-free cache) plus their own local prompt."""
    import torch
    from kv_cache_chunk_ring_b200.kvcr import Cache
    spec = wl.shrink(wl.VIDEO_720P_DYN, grid_h=9, grid_w=16, n_chunks=3, heads=4)
    cache = Cache(1, 0, spec.text_env, spec.heads, spec.head_dim, 1, rope=None)
    for item in wl.text_kv(spec):
        if item["chunk"] == 0:
            cache.append(to_dev(item["env_k"], "bf16"), to_dev(item["env_v"], "bf16"), [0])
        q = to_dev(item["q"], "bf16")
        o, lse = cache.attention(q, to_dev(item["k"], "bf16"), to_dev(item["v"], "bf16"),
                                 [item["chunk"] + 1], want_lse=True)
        kk = np.concatenate([item["env_k"], item["k"]])
        vv = np.concatenate([item["env_v"], item["v"]])
        o_ref, l_ref = attention(item["q"], kk, vv, 1 / math.sqrt(spec.head_dim))
        assert_close(to_np(o), o_ref, f"cross chunk {item['chunk']}")
        assert np.abs(lse.cpu().numpy() - l_ref).max() <= TOL_LSE


def test_dynamic_window_rollout():
    spec = wl.shrink(wl.VIDEO_720P_DYN, grid_h=9, grid_w=16, heads=4, n_chunks=14)
    sched = spec.window_schedule()
    _compare_rollouts(spec, list(wl.rollout_chunks(spec)), sched=sched)


def test_device_status_clean():
    from kv_cache_chunk_ring_b200 import kvcr
    kvcr.kvcr_check_status()
