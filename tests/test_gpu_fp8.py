"""GPU parity of the e4m3 QK^T chunk attention (chunk_attention_fwd_fp8) and of the
e4m3 K copies the cache keeps, against the oracle's quantizing rollout.

The oracle quantizes exactly what the kernels quantize: RoPE'd Q and K rounded to
bf16, blocks of 128 tokens of each cached / auxiliary frame and of the current
chunk, amax / 448 scales and e4m3 codes in fp32 (oracle/fp8.py).  Against it the
kernel is held to the bf16 tolerance (max-abs 2e-2, rel-RMS 5e-3): what remains is
the rounding of P and O to bf16 and fp32 accumulation order.  Against the exact
(unquantized) oracle it is held to a looser bound, 8e-2 max-abs and 6e-2 rel-RMS:
e4m3 codes carry 3 mantissa bits, which moves O by about 4 % rel-RMS on N(0, 1)
inputs.
"""
import math

import numpy as np
import pytest

from kv_cache_chunk_ring_b200 import workloads as wl
from oracle import fp8
from oracle.rollout import rollout
from oracle.rope import rope3d, rope_positions
from tests.gpu_helpers import TOL_LSE, assert_close, to_dev, to_np

pytestmark = pytest.mark.gpu

EXACT_MAX_ABS = 8e-2
EXACT_REL_RMS = 6e-2


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_chunk_ring_b200 import build
    build.build()


def _gpu_rollout_fp8(spec, chunks, rows_for=None, use_rope=True, aux_for=None, aux_frames=0,
                     window_schedule=None):
    import torch
    from kv_cache_chunk_ring_b200.kvcr import Cache
    cap = spec.window if window_schedule is None else max(spec.window, max(window_schedule))
    cache = Cache(spec.sinks, cap, spec.tokens_per_frame, spec.heads, spec.head_dim,
                  spec.chunk_frames, rope=spec.rope() if use_rope else None, aux_frames=aux_frames,
                  fp8_k=True)
    out = dict(outputs=[], lses=[], slot_maps=[], cache=cache)
    for item in chunks:
        c, s, frames = item["chunk"], item["step"], item["frames"]
        if s == 0 and window_schedule is not None:
            cache.evict(window_schedule[c])
        if s == 0 and aux_for is not None:
            aux = aux_for(c)
            if aux is not None:
                cache.set_aux(to_dev(aux[0], "bf16"), to_dev(aux[1], "bf16"), aux[2])
        q, k, v = (to_dev(item[x], "bf16") for x in ("q", "k", "v"))
        o, lse = cache.attention(q, k, v, frames, want_lse=True, fp8=True)
        rows = np.arange(q.shape[0]) if rows_for is None else np.asarray(rows_for(c, s))
        idx = torch.from_numpy(rows).cuda()
        out["outputs"].append(to_np(o.index_select(0, idx)))
        out["lses"].append(lse.index_select(1, idx).cpu().numpy().astype(np.float64))
        if s == spec.steps - 1:
            cache.append(k, v, frames)
            out["slot_maps"].append(cache.slot_map())
    torch.cuda.synchronize()
    return out


def _compare(spec, rows_for=None, use_rope=True, aux_for=None, aux_frames=0, sched=None,
             exact_too=True):
    kw = dict(rows_for=rows_for, use_rope=use_rope, aux_for=aux_for, window_schedule=sched)
    ref = rollout(spec, wl.rollout_chunks(spec), qk_fp8=True, **kw)
    got = _gpu_rollout_fp8(spec, wl.rollout_chunks(spec), rows_for=rows_for, use_rope=use_rope,
                           aux_for=aux_for, aux_frames=aux_frames, window_schedule=sched)
    exact = rollout(spec, wl.rollout_chunks(spec), **kw) if exact_too else None
    worst, worst_exact = (0.0, 0.0), (0.0, 0.0)
    for n, (o, o_ref, l, l_ref) in enumerate(zip(got["outputs"], ref.outputs, got["lses"],
                                                 ref.lses)):
        ma, rr = assert_close(o, o_ref, f"call {n} vs quantizing oracle")
        assert np.abs(l - l_ref).max() <= TOL_LSE, f"call {n}: lse"
        worst = (max(worst[0], ma), max(worst[1], rr))
        if exact is not None:
            ma, rr = assert_close(o, exact.outputs[n], f"call {n} vs exact oracle",
                                  max_abs=EXACT_MAX_ABS, rel_rms=EXACT_REL_RMS)
            worst_exact = (max(worst_exact[0], ma), max(worst_exact[1], rr))
    assert got["slot_maps"] == ref.slot_maps
    return worst, worst_exact, got


@pytest.mark.parametrize("kw", [
    dict(grid_h=4, grid_w=4, heads=2, chunk_frames=2, sinks=2, window=2, n_chunks=6),
    dict(grid_h=12, grid_w=11, heads=2, chunk_frames=3, sinks=1, window=3, n_chunks=5),
    dict(grid_h=16, grid_w=8, heads=1, chunk_frames=1, sinks=0, window=3, n_chunks=6),
    dict(grid_h=3, grid_w=5, heads=2, chunk_frames=4, sinks=2, window=0, n_chunks=4),
    dict(grid_h=10, grid_w=26, heads=3, chunk_frames=2, sinks=2, window=4, n_chunks=6),
], ids=["4x4", "12x11-ragged", "16x8-nosink", "3x5-nowindow", "10x26"])
def test_fp8_rollouts_small(kw):
    spec = wl.shrink(wl.VIDEO_832x464, dtype="bf16", seed=17, **kw)
    worst, worst_exact, _ = _compare(spec)
    print(f"fp8 {kw}: vs quantizing {worst}, vs exact {worst_exact}")


def test_fp8_multi_step_and_aux_frames():
    spec = wl.shrink(wl.VIDEO_832x464_30L, grid_h=6, grid_w=10, heads=2, n_chunks=4, layers=1,
                     steps=3, sinks=2, window=3, seed=18)
    aux = {c: wl.aux_frames(spec, c, 2) for c in range(spec.n_chunks)}
    _compare(spec, aux_for=lambda c: aux[c] if c >= 1 else None, aux_frames=2)


def test_fp8_dynamic_window():
    spec = wl.shrink(wl.VIDEO_720P_DYN, grid_h=9, grid_w=16, heads=2, n_chunks=10)
    _compare(spec, sched=spec.window_schedule())


def test_fp8_832x464_rollout_sampled_rows():
    """Full 832x464 shapes over the fill-up chunks and the first steady-state chunks."""
    spec = wl.shrink(wl.VIDEO_832x464, n_chunks=6)
    L = spec.chunk_tokens

    def rows_for(c, s):
        return wl.sample_rows(L, 384, 1100 + c, list(range(128)) + list(range(L - 16, L)))

    worst, worst_exact, _ = _compare(spec, rows_for=rows_for)
    print(f"fp8 832x464: worst vs quantizing oracle max_abs={worst[0]:.3e} "
          f"rel_rms={worst[1]:.3e}; vs exact max_abs={worst_exact[0]:.3e} "
          f"rel_rms={worst_exact[1]:.3e}")


def test_fp8_cross_attention_without_rope():
    """A RoPE-free cache (env prompt as its anchor); the queries are quantized as given."""
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    spec = wl.shrink(wl.VIDEO_720P_DYN, grid_h=4, grid_w=8, n_chunks=3, heads=4)
    n_q = 2 * spec.text_local                        # two query blocks per call
    cache = kvcr.Cache(1, 0, spec.text_env, spec.heads, spec.head_dim, 2, rope=None, fp8_k=True)
    scale = 1 / math.sqrt(spec.head_dim)
    for item in wl.text_kv(spec):
        if item["chunk"] == 0:
            cache.append(to_dev(item["env_k"], "bf16"), to_dev(item["env_v"], "bf16"), [0])
        q = item["q"][:n_q]
        o, lse = cache.attention(to_dev(q, "bf16"), to_dev(item["k"], "bf16"),
                                 to_dev(item["v"], "bf16"), [item["chunk"] + 1], want_lse=True,
                                 fp8=True)
        keys = np.concatenate([fp8.fp8_operand(item["env_k"]), fp8.fp8_operand(item["k"])])
        from oracle.attn import attention
        o_ref, l_ref = attention(fp8.fp8_operand(q), keys,
                                 np.concatenate([item["env_v"], item["v"]]), scale)
        assert_close(to_np(o), o_ref, f"fp8 cross chunk {item['chunk']}")
        assert np.abs(lse.cpu().numpy() - l_ref).max() <= TOL_LSE
    with pytest.raises(kvcr.KvcrError) as e:          # more queries than the staging holds
        big = torch.zeros((2 * spec.text_env + 1, spec.heads, spec.head_dim),
                          dtype=torch.bfloat16, device="cuda")
        kv = torch.zeros((spec.text_env, spec.heads, spec.head_dim), dtype=torch.bfloat16,
                         device="cuda")
        cache.attention(big, kv, kv, [9], fp8=True)
    assert e.value.code == kvcr.KVCR_ESHAPE


def _codes_to_values(codes):
    return fp8.e4m3_values()[codes.cpu().numpy().astype(np.int64)]


def test_cache_e4m3_copies_bit_exact_without_rope():
    """Without RoPE the cache holds K as given: the e4m3 codes and scales of every
    block equal the oracle's, bit for bit (both take the same fp32 steps)."""
    import torch
    from kv_cache_chunk_ring_b200.kvcr import Cache
    spec = wl.shrink(wl.VIDEO_832x464, grid_h=10, grid_w=30, heads=3, chunk_frames=2, sinks=1,
                     window=2, n_chunks=3, seed=19)
    cache = Cache(spec.sinks, spec.window, spec.tokens_per_frame, spec.heads, spec.head_dim,
                  spec.chunk_frames, rope=None, fp8_k=True)
    T = spec.tokens_per_frame
    items = list(wl.rollout_chunks(spec))
    for it in items:
        k = it["k"].copy()
        k[:128, 0, :] = 0.0                           # one all-zero block: zero codes and scale
        k[5, 1, 7] = 32768.0                          # a large element: the rest of its block
        slots, _ = cache.append(to_dev(k, "bf16"), to_dev(it["v"], "bf16"), it["frames"])
        torch.cuda.synchronize()
        smap = cache.slot_map()
        for n, sl in enumerate(slots):
            if sl < 0 or smap[sl] != it["frames"][n]:
                continue                            # evicted again within this append
            codes, scales = cache.slot_tensors_fp8(sl)
            ref_codes, ref_scales = fp8.quantize_blocks(k[n * T:(n + 1) * T])
            assert np.array_equal(scales.cpu().numpy(), ref_scales)
            assert np.array_equal(_codes_to_values(codes), ref_codes)


def test_cache_e4m3_copies_with_rope():
    """With RoPE the kernel rotates in fp32 and the oracle in fp64, so a rotated value
    can land on the other side of a rounding boundary: codes then differ by one step.
    Everything else is identical."""
    import torch
    from kv_cache_chunk_ring_b200.kvcr import Cache
    spec = wl.shrink(wl.VIDEO_832x464, n_chunks=2, sinks=2, window=2, heads=4, seed=20)
    cache = Cache(spec.sinks, spec.window, spec.tokens_per_frame, spec.heads, spec.head_dim,
                  spec.chunk_frames, rope=spec.rope(), fp8_k=True)
    pairs = (spec.rope().pairs_t, spec.rope().pairs_h, spec.rope().pairs_w)
    T = spec.tokens_per_frame
    vals = fp8.e4m3_values()
    n_diff = n_all = 0
    for it in wl.rollout_chunks(spec):
        slots, _ = cache.append(to_dev(it["k"], "bf16"), to_dev(it["v"], "bf16"), it["frames"])
        torch.cuda.synchronize()
        t, h, w = rope_positions(it["frames"], spec.grid_h, spec.grid_w)
        kr = fp8.round_bf16(rope3d(it["k"], t, h, w, pairs))
        smap = cache.slot_map()
        for n, sl in enumerate(slots):
            if sl < 0 or smap[sl] != it["frames"][n]:
                continue                            # evicted again within this append
            codes, scales = cache.slot_tensors_fp8(sl)
            ref_codes, ref_scales = fp8.quantize_blocks(kr[n * T:(n + 1) * T])
            np.testing.assert_allclose(scales.cpu().numpy(), ref_scales, rtol=2.0 ** -7, atol=0)
            got = codes.cpu().numpy().astype(np.int64)
            mag = np.searchsorted(vals[:127], np.abs(ref_codes))     # oracle's magnitude code
            neg = np.signbit(ref_codes) & (mag > 0)
            g_neg = (got >= 128) & ((got & 127) > 0)
            same = ((got & 127) == mag) & (g_neg == neg)
            n_diff += int((~same).sum())
            n_all += got.size
            # a differing code is a neighbour of the oracle's (same sign, one step)
            assert np.all(np.abs((got & 127) - mag)[~same] <= 1)
            assert np.all((g_neg == neg) | ((got & 127) == 0) | (mag == 0))
    assert n_diff <= 1e-4 * n_all, (n_diff, n_all)
    print(f"e4m3 K copies with RoPE: {n_diff} of {n_all} codes one step off")


def test_fp8_needs_an_fp8_cache_and_is_deterministic():
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    spec = wl.shrink(wl.VIDEO_832x464, grid_h=9, grid_w=17, heads=2, n_chunks=2, seed=21)
    items = list(wl.rollout_chunks(spec))
    plain = kvcr.Cache(spec.sinks, spec.window, spec.tokens_per_frame, spec.heads, spec.head_dim,
                       spec.chunk_frames, rope=spec.rope())
    q, k, v = (to_dev(items[0][x], "bf16") for x in ("q", "k", "v"))
    with pytest.raises(kvcr.KvcrError) as e:
        plain.attention(q, k, v, items[0]["frames"], fp8=True)
    assert e.value.code == kvcr.KVCR_ESTATE
    c8 = kvcr.Cache(spec.sinks, spec.window, spec.tokens_per_frame, spec.heads, spec.head_dim,
                    spec.chunk_frames, rope=spec.rope(), fp8_k=True)
    for it in items:
        q, k, v = (to_dev(it[x], "bf16") for x in ("q", "k", "v"))
        o1, l1 = c8.attention(q, k, v, it["frames"], want_lse=True, fp8=True)
        o2, l2 = c8.attention(q, k, v, it["frames"], want_lse=True, fp8=True)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        c8.append(k, v, it["frames"])
    kvcr.kvcr_check_status()


def test_fp8_batched_append_writes_the_same_copies():
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    spec = wl.shrink(wl.VIDEO_832x464, grid_h=7, grid_w=20, heads=2, n_chunks=3, seed=22)
    mk = lambda: kvcr.Cache(spec.sinks, spec.window, spec.tokens_per_frame, spec.heads,  # noqa
                            spec.head_dim, spec.chunk_frames, rope=spec.rope(), fp8_k=True)
    a, b, single = mk(), mk(), mk()
    for it in wl.rollout_chunks(spec):
        k, v = to_dev(it["k"], "bf16"), to_dev(it["v"], "bf16")
        kvcr.append_batch([a, b], [k, k], [v, v], it["frames"])
        single.append(k, v, it["frames"])
    torch.cuda.synchronize()
    assert a.slot_map() == b.slot_map() == single.slot_map()
    for slot, frame in enumerate(single.slot_map()):
        if frame < 0:
            continue                                # never written: nothing to compare
        for c in (a, b):
            for x, y in zip(c.slot_tensors_fp8(slot), single.slot_tensors_fp8(slot)):
                assert torch.equal(x, y)
