"""Pins of the oracle's e4m3 quantization and the low-precision QK^T attention."""
import math

import numpy as np
import pytest

from oracle import fp8
from oracle.attn import attention


def test_code_table_from_the_format():
    vals = fp8.e4m3_values()
    assert vals[0] == 0.0 and vals[1] == 2.0 ** -9 and vals[7] == 7 * 2.0 ** -9
    assert vals[8] == 2.0 ** -6                         # smallest normal: exponent 1
    assert vals[0x38] == 1.0                            # exponent 7 (bias), mantissa 0
    assert vals[126] == 448.0 and np.isnan(vals[127]) and np.isnan(vals[255])
    assert vals[128 + 0x38] == -1.0
    finite = vals[:127]
    assert np.all(np.diff(finite) > 0)                  # codes 0..126 ascend


def test_every_finite_code_rounds_to_itself():
    vals = fp8.e4m3_values()
    finite = vals[~np.isnan(vals)]
    assert np.array_equal(fp8.e4m3_round(finite), finite)


def test_ties_go_to_the_even_mantissa():
    pos = fp8.e4m3_values()[:127]
    mids = (pos[:-1] + pos[1:]) / 2
    r = fp8.e4m3_round(mids)
    idx = np.searchsorted(pos, r)
    assert np.all(idx % 2 == 0)
    assert fp8.e4m3_round(1.0625) == 1.0 and fp8.e4m3_round(1.1875) == 1.25


def test_matches_torch_float8_below_saturation():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.1, 1, 30, 200)])
    x = x[np.abs(x) < 464].astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    assert np.array_equal(fp8.e4m3_round(x), ref)


def test_saturates_and_keeps_nan():
    r = fp8.e4m3_round(np.array([463.9, 464.0, 1e9, -1e9, np.nan]))
    assert list(r[:4]) == [448.0, 448.0, 448.0, -448.0] and np.isnan(r[4])


def test_relative_error_bound_in_the_normal_range():
    x = np.geomspace(2.0 ** -6, 440.0, 100000)
    r = fp8.e4m3_round(x)
    assert np.max(np.abs(r / x - 1)) <= 2.0 ** -4 + 1e-15


def test_block_quantization():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((300, 2, 64)).astype(np.float32)
    x[128:256, 1] = 0.0                                  # one all-zero block
    codes, scales = fp8.quantize_blocks(x)
    assert scales.shape == (3, 2) and scales[1, 1] == 0.0
    assert np.abs(codes).max() <= 448.0
    for b in range(3):
        for h in range(2):
            blk = codes[b * 128:(b + 1) * 128, h]
            if scales[b, h] > 0:
                assert np.abs(blk).max() == 448.0          # the amax element maps to the top code
    y = fp8.dequantize_blocks(codes, scales)
    err = np.abs(y - x)
    bound = np.repeat(scales.astype(np.float64), 128, axis=0)[:300][:, :, None]
    # half a step of the coarsest binade (2^-4 relative at 448) or a subnormal half-step
    assert np.all(err <= np.maximum(np.abs(x) * 2.0 ** -4, bound * 2.0 ** -10) + 1e-12)


def test_exactly_representable_blocks_give_plain_attention():
    """Blocks of e4m3 values whose amax is 448 have scale 1 and codes equal to the
    inputs, so the low-precision attention is the plain attention exactly."""
    rng = np.random.default_rng(2)
    pos = fp8.e4m3_values()[:127]
    def draw(shape):
        v = rng.choice(pos, size=shape) * rng.choice([-1.0, 1.0], size=shape)
        v[0::128, :, 0] = 448.0
        return v.astype(np.float32)
    q, k = draw((200, 2, 16)), draw((260, 2, 16))
    v = rng.standard_normal((260, 2, 16))
    o1, l1 = fp8.attention_fp8_qk(q, k, v, 1e-3)
    o2, l2 = attention(q, k, v, 1e-3)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_low_precision_attention_is_close_to_exact():
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((256, 2, 128)).astype(np.float32) for _ in range(3))
    o1, _ = fp8.attention_fp8_qk(q, k, v, 1 / math.sqrt(128))
    o2, _ = attention(q, k, v, 1 / math.sqrt(128))
    rel = np.linalg.norm(o1 - o2) / np.linalg.norm(o2)
    assert 1e-4 < rel < 0.1


# ------------------------------------------------------- rollout with e4m3 QK^T --

def test_round_bf16_matches_torch_and_ties_go_even():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(50000) * s for s in (1e-30, 1e-3, 1, 1e3)])
    x32 = x.astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).float().numpy().astype(np.float64)
    assert np.array_equal(fp8.round_bf16(x32), ref)
    # exact ties between neighbours at 1: 1 + 2^-8 -> 1, 1 + 3 * 2^-8 -> 1 + 2^-6
    assert fp8.round_bf16(1 + 2.0 ** -8) == 1.0
    assert fp8.round_bf16(1 + 3 * 2.0 ** -8) == 1 + 2.0 ** -6
    assert fp8.round_bf16(-(1 + 3 * 2.0 ** -8)) == -(1 + 2.0 ** -6)
    # an fp64 value just above a tie rounds up (no double rounding through fp32)
    assert fp8.round_bf16(1 + 2.0 ** -8 + 2.0 ** -40) == 1 + 2.0 ** -7


def _small_spec(**kw):
    from kv_cache_chunk_ring_b200 import workloads as wl
    base = dict(grid_h=8, grid_w=16, heads=2, head_dim=64, chunk_frames=2, sinks=1, window=2,
                n_chunks=3, seed=51)
    base.update(kw)
    return wl.shrink(wl.VIDEO_832x464, **base)


def test_fp8_rollout_first_chunk_is_fp8_attention_of_the_rotated_bf16_operands():
    from kv_cache_chunk_ring_b200 import workloads as wl
    from oracle.rollout import rollout
    from oracle.rope import rope3d, rope_positions
    spec = _small_spec(grid_h=5, grid_w=7)              # 35 tokens per frame: ragged blocks
    items = list(wl.rollout_chunks(spec))
    res = rollout(spec, items, qk_fp8=True)
    it = items[0]
    pairs = (spec.rope().pairs_t, spec.rope().pairs_h, spec.rope().pairs_w)
    t, h, w = rope_positions(it["frames"], spec.grid_h, spec.grid_w)
    qb = fp8.round_bf16(rope3d(it["q"], t, h, w, pairs))
    kb = fp8.round_bf16(rope3d(it["k"], t, h, w, pairs))
    o, lse = fp8.attention_fp8_qk(qb, kb, it["v"], 1 / math.sqrt(spec.head_dim))
    np.testing.assert_allclose(res.outputs[0], o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(res.lses[0], lse, rtol=0, atol=1e-13)


def test_fp8_rollout_quantizes_cached_keys_frame_by_frame():
    """Chunk 1 reads chunk 0's two frames from the cache (blocks of 128 tokens of each
    frame, 160 tokens = 128 + 32) and its own keys (blocks over the chunk's 320 tokens)."""
    from kv_cache_chunk_ring_b200 import workloads as wl
    from oracle.rollout import rollout
    from oracle.rope import rope3d, rope_positions
    spec = _small_spec(grid_h=10, grid_w=16)
    items = list(wl.rollout_chunks(spec))
    res = rollout(spec, items, qk_fp8=True)
    pairs = (spec.rope().pairs_t, spec.rope().pairs_h, spec.rope().pairs_w)
    T = spec.tokens_per_frame

    def rot(it, x):
        t, h, w = rope_positions(it["frames"], spec.grid_h, spec.grid_w)
        return rope3d(x, t, h, w, pairs)
    k0 = rot(items[0], items[0]["k"])
    keys = [fp8.fp8_operand(k0[:T]), fp8.fp8_operand(k0[T:]), fp8.fp8_operand(rot(items[1],
                                                                                 items[1]["k"]))]
    v = np.concatenate([items[0]["v"], items[1]["v"]])
    o, lse = attention(fp8.fp8_operand(rot(items[1], items[1]["q"])), np.concatenate(keys), v,
                       1 / math.sqrt(spec.head_dim))
    np.testing.assert_allclose(res.outputs[1], o, rtol=0, atol=1e-13)
    # quantizing the cached keys as one 320-token block sequence differs
    o_wrong, _ = attention(fp8.fp8_operand(rot(items[1], items[1]["q"])),
                           np.concatenate([fp8.fp8_operand(k0), keys[2]]), v,
                           1 / math.sqrt(spec.head_dim))
    assert np.abs(o_wrong - res.outputs[1]).max() > 1e-6


def test_fp8_rollout_of_representable_blocks_is_the_plain_rollout():
    """Without RoPE, inputs whose every 128-token block holds e4m3 values with one
    element at 448 quantize with scale 1 to themselves: the e4m3 rollout is exact."""
    from kv_cache_chunk_ring_b200 import workloads as wl
    from oracle.rollout import rollout
    spec = _small_spec(grid_h=8, grid_w=16)             # 128 tokens per frame
    pos = fp8.e4m3_values()[:127]
    rng = np.random.default_rng(4)
    items = []
    for it in wl.rollout_chunks(spec):
        d = dict(it)
        for x in ("q", "k"):
            a = rng.choice(pos[pos <= 8], size=it[x].shape) * rng.choice([-1, 1], size=it[x].shape)
            a[::128, :, 0] = 448.0
            d[x] = (a / 64.0 * 64.0)                     # exact e4m3 values
        items.append(d)
    plain = rollout(spec, items, use_rope=False)
    low = rollout(spec, items, use_rope=False, qk_fp8=True)
    for a, b in zip(plain.outputs, low.outputs):
        assert np.array_equal(a, b)


def test_fp8_rollout_error_against_exact_is_a_few_percent():
    """On N(0, 1) inputs the e4m3 QK^T moves O by a few percent (rel-RMS), which is why
    the low-precision kernel is held to the bf16 tolerance only against this oracle."""
    from kv_cache_chunk_ring_b200 import workloads as wl
    from oracle.rollout import rollout
    spec = _small_spec(head_dim=128, n_chunks=3)
    items = list(wl.rollout_chunks(spec))
    exact = rollout(spec, items)
    low = rollout(spec, items, qk_fp8=True)
    for a, b in zip(exact.outputs, low.outputs):
        rel = np.linalg.norm(a - b) / np.linalg.norm(a)
        assert 1e-3 < rel < 8e-2, rel


def test_input_draws_round_to_bf16_like_torch():
    """The seeded inputs are N(0, 1) float32 draws rounded to bf16 (nearest, ties to even);
    the shared generator's rounding agrees with torch's conversion, ties included."""
    torch = pytest.importorskip("torch")
    from kv_cache_chunk_ring_b200 import workloads as wl
    rng = np.random.default_rng(5)
    x = rng.standard_normal(200000).astype(np.float32) * np.float32(3.0)
    ties = (np.arange(1, 2000, dtype=np.uint32) << 16 | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, ties, -ties])
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(wl.round_to_bf16(x), ref)
