"""GPU parity at the full workload sizes, on sampled rows the fp64 oracle can compute:

* the 30-layer x 4-step rollout at 832x464 (each layer its own cache): layers 0 and 29,
  every call of all 10 chunks;
* the 720p rollout with a dynamic window and causal cross-attention (first 16 chunks);
* MoBA over the 144768-token training sequence with more sampled rows.
Inputs are streamed chunk by chunk (the same seeded draws feed both sides)."""
import math

import numpy as np
import pytest

from kv_cache_chunk_ring_b200 import workloads as wl
from oracle.attn import attention
from oracle.moba import MobaLayout, moba_attention_rows
from oracle.rollout import rollout
from tests.gpu_helpers import TOL_LSE, assert_close, gpu_rollout, oracle_and_gpu, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_chunk_ring_b200 import build
    build.build()


def _rows(L, n, seed, edge=32):
    return wl.sample_rows(L, n, seed, list(range(edge)) + list(range(L - edge, L)))


def _check(ref, got, what):
    worst = (0.0, 0.0)
    for n, (o, o_ref, l, l_ref) in enumerate(zip(got["outputs"], ref.outputs, got["lses"],
                                                 ref.lses)):
        ma, rr = assert_close(o, o_ref, f"{what} call {n}")
        assert np.abs(l - l_ref).max() <= TOL_LSE, f"{what} call {n}: lse"
        worst = (max(worst[0], ma), max(worst[1], rr))
    assert got["slot_maps"] == ref.slot_maps
    return worst


@pytest.mark.parametrize("layer", [0, 29])
def test_30layer_rollout_layer(layer):
    spec = wl.VIDEO_832x464_30L
    L = spec.chunk_tokens

    def rows_for(c, s):
        return _rows(L, 48, 5000 + 100 * layer + 10 * c + s)

    ref, got = oracle_and_gpu(wl.rollout_chunks(spec, layer),
                              lambda it: rollout(spec, it, rows_for=rows_for),
                              lambda it: gpu_rollout(spec, it, rows_for=rows_for))
    assert len(got["outputs"]) == spec.n_chunks * spec.steps
    worst = _check(ref, got, f"layer {layer}")
    print(f"30-layer rollout layer {layer}: worst max_abs={worst[0]:.3e} rel_rms={worst[1]:.3e}")


def test_720p_dynamic_window_and_cross_attention():
    """All 60 chunks of the 720p rollout: every window of the seeded U{2..8} schedule,
    the evicted and reused slots, 256 random plus the first and last 32 rows of every
    self-attention call, and every row of every cross-attention call."""
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    spec = wl.VIDEO_720P_DYN
    sched = spec.window_schedule()
    L = spec.chunk_tokens

    def rows_for(c, s):
        return _rows(L, 256, 7000 + c)

    ref, got = oracle_and_gpu(
        wl.rollout_chunks(spec),
        lambda it: rollout(spec, it, rows_for=rows_for, window_schedule=sched),
        lambda it: gpu_rollout(spec, it, rows_for=rows_for, window_schedule=sched))
    assert len(got["outputs"]) == spec.n_chunks == 60
    worst = _check(ref, got, "720p dynamic window")
    assert [a[0] for a in got["appended"]] == ref.appended_slots
    print(f"720p dynamic window, 60 chunks: worst max_abs={worst[0]:.3e} rel_rms={worst[1]:.3e}")

    cross = kvcr.Cache(1, 0, spec.text_env, spec.heads, spec.head_dim, 1, rope=None)
    scale = 1.0 / math.sqrt(spec.head_dim)
    worst = (0.0, 0.0)
    for item in wl.text_kv(spec):
        if item["chunk"] == 0:
            cross.append(to_dev(item["env_k"], "bf16"), to_dev(item["env_v"], "bf16"), [0])
        o, lse = cross.attention(to_dev(item["q"], "bf16"), to_dev(item["k"], "bf16"),
                                 to_dev(item["v"], "bf16"), [item["chunk"] + 1], want_lse=True)
        o_ref, l_ref = attention(item["q"], np.concatenate([item["env_k"], item["k"]]),
                                 np.concatenate([item["env_v"], item["v"]]), scale)
        ma, rr = assert_close(to_np(o), o_ref, f"cross chunk {item['chunk']}")
        assert np.abs(lse.cpu().numpy() - l_ref).max() <= TOL_LSE
        worst = (max(worst[0], ma), max(worst[1], rr))
    print(f"720p cross-attention, 60 chunks, all rows: worst max_abs={worst[0]:.3e} "
          f"rel_rms={worst[1]:.3e}")


def test_moba_full_size_more_rows():
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    spec = wl.MOBA_8x6032
    c, L = spec.chunk_tokens, spec.seq_len
    q, k, v = wl.moba_inputs(spec)
    qd, kd, vd = (to_dev(x, "bf16") for x in (q, k, v))
    o = torch.empty_like(qd)
    lse = torch.empty((spec.heads, L), dtype=torch.float32, device="cuda")
    kvcr.moba_attention_fwd(qd, kd, vd, spec.n_chunks, c, spec.n_bidir_chunks, o, lse)
    torch.cuda.synchronize()
    always = []
    for start in (0, 7 * c, 8 * c, 15 * c, 16 * c, L - c):   # C1, C8, N1, N8, B first / last chunk
        always += list(range(start, start + 128)) + list(range(start + c - 128, start + c))
    rows = wl.sample_rows(L, 1024, 1003, always)
    o_ref, l_ref = moba_attention_rows(q, k, v, MobaLayout(spec.n_chunks, c, spec.n_bidir_chunks),
                                       rows, 1 / math.sqrt(spec.head_dim))
    idx = torch.from_numpy(rows).cuda()
    ma, rr = assert_close(to_np(o.index_select(0, idx)), o_ref, "moba full")
    assert np.abs(lse.index_select(1, idx).cpu().numpy() - l_ref).max() <= TOL_LSE
    print(f"moba {rows.size} rows: max_abs={ma:.3e} rel_rms={rr:.3e}")
