"""GPU parity of chunk_attention_fwd_finalize: a chunk's last step as one call that
attends and appends, writing the chunk's rotated K and its V once (into spare slots)
and making them cached frames by relabelling.  Against the fp64 oracle (outputs at the
bf16 tolerance, slot maps and appended slots bit-exact), and against the same rollout
run with separate attention and append calls (every slot's K and V bit-identical)."""
import numpy as np
import pytest

from kv_cache_chunk_ring_b200 import workloads as wl
from oracle.rollout import rollout
from tests.gpu_helpers import TOL_LSE, assert_close, gpu_rollout

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_chunk_ring_b200 import build
    build.build()


def _run(spec, sched=None, aux=None, aux_frames=0, rows_for=None):
    import torch
    kw = dict(rows_for=rows_for, window_schedule=sched)
    aux_for = (lambda c: aux.get(c)) if aux is not None else None
    ref = rollout(spec, wl.rollout_chunks(spec), aux_for=aux_for, **kw)
    fused = gpu_rollout(spec, wl.rollout_chunks(spec), aux_for=aux_for, aux_frames=aux_frames,
                        finalize=True, **kw)
    plain = gpu_rollout(spec, wl.rollout_chunks(spec), aux_for=aux_for, aux_frames=aux_frames,
                        **kw)
    worst = (0.0, 0.0)
    for n, (o, o_ref, l, l_ref) in enumerate(zip(fused["outputs"], ref.outputs, fused["lses"],
                                                 ref.lses)):
        ma, rr = assert_close(o, o_ref, f"call {n}")
        assert np.abs(l - l_ref).max() <= TOL_LSE, f"call {n}: lse"
        worst = (max(worst[0], ma), max(worst[1], rr))
    assert fused["slot_maps"] == ref.slot_maps == plain["slot_maps"]
    assert [a[0] for a in fused["appended"]] == ref.appended_slots
    assert [a[1] for a in fused["appended"]] == [a[1] for a in plain["appended"]]
    # what the cache holds is what the separate append wrote, bit for bit
    for slot in range(spec.sinks + (spec.window if sched is None else max(spec.window,
                                                                            max(sched)))):
        if fused["slot_maps"][-1][slot] < 0:
            continue
        for a, b in zip(fused["cache"].slot_tensors(slot), plain["cache"].slot_tensors(slot)):
            assert torch.equal(a, b), slot
    return worst


@pytest.mark.parametrize("kw", [
    dict(grid_h=4, grid_w=4, heads=2, head_dim=128, chunk_frames=2, sinks=2, window=2, n_chunks=7),
    dict(grid_h=5, grid_w=7, heads=3, head_dim=64, chunk_frames=2, sinks=1, window=3, n_chunks=7),
    dict(grid_h=12, grid_w=11, heads=2, head_dim=128, chunk_frames=3, sinks=1, window=3, n_chunks=6),
    dict(grid_h=16, grid_w=8, heads=1, head_dim=128, chunk_frames=1, sinks=0, window=3, n_chunks=7),
    dict(grid_h=3, grid_w=5, heads=2, head_dim=128, chunk_frames=4, sinks=2, window=0, n_chunks=4),
    dict(grid_h=2, grid_w=4, heads=2, head_dim=128, chunk_frames=4, sinks=1, window=2, n_chunks=5),
], ids=["4x4", "5x7-d64", "12x11", "16x8-nosink", "3x5-nowindow", "evict-within-chunk"])
def test_finalize_rollouts(kw):
    spec = wl.shrink(wl.VIDEO_832x464, dtype="bf16", seed=23, **kw)
    _run(spec)


def test_finalize_multi_step_with_aux_frames():
    spec = wl.shrink(wl.VIDEO_832x464_30L, grid_h=6, grid_w=10, heads=2, n_chunks=5, layers=1,
                     steps=3, sinks=2, window=3, seed=24)
    aux = {c: wl.aux_frames(spec, c, 2) for c in range(1, spec.n_chunks)}
    _run(spec, aux=aux, aux_frames=2)


def test_finalize_dynamic_window():
    spec = wl.shrink(wl.VIDEO_720P_DYN, grid_h=9, grid_w=16, heads=2, n_chunks=12)
    _run(spec, sched=spec.window_schedule())


def test_finalize_832x464_rollout_sampled_rows():
    spec = wl.shrink(wl.VIDEO_832x464, n_chunks=7)
    L = spec.chunk_tokens

    def rows_for(c, s):
        return wl.sample_rows(L, 256, 1200 + c, list(range(64)) + list(range(L - 16, L)))

    worst = _run(spec, rows_for=rows_for)
    print(f"fused finalize 832x464: worst max_abs={worst[0]:.3e} rel_rms={worst[1]:.3e}")
