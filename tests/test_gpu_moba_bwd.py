"""GPU parity of the MoBA attention backward (dQ, dK, dV) against the fp64 oracle.

The GPU path is the training step as a user runs it: moba_attention_fwd on the
device, then moba_attention_bwd from its O and LSE.  The oracle recomputes
everything from Q, K, V, dO in fp64.

Tolerance (per tensor, against the oracle): max |g - g*| <= 1e-2 * max |g*| and
||g - g*||_2 <= 1e-2 * ||g*||_2.  Sources of error: bf16 rounding of the outputs
(2^-9 relative), of P and dS as tensor-core operands (2^-9 relative per term),
and of the forward's O, which enters D = rowsum(dO o O); each is a few 1e-3 of
the gradient's scale, all accumulated in fp32.
"""
import math

import numpy as np
import pytest

from kv_cache_chunk_ring_b200 import workloads as wl
from oracle.moba import MobaLayout
from oracle import moba_bwd as mb
from tests.gpu_helpers import errors, to_dev, to_np

pytestmark = pytest.mark.gpu

TOL_GRAD_MAX = 1e-2   # max |g - g*| / max |g*|
TOL_GRAD_RMS = 1e-2   # ||g - g*||_2 / ||g*||_2


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_chunk_ring_b200 import build
    build.build()


def assert_grad_close(got, ref, what):
    ma, rr = errors(got, ref)
    scale = float(np.abs(ref).max()) or 1.0
    assert ma <= TOL_GRAD_MAX * scale and rr <= TOL_GRAD_RMS, \
        f"{what}: max_abs={ma:.3e} (max|ref|={scale:.3e}) rel_rms={rr:.3e}"
    return ma / scale, rr


def _gpu_fwd_bwd(spec, inputs=None):
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    q, k, v = wl.moba_inputs(spec) if inputs is None else inputs[:3]
    do = wl.moba_grad_output(spec) if inputs is None else inputs[3]
    qd, kd, vd, dod = (to_dev(x, "bf16") for x in (q, k, v, do))
    o = torch.empty_like(qd)
    lse = torch.empty((spec.heads, spec.seq_len), dtype=torch.float32, device="cuda")
    lay = (spec.n_chunks, spec.chunk_tokens, spec.n_bidir_chunks)
    kvcr.moba_attention_fwd(qd, kd, vd, *lay, o, lse)
    dq, dk, dv = (torch.empty_like(qd) for _ in range(3))
    kvcr.moba_attention_bwd(qd, kd, vd, o, dod, lse, *lay, dq, dk, dv)
    torch.cuda.synchronize()
    kvcr.kvcr_check_status()
    return (q, k, v, do), (qd, kd, vd, dod, o, lse), (dq, dk, dv)


@pytest.mark.parametrize("n,c,m,H,D", [(1, 200, 1, 2, 128), (2, 200, 1, 2, 128),
                                       (3, 100, 2, 2, 64), (2, 128, 1, 1, 128),
                                       (3, 77, 0, 2, 128), (4, 50, 3, 2, 128),
                                       (1, 5, 0, 1, 128), (2, 300, 2, 1, 64),
                                       (1, 1, 0, 1, 128), (1, 1, 0, 2, 64)])   # one key per query
def test_small_layouts_every_gradient(n, c, m, H, D):
    spec = wl.MobaSpec("t", heads=H, head_dim=D, n_chunks=n, chunk_tokens=c, n_bidir_chunks=m,
                       seed=60 + n + c + m)
    (q, k, v, do), _, grads = _gpu_fwd_bwd(spec)
    lay = MobaLayout(n, c, m)
    ref = mb.moba_bwd_dense(q, k, v, do, lay, 1 / math.sqrt(D))
    for name, g, r in zip(("dq", "dk", "dv"), grads, ref):
        assert_grad_close(to_np(g), r, f"{name} n={n} c={c} m={m} D={D}")


def test_deterministic():
    """No atomics: two calls give bit-identical gradients."""
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    spec = wl.MobaSpec("t", heads=3, head_dim=128, n_chunks=3, chunk_tokens=300, n_bidir_chunks=2,
                       seed=71)
    _, (qd, kd, vd, dod, o, lse), g1 = _gpu_fwd_bwd(spec)
    g2 = tuple(torch.empty_like(qd) for _ in range(3))
    kvcr.moba_attention_bwd(qd, kd, vd, o, dod, lse, 3, 300, 2, *g2)
    torch.cuda.synchronize()
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_argument_errors():
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    x = torch.zeros((256, 1, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 256), dtype=torch.float32, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(kvcr.KvcrError) as e:        # workspace too small
        kvcr.moba_attention_bwd(x, x, x, x, x, lse, 1, 128, 0, x, x, x, workspace=ws)
    assert e.value.code == kvcr.KVCR_ESTORAGE
    y = torch.zeros((256, 1, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kvcr.KvcrError) as e:        # head_dim 96
        kvcr.moba_attention_bwd(y, y, y, y, y, lse, 1, 128, 0, y, y, y)
    assert e.value.code == kvcr.KVCR_EUNSUPPORTED


def test_withheld_signal_times_out_and_context_survives():
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    spec = wl.MobaSpec("t", heads=2, head_dim=128, n_chunks=2, chunk_tokens=150, n_bidir_chunks=1,
                       seed=72)
    _, (qd, kd, vd, dod, o, lse), ref = _gpu_fwd_bwd(spec)
    kvcr.kvcr_debug_inject(1, 50_000_000)           # withhold one signal, 50 ms bound
    try:
        bad = tuple(torch.zeros_like(qd) for _ in range(3))
        kvcr.moba_attention_bwd(qd, kd, vd, o, dod, lse, 2, 150, 1, *bad)
        with pytest.raises(kvcr.KvcrError) as e:
            kvcr.kvcr_check_status()
        assert e.value.code == kvcr.KVCR_ETIMEOUT
    finally:
        kvcr.kvcr_debug_inject(0, 0)
    again = tuple(torch.empty_like(qd) for _ in range(3))
    kvcr.moba_attention_bwd(qd, kd, vd, o, dod, lse, 2, 150, 1, *again)
    torch.cuda.synchronize()
    kvcr.kvcr_check_status()
    for a, b in zip(again, ref):
        assert torch.equal(a, b)


def test_full_size_sampled():
    """8 clean + 8 noisy chunks of 6032 tokens + an 8-chunk bidirectional block,
    12 heads, head_dim 128: dQ on sampled rows of every block kind, dK / dV on
    keys of the first noisy chunk (read only by that chunk), all heads; and, over
    every key, sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i per head (each row of
    dS sums to zero, each row of P to one)."""
    spec = wl.MOBA_8x6032
    c, L, H = spec.chunk_tokens, spec.seq_len, spec.heads
    nc = spec.n_chunks * c
    (q, k, v, do), _, (dq, dk, dv) = _gpu_fwd_bwd(spec)
    lay = MobaLayout(spec.n_chunks, c, spec.n_bidir_chunks)
    scale = 1 / math.sqrt(spec.head_dim)
    always = []
    for start in (0, 7 * c, nc, nc + 7 * c, 2 * nc, L - c):
        always += list(range(start, start + 16)) + list(range(start + c - 16, start + c))
    rows = wl.sample_rows(L, 96, 1010, always)
    keys = np.array(sorted(set(list(range(nc, nc + 24)) + list(range(nc + c - 24, nc + c)) +
                               list(wl.sample_rows(c, 48, 1011) + nc))))
    import torch
    ridx = torch.from_numpy(rows).cuda()
    kidx = torch.from_numpy(keys).cuda()
    got_dq = to_np(dq.index_select(0, ridx))
    got_dk = to_np(dk.index_select(0, kidx))
    got_dv = to_np(dv.index_select(0, kidx))
    ref_dq = np.zeros_like(got_dq)
    ref_dk = np.zeros_like(got_dk)
    ref_dv = np.zeros_like(got_dv)
    for h in range(H):
        sl = slice(h, h + 1)
        ref_dq[:, sl] = mb.moba_dq_rows(q[:, sl], k[:, sl], v[:, sl], do[:, sl], lay, rows, scale)
        ref_dk[:, sl], ref_dv[:, sl] = mb.moba_dkdv_keys(q[:, sl], k[:, sl], v[:, sl], do[:, sl],
                                                         lay, keys, scale)
    r = [assert_grad_close(got_dq, ref_dq, "dq full"),
         assert_grad_close(got_dk, ref_dk, "dk full"),
         assert_grad_close(got_dv, ref_dv, "dv full")]
    print("moba bwd full-size (max_abs/max|ref|, rel_rms) dq/dk/dv:", r)

    # key blocks read by many query chunks, element-wise on a few heads (the oracle
    # evaluates every reader's whole row of P): C1 (read by all 8 clean chunks and noisy
    # chunks 2-8), C8, N8 and both ends of the bidirectional block (read by all of B)
    def keyset(start, n_edge, n_rand, seed):
        ks = set(range(start, start + n_edge)) | set(range(start + c - n_edge, start + c))
        ks |= set((wl.sample_rows(c, n_rand, seed) + start).tolist())
        return np.array(sorted(ks))
    heavy = [("C1", keyset(0, 8, 16, 1012), [0, 6]),
             ("C8", keyset(7 * c, 8, 16, 1013), [3, 11]),
             ("N8", keyset(nc + 7 * c, 8, 16, 1014), [5, 8]),
             ("B ends", np.array(list(range(2 * nc, 2 * nc + 16)) + list(range(L - 16, L))),
              [1, 7])]
    for name, keys, heads in heavy:
        kidx = torch.from_numpy(keys).cuda()
        got_k = to_np(dk.index_select(0, kidx))[:, heads]
        got_v = to_np(dv.index_select(0, kidx))[:, heads]
        ref_k, ref_v = np.zeros_like(got_k), np.zeros_like(got_v)
        for j, h in enumerate(heads):
            sl = slice(h, h + 1)
            ref_k[:, j:j + 1], ref_v[:, j:j + 1] = mb.moba_dkdv_keys(
                q[:, sl], k[:, sl], v[:, sl], do[:, sl], lay, keys, scale)
        rk = assert_grad_close(got_k, ref_k, f"dk {name}")
        rv = assert_grad_close(got_v, ref_v, f"dv {name}")
        print(f"moba bwd full-size dk/dv on {name} keys, heads {heads}: {rk} {rv}")

    sum_dk = dk.float().sum(0).double().cpu().numpy()               # [H, D]
    sum_dv = dv.float().sum(0).double().cpu().numpy()
    sum_do = do.astype(np.float64).sum(0)
    for h in range(H):
        nk = float(dk[:, h].float().norm())
        # P is a bf16 operand: each row's sum is off by up to 2^-9, so sum_j dV_j - sum_i dO_i
        # is a random walk of size ~2^-9 ||dO||_F (bounded here with a factor 4)
        bound_v = 4 * 2.0 ** -9 * float(np.linalg.norm(do[:, h]))
        assert np.linalg.norm(sum_dk[h]) <= 1e-2 * nk, (h, np.linalg.norm(sum_dk[h]), nk)
        assert np.linalg.norm(sum_dv[h] - sum_do[h]) <= bound_v, \
            (h, np.linalg.norm(sum_dv[h] - sum_do[h]), bound_v)


def test_mid_size_head_dim_64_sampled():
    """4 + 4 chunks of 1000 tokens + a 2-chunk bidirectional block (10000 tokens), 4 heads of
    head_dim 64: dQ on sampled rows, dK / dV on sampled keys of three block kinds."""
    spec = wl.MobaSpec("t", heads=4, head_dim=64, n_chunks=4, chunk_tokens=1000,
                       n_bidir_chunks=2, seed=73)
    c, L = spec.chunk_tokens, spec.seq_len
    nc = spec.n_chunks * c
    (q, k, v, do), _, (dq, dk, dv) = _gpu_fwd_bwd(spec)
    lay = MobaLayout(spec.n_chunks, c, spec.n_bidir_chunks)
    scale = 1 / math.sqrt(64)
    rows = wl.sample_rows(L, 128, 1040, [0, c - 1, c, nc, nc + c - 1, 2 * nc, L - 1])
    keys = np.array(sorted({3 * c + 5, 3 * c + 999, nc + 2 * c + 7, 2 * nc + 11, L - 1, 0, 130}))
    import torch
    ridx = torch.from_numpy(rows).cuda()
    kidx = torch.from_numpy(keys).cuda()
    assert_grad_close(to_np(dq.index_select(0, ridx)),
                      mb.moba_dq_rows(q, k, v, do, lay, rows, scale), "dq d64")
    ref_dk, ref_dv = mb.moba_dkdv_keys(q, k, v, do, lay, keys, scale)
    assert_grad_close(to_np(dk.index_select(0, kidx)), ref_dk, "dk d64")
    assert_grad_close(to_np(dv.index_select(0, kidx)), ref_dv, "dv d64")
