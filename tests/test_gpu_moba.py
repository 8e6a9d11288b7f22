"""GPU parity of the MoBA block-sparse attention against the fp64 oracle."""
import math

import numpy as np
import pytest

from kv_cache_chunk_ring_b200 import workloads as wl
from oracle.moba import MobaLayout, moba_attention_rows
from tests.gpu_helpers import TOL_LSE, assert_close, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_chunk_ring_b200 import build
    build.build()


def _run(spec, rows=None):
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    q, k, v = wl.moba_inputs(spec)
    qd, kd, vd = (to_dev(x, "bf16") for x in (q, k, v))
    o = torch.empty_like(qd)
    lse = torch.empty((spec.heads, spec.seq_len), dtype=torch.float32, device="cuda")
    kvcr.moba_attention_fwd(qd, kd, vd, spec.n_chunks, spec.chunk_tokens, spec.n_bidir_chunks, o,
                            lse)
    torch.cuda.synchronize()
    lay = MobaLayout(spec.n_chunks, spec.chunk_tokens, spec.n_bidir_chunks)
    if rows is None:
        rows = np.arange(spec.seq_len)
    o_ref, l_ref = moba_attention_rows(q, k, v, lay, rows, 1 / math.sqrt(spec.head_dim))
    idx = torch.from_numpy(np.asarray(rows)).cuda()
    o_got = to_np(o.index_select(0, idx))
    l_got = lse.index_select(1, idx).cpu().numpy()
    return (q, k, v), (qd, kd, vd, o, lse), o_got, o_ref, l_got, l_ref


@pytest.mark.parametrize("n,c,m,H,D", [(1, 200, 1, 2, 128), (2, 200, 1, 2, 128), (3, 100, 2, 2, 64),
                                       (2, 300, 2, 1, 128), (4, 50, 3, 2, 128), (2, 128, 1, 1, 128),
                                       (3, 77, 0, 2, 128)])
def test_small_layouts_all_rows(n, c, m, H, D):
    spec = wl.MobaSpec("t", heads=H, head_dim=D, n_chunks=n, chunk_tokens=c, n_bidir_chunks=m,
                       seed=30 + n + c)
    _, _, o, o_ref, l, l_ref = _run(spec)
    assert_close(o, o_ref, "moba small")
    assert np.abs(l - l_ref).max() <= TOL_LSE


def test_full_size_sampled_rows():
    """8 clean + 8 noisy chunks of 6032 tokens + an 8-chunk bidirectional block."""
    spec = wl.MOBA_8x6032
    c = spec.chunk_tokens
    L = spec.seq_len
    always = []
    for start in (0, 7 * c, 8 * c, 15 * c, 16 * c, L - c):       # C1, C8, N1, N8, B first/last chunk
        always += list(range(start, start + 64)) + list(range(start + c - 64, start + c))
    rows = wl.sample_rows(L, 384, 1004, always)
    _, _, o, o_ref, l, l_ref = _run(spec, rows)
    ma, rr = assert_close(o, o_ref, "moba full")
    assert np.abs(l - l_ref).max() <= TOL_LSE
    print(f"moba full-size max_abs={ma:.3e} rel_rms={rr:.3e}")


def test_disallowed_keys_do_not_matter():
    """Changing keys/values a query may not read leaves its output bit-identical."""
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    spec = wl.MobaSpec("t", heads=2, head_dim=128, n_chunks=3, chunk_tokens=150, n_bidir_chunks=2,
                       seed=41)
    (q, k, v), (qd, kd, vd, o, lse), *_ = _run(spec, rows=[0])
    c = spec.chunk_tokens
    # rows of C1 read only C1: change everything after C1
    k2, v2 = kd.clone(), vd.clone()
    k2[c:] = torch.randn_like(k2[c:])
    v2[c:] = torch.randn_like(v2[c:])
    o2 = torch.empty_like(o)
    kvcr.moba_attention_fwd(qd, k2, v2, spec.n_chunks, c, spec.n_bidir_chunks, o2)
    torch.cuda.synchronize()
    assert torch.equal(o[:c], o2[:c])
    # rows of B read only B: change everything before B
    b0 = 2 * spec.n_chunks * c
    k3, v3 = kd.clone(), vd.clone()
    k3[:b0] = torch.randn_like(k3[:b0])
    v3[:b0] = torch.randn_like(v3[:b0])
    o3 = torch.empty_like(o)
    kvcr.moba_attention_fwd(qd, k3, v3, spec.n_chunks, c, spec.n_bidir_chunks, o3)
    torch.cuda.synchronize()
    assert torch.equal(o[b0:], o3[b0:])
