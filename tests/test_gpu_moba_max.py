"""MoBA forward and backward at the longest sequence the calls accept: 4096 tiles of
128 tokens (16 clean + 16 noisy chunks of 16384 tokens, 524288 tokens), one head."""
import math

import numpy as np
import pytest

from kv_cache_chunk_ring_b200 import workloads as wl
from oracle.moba import MobaLayout, moba_attention_rows
from oracle import moba_bwd as mb
from tests.gpu_helpers import TOL_LSE, assert_close, errors, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_chunk_ring_b200 import build
    build.build()


def test_longest_sequence_forward_and_backward():
    import torch
    from kv_cache_chunk_ring_b200 import kvcr
    spec = wl.MobaSpec("moba_max", heads=1, head_dim=128, n_chunks=16, chunk_tokens=16384,
                       n_bidir_chunks=0, seed=81)
    L, c = spec.seq_len, spec.chunk_tokens
    nc = spec.n_chunks * c
    assert L == 4096 * 128
    q, k, v = wl.moba_inputs(spec)
    do = wl.moba_grad_output(spec)
    qd, kd, vd, dod = (to_dev(x, "bf16") for x in (q, k, v, do))
    o = torch.empty_like(qd)
    lse = torch.empty((1, L), dtype=torch.float32, device="cuda")
    lay = (spec.n_chunks, c, 0)
    kvcr.moba_attention_fwd(qd, kd, vd, *lay, o, lse)
    dq, dk, dv = (torch.empty_like(qd) for _ in range(3))
    kvcr.moba_attention_bwd(qd, kd, vd, o, dod, lse, *lay, dq, dk, dv)
    torch.cuda.synchronize()
    kvcr.kvcr_check_status()

    ol = MobaLayout(spec.n_chunks, c, 0)
    scale = 1 / math.sqrt(128)
    edges = []
    for start in (0, 15 * c, nc, nc + 15 * c):          # C1, C16, N1, N16
        edges += list(range(start, start + 8)) + list(range(start + c - 8, start + c))
    rows = wl.sample_rows(L, 48, 1030, edges)
    idx = torch.from_numpy(rows).cuda()
    o_ref, l_ref = moba_attention_rows(q, k, v, ol, rows, scale)
    assert_close(to_np(o.index_select(0, idx)), o_ref, "forward")
    assert np.abs(lse.index_select(1, idx).cpu().numpy() - l_ref).max() <= TOL_LSE

    ref_dq = mb.moba_dq_rows(q, k, v, do, ol, rows, scale)
    got_dq = to_np(dq.index_select(0, idx))
    ma, rr = errors(got_dq, ref_dq)
    assert ma <= 1e-2 * np.abs(ref_dq).max() and rr <= 1e-2, (ma, rr)

    keys = np.array(list(range(nc, nc + 8)) + list(range(nc + c - 8, nc + c)))   # read by N1 only
    ref_dk, ref_dv = mb.moba_dkdv_keys(q, k, v, do, ol, keys, scale)
    kidx = torch.from_numpy(keys).cuda()
    for name, got, ref in (("dk", dk, ref_dk), ("dv", dv, ref_dv)):
        g = to_np(got.index_select(0, kidx))
        ma, rr = errors(g, ref)
        assert ma <= 1e-2 * np.abs(ref).max() and rr <= 1e-2, (name, ma, rr)
    # every row of dS sums to zero and every row of P to one; P is a bf16 operand, so each
    # row's sum is off by up to 2^-9 and sum_j dV_j - sum_i dO_i is a random walk of size
    # ~2^-9 ||dO||_F (bounded here with a factor 4)
    nk = float(dk.float().norm())
    assert float(dk.float().sum(0).norm()) <= 1e-2 * nk
    sum_do = torch.from_numpy(do.astype(np.float32).sum(0)).cuda()
    assert float((dv.float().sum(0) - sum_do).norm()) <= 4 * 2.0 ** -9 * float(np.linalg.norm(do))
