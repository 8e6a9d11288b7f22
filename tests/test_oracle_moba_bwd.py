"""Pins of the oracle's MoBA backward: central finite differences of the forward
oracle's loss, invariances, and agreement of the row-sampled and dense forms."""
import numpy as np
import pytest

from oracle.attn import masked_attention
from oracle.moba import MobaLayout, moba_mask
from oracle import moba_bwd as mb


def _inputs(lay, H=1, D=4, seed=0):
    rng = np.random.default_rng(seed)
    L = lay.seq_len
    return tuple(rng.standard_normal((L, H, D)) for _ in range(4))


def _loss(q, k, v, do, lay, scale):
    o, _ = masked_attention(q, k, v, moba_mask(lay), scale)
    return float((o * do).sum())


@pytest.mark.parametrize("n,c,m", [(2, 3, 1), (1, 4, 1), (3, 2, 2)])
def test_matches_central_finite_differences(n, c, m):
    lay = MobaLayout(n, c, m)
    scale = 0.4
    q, k, v, do = _inputs(lay, H=1, D=3, seed=n + c + m)
    dq, dk, dv = mb.moba_bwd_dense(q, k, v, do, lay, scale)
    eps = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            old = x[i]
            x[i] = old + eps
            lp = _loss(q, k, v, do, lay, scale)
            x[i] = old - eps
            lm = _loss(q, k, v, do, lay, scale)
            x[i] = old
            num[i] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(g, num, atol=1e-7, rtol=1e-6)


def test_dv_is_explicit_probability_sum():
    lay = MobaLayout(2, 3, 1)
    scale = 0.7
    q, k, v, do = _inputs(lay, H=2, D=4, seed=3)
    _, _, dv = mb.moba_bwd_dense(q, k, v, do, lay, scale)
    mask = moba_mask(lay)
    for h in range(2):
        for key in range(lay.seq_len):
            acc = np.zeros(4)
            for r in range(lay.seq_len):
                if not mask[r, key]:
                    continue
                z = np.array([scale * q[r, h] @ k[j, h] if mask[r, j] else -np.inf
                              for j in range(lay.seq_len)])
                p = np.exp(z - z.max())
                p /= p.sum()
                acc += p[key] * do[r, h]
            np.testing.assert_allclose(dv[key, h], acc, atol=1e-12)


def test_dq_unchanged_by_common_key_shift():
    """Adding one vector to every key shifts each query's logits by a constant, so O and
    therefore dQ do not change."""
    lay = MobaLayout(2, 4, 1)
    q, k, v, do = _inputs(lay, H=1, D=5, seed=4)
    dq1, _, _ = mb.moba_bwd_dense(q, k, v, do, lay, 0.5)
    dq2, _, _ = mb.moba_bwd_dense(q, k + np.random.default_rng(9).standard_normal(5), v, do, lay, 0.5)
    np.testing.assert_allclose(dq1, dq2, atol=1e-12)


def test_zero_upstream_gradient_gives_zero():
    lay = MobaLayout(2, 3, 2)
    q, k, v, _ = _inputs(lay, H=1, D=4, seed=5)
    for g in mb.moba_bwd_dense(q, k, v, np.zeros_like(q), lay, 0.3):
        assert np.all(g == 0.0)


@pytest.mark.parametrize("n,c,m", [(2, 5, 1), (3, 4, 2)])
def test_sampled_forms_match_dense(n, c, m):
    lay = MobaLayout(n, c, m)
    q, k, v, do = _inputs(lay, H=2, D=6, seed=6)
    dq, dk, dv = mb.moba_bwd_dense(q, k, v, do, lay, 0.45)
    rows = [0, 3, c, 2 * n * c - 1, lay.seq_len - 1]
    np.testing.assert_allclose(mb.moba_dq_rows(q, k, v, do, lay, rows, 0.45), dq[rows], atol=1e-12)
    keys = [1, c + 2, n * c, 2 * n * c + 1]
    dk_s, dv_s = mb.moba_dkdv_keys(q, k, v, do, lay, keys, 0.45)
    np.testing.assert_allclose(dk_s, dk[keys], atol=1e-12)
    np.testing.assert_allclose(dv_s, dv[keys], atol=1e-12)


def test_planted_mistake_is_caught(monkeypatch):
    """Dropping the D term (a plausible slip) must fail the finite-difference pin."""
    real = mb.attention_bwd_masked

    def no_d(q, k, v, do, allowed, scale):
        q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
        dq, dk, dv = real(q, k, v, do, allowed, scale)
        h = 0
        z = np.where(allowed, scale * (q[:, h] @ k[:, h].T), -np.inf)
        p = np.exp(z - z.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        ds = p * (do[:, h] @ v[:, h].T)
        dq[:, h] = scale * ds @ k[:, h]
        return dq, dk, dv
    monkeypatch.setattr(mb, "attention_bwd_masked", no_d)
    with pytest.raises(AssertionError):
        test_matches_central_finite_differences(2, 3, 1)


def test_single_readable_key_closed_form():
    """n = 1, one-token chunks, no bidirectional block: the query of C1 reads only C1's key
    and the query of N1 only N1's (N1 reads no clean chunk before it).  P = 1 on that key,
    O = its V, dP = dO . V = D, so dS = 0: dV = dO, dQ = dK = 0."""
    lay = MobaLayout(1, 1, 0)
    q, k, v, do = _inputs(lay, H=3, D=5, seed=11)
    dq, dk, dv = mb.moba_bwd_dense(q, k, v, do, lay, 0.6)
    np.testing.assert_allclose(dv, do, atol=1e-12)
    np.testing.assert_allclose(dq, 0.0, atol=1e-12)
    np.testing.assert_allclose(dk, 0.0, atol=1e-12)
    rows = [0, 1]
    np.testing.assert_allclose(mb.moba_dq_rows(q, k, v, do, lay, rows, 0.6), 0.0, atol=1e-12)
    dk_s, dv_s = mb.moba_dkdv_keys(q, k, v, do, lay, rows, 0.6)
    np.testing.assert_allclose(dv_s, do, atol=1e-12)
    np.testing.assert_allclose(dk_s, 0.0, atol=1e-12)
