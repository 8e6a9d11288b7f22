"""Pins of the oracle's attention: brute force, closed forms, invariances."""
import math

import numpy as np
import pytest

from oracle.attn import attention, masked_attention, attention_bruteforce


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_matches_bruteforce_loops():
    rng = np.random.default_rng(1)
    q, k, v = _rand(rng, 5, 2, 8), _rand(rng, 7, 2, 8), _rand(rng, 7, 2, 8)
    o, lse = attention(q, k, v, 0.3)
    ob, lb = attention_bruteforce(q.tolist(), k.tolist(), v.tolist(), 0.3)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-12)


def test_masked_matches_bruteforce():
    rng = np.random.default_rng(2)
    q, k, v = _rand(rng, 6, 1, 4), _rand(rng, 9, 1, 4), _rand(rng, 9, 1, 4)
    allowed = rng.random((6, 9)) < 0.5
    allowed[3] = False                      # a row with nothing to read
    o, lse = masked_attention(q, k, v, allowed, 0.5)
    ob, lb = attention_bruteforce(q.tolist(), k.tolist(), v.tolist(), 0.5, allowed.tolist())
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-12)
    assert np.all(o[3] == 0.0) and np.all(np.isneginf(lse[:, 3]))


def test_zero_query_gives_mean_and_log_n():
    rng = np.random.default_rng(3)
    k, v = _rand(rng, 37, 3, 16), _rand(rng, 37, 3, 16)
    q = np.zeros((4, 3, 16))
    o, lse = attention(q, k, v, 1 / math.sqrt(16))
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=0), o.shape), atol=1e-13)
    np.testing.assert_allclose(lse, math.log(37), atol=1e-13)


def test_constant_v_and_single_key():
    rng = np.random.default_rng(4)
    q, k = _rand(rng, 6, 2, 8), _rand(rng, 11, 2, 8)
    v = np.full((11, 2, 8), 0.75)
    o, _ = attention(q, k, v, 1.0)
    np.testing.assert_allclose(o, 0.75, atol=1e-14)
    o1, lse1 = attention(q, k[:1], k[:1] * 2, 0.2)
    np.testing.assert_allclose(o1, np.broadcast_to(k[:1] * 2, o1.shape), atol=1e-14)
    np.testing.assert_allclose(lse1[0], 0.2 * (q[:, 0] @ k[0, 0]), atol=1e-13)


def test_key_permutation_invariance():
    rng = np.random.default_rng(5)
    q, k, v = _rand(rng, 5, 2, 8), _rand(rng, 13, 2, 8), _rand(rng, 13, 2, 8)
    p = rng.permutation(13)
    o, lse = attention(q, k, v, 0.4)
    o2, lse2 = attention(q, k[p], v[p], 0.4)
    np.testing.assert_allclose(o, o2, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, atol=1e-13)


def test_two_keys_closed_form():
    """Two keys with scores a, b: o = (e^a v1 + e^b v2) / (e^a + e^b)."""
    q = np.array([[[1.0, 0.0]]])
    k = np.array([[[2.0, 0.0]], [[-1.0, 0.0]]])
    v = np.array([[[1.0, 3.0]], [[5.0, -1.0]]])
    o, lse = attention(q, k, v, 1.0)
    wa, wb = math.exp(2.0), math.exp(-1.0)
    assert o[0, 0, 0] == pytest.approx((wa * 1 + wb * 5) / (wa + wb), abs=1e-14)
    assert o[0, 0, 1] == pytest.approx((wa * 3 - wb * 1) / (wa + wb), abs=1e-14)
    assert lse[0, 0] == pytest.approx(math.log(wa + wb), abs=1e-14)
