"""Pins of the oracle's 3D RoPE against facts other than its own formula."""
import math
import os

import numpy as np
import pytest

from oracle.rope import rope3d, rope_positions, rope_pairs_default, axis_of_pair

GOLD = os.path.join(os.path.dirname(__file__), "golden", "rope_angles.txt")


def _read_golden():
    rows = []
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        a, b, c = [x.strip() for x in line.split("|")]
        pairs = tuple(int(x) for x in a.split())
        pos = tuple(int(x) for x in b.split())
        angles = [float(eval(x, {"__builtins__": {}})) for x in c.split()]
        rows.append((pairs, pos, angles))
    return rows


@pytest.mark.parametrize("pairs,pos,angles", _read_golden())
def test_hand_derived_angles(pairs, pos, angles):
    D = 2 * sum(pairs)
    x = np.zeros((1, 1, D))
    x[0, 0, 0::2] = 1.0                       # every pair = (1, 0)
    t, h, w = (np.array([p]) for p in pos)
    y = rope3d(x, t, h, w, pairs)
    got = y[0, 0]
    for i, a in enumerate(angles):
        assert got[2 * i] == pytest.approx(math.cos(a), abs=1e-13)
        assert got[2 * i + 1] == pytest.approx(math.sin(a), abs=1e-13)
    # (0, 1) turns to (-sin a, cos a)
    x2 = np.zeros((1, 1, D))
    x2[0, 0, 1::2] = 1.0
    y2 = rope3d(x2, t, h, w, pairs)[0, 0]
    for i, a in enumerate(angles):
        assert y2[2 * i] == pytest.approx(-math.sin(a), abs=1e-13)
        assert y2[2 * i + 1] == pytest.approx(math.cos(a), abs=1e-13)


def test_default_split_matches_workload_statement():
    # 832x464 workload: split 44/42/42 rotary dims over head_dim 128
    pt, ph, pw = rope_pairs_default(128)
    assert (2 * pt, 2 * ph, 2 * pw) == (44, 42, 42)
    assert sum(rope_pairs_default(64)) * 2 == 64


def test_position_zero_is_identity():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((7, 3, 128))
    z = np.zeros(7, dtype=np.int64)
    assert np.array_equal(rope3d(x, z, z, z, rope_pairs_default(128)), x)


def test_pair_norms_preserved():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((50, 2, 64))
    t = rng.integers(0, 10_000, 50)
    h = rng.integers(0, 45, 50)
    w = rng.integers(0, 80, 50)
    y = rope3d(x, t, h, w, rope_pairs_default(64))
    nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-12, atol=1e-12)


def test_relative_position_property():
    """<R(p) q, R(p') k> depends on p' - p only, on every axis."""
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 1, 128))
    k = rng.standard_normal((1, 1, 128))
    pairs = rope_pairs_default(128)

    def dot(pq, pk):
        a = rope3d(q, *[np.array([v]) for v in pq], pairs)
        b = rope3d(k, *[np.array([v]) for v in pk], pairs)
        return float((a * b).sum())

    base = dot((3, 4, 5), (10, 6, 9))
    for shift in [(1, 0, 0), (0, 7, 0), (0, 0, 11), (500, 20, 30)]:
        pq = tuple(a + s for a, s in zip((3, 4, 5), shift))
        pk = tuple(a + s for a, s in zip((10, 6, 9), shift))
        assert dot(pq, pk) == pytest.approx(base, rel=1e-9, abs=1e-9)
    # ... and it does depend on the offset
    assert abs(dot((3, 4, 5), (11, 6, 9)) - base) > 1e-6


def test_single_axis_reduces_to_textbook_rope():
    """One axis owning every pair is 1D RoPE: RoFormer's theta_i = 10000^(-2(i-1)/d),
    i = 1..d/2, applied to (x_{2i-1}, x_{2i}) as a complex multiplication."""
    d = 32
    rng = np.random.default_rng(8)
    x = rng.standard_normal((9, 2, d))
    pos = rng.integers(0, 4000, 9)
    z = np.zeros(9, dtype=np.int64)
    for axis in range(3):
        pairs = [0, 0, 0]
        pairs[axis] = d // 2
        args = [z, z, z]
        args[axis] = pos
        got = rope3d(x, *args, tuple(pairs))
        xc = x[..., 0::2] + 1j * x[..., 1::2]
        i = np.arange(1, d // 2 + 1)
        theta = 10000.0 ** (-2.0 * (i - 1) / d)
        ref = xc * np.exp(1j * pos[:, None, None] * theta[None, None, :])
        np.testing.assert_allclose(got[..., 0::2], ref.real, atol=1e-12)
        np.testing.assert_allclose(got[..., 1::2], ref.imag, atol=1e-12)


def test_axes_are_separate():
    """Moving along one axis changes only that axis' pairs."""
    pairs = rope_pairs_default(128)
    rng = np.random.default_rng(9)
    x = rng.standard_normal((1, 1, 128))
    ref = rope3d(x, np.array([3]), np.array([4]), np.array([5]), pairs)
    owner = np.array([axis_of_pair(i, pairs)[0] for i in range(64)])
    for axis in range(3):
        pos = [np.array([3]), np.array([4]), np.array([5])]
        pos[axis] = pos[axis] + 1
        y = rope3d(x, *pos, pairs)
        changed = ~np.isclose(y[0, 0, 0::2], ref[0, 0, 0::2]) | ~np.isclose(y[0, 0, 1::2], ref[0, 0, 1::2])
        assert np.all(owner[changed] == axis)
        assert changed[owner == axis].all()
    # pair order: t pairs first, then h, then w
    assert list(owner[:22]) == [0] * 22 and list(owner[22:43]) == [1] * 21 and list(owner[43:]) == [2] * 21


def test_composition():
    """R(p) R(p') = R(p + p') for each axis."""
    pairs = (3, 3, 2)
    rng = np.random.default_rng(10)
    x = rng.standard_normal((4, 1, 16))
    a = (np.array([1, 2, 3, 4]), np.array([0, 5, 1, 2]), np.array([7, 0, 2, 9]))
    b = (np.array([10, 0, 3, 1]), np.array([2, 2, 8, 0]), np.array([1, 1, 4, 3]))
    two = rope3d(rope3d(x, *a, pairs), *b, pairs)
    one = rope3d(x, *(u + v for u, v in zip(a, b)), pairs)
    np.testing.assert_allclose(two, one, atol=1e-12)


def test_positions_row_major():
    t, h, w = rope_positions([7, 8], 3, 4)
    assert list(t) == [7] * 12 + [8] * 12
    assert list(h[:12]) == [0] * 4 + [1] * 4 + [2] * 4
    assert list(w[:12]) == [0, 1, 2, 3] * 3
