"""Pins for oracle.rope: identity at position 0, inverse, composition, the
relative-position property and the textbook angle at position 1."""
import math

import numpy as np

from oracle.rope import rope_angles, rope_rotate


def _x(n=6, d=512, seed=0):
    return np.random.default_rng(seed).standard_normal((n, d))


def test_position_zero_is_identity():
    x = _x()
    assert np.array_equal(rope_rotate(x, 0), x)


def test_only_rope_dims_change():
    x = _x()
    y = rope_rotate(x, 12345)
    assert np.array_equal(y[:, :448], x[:, :448])
    assert not np.allclose(y[:, 448:], x[:, 448:])


def test_inverse_undoes_forward_and_preserves_pair_norms():
    x = _x()
    pos = np.array([0, 1, 7, 1000, 65537, 999_999])
    y = rope_rotate(x, pos)
    z = rope_rotate(y, pos, inverse=True)
    assert np.allclose(z, x, atol=1e-12)
    n0 = x[:, 448::2] ** 2 + x[:, 449::2] ** 2
    n1 = y[:, 448::2] ** 2 + y[:, 449::2] ** 2
    assert np.allclose(n0, n1, rtol=1e-13)


def test_composition_adds_positions():
    x = _x()
    a = rope_rotate(rope_rotate(x, 300), 4000)
    b = rope_rotate(x, 4300)
    assert np.allclose(a, b, atol=1e-10)


def test_relative_position_property():
    # <R(p) a, R(s) b> depends only on s - p: the property inverse RoPE on the
    # shared K=V output relies on
    a, b = _x(1, seed=1)[0], _x(1, seed=2)[0]
    d1 = rope_rotate(a, 17) @ rope_rotate(b, 5)
    d2 = rope_rotate(a, 17 + 100_000) @ rope_rotate(b, 5 + 100_000)
    assert abs(d1 - d2) < 1e-9


def test_textbook_angles():
    # pair 0 has frequency theta^0 = 1: (1, 0) at position 1 -> (cos 1, sin 1)
    x = np.zeros(512)
    x[448] = 1.0
    y = rope_rotate(x, 1)
    assert abs(y[448] - 0.5403023058681398) < 1e-15
    assert abs(y[449] - 0.8414709848078965) < 1e-15
    # pair 16 has frequency theta^(-32/64) = 1e6^-0.5 = 1e-3
    ang = rope_angles(1000, 1e6, 64)
    assert abs(ang[16] - 1.0) < 1e-12
    assert abs(ang[0] - 1000.0) == 0.0
    assert math.isclose(ang[31], 1000 * 1e6 ** (-62 / 64), rel_tol=1e-14)
