"""Pins of the rotary-embedding oracle (oracle/rope.py) against formulations other
than its own: complex multiplication, the relative-position identity, the
sinusoidal table of the pages' PositionalEncoding, and closed forms. Planted
mistakes in it (on the CPU) must each fail at least one pin."""
import math

import numpy as np
import pytest

from oracle import rope as R


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def pin_complex_rotation(fn, D):
    # Feature pair (2i, 2i+1) as the complex number x[2i] + j x[2i+1], multiplied
    # by exp(j p theta_i); theta_i from the power written as exp of a log.
    x = _rand((3, 5, 2, D), 1)                       # [batch, P, H, D]
    pos = np.array([0, 1, 7, 4093, 131071])
    z = x[..., 0::2] + 1j * x[..., 1::2]
    th = np.exp(-np.arange(D // 2) * 2.0 / D * math.log(10000.0))
    rot = np.exp(1j * pos[:, None] * th[None, :])[None, :, None, :]
    ref = np.empty_like(x)
    ref[..., 0::2] = (z * rot).real
    ref[..., 1::2] = (z * rot).imag
    np.testing.assert_allclose(fn(x, pos), ref, rtol=0, atol=1e-9)


def pin_relative_position(fn):
    # <rope(q, p), rope(k, p')> depends only on p - p'.
    D = 64
    q = _rand((1, 1, D), 2)
    k = _rand((1, 1, D), 3)
    for p, pp in ((5, 2), (1000, 13), (70000, 69999), (3, 40)):
        a = np.sum(fn(q, np.array([p])) * fn(k, np.array([pp])))
        b = np.sum(fn(q, np.array([p - pp])) * k)
        assert abs(a - b) < 1e-9 * max(1.0, abs(a))


def pin_position_zero_and_norms(fn):
    x = _rand((4, 3, 32), 4)
    np.testing.assert_array_equal(fn(x, np.zeros(4, dtype=np.int64)), x)
    y = fn(x, np.array([1, 99, 12345, 7]))
    n_x = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    n_y = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(n_y, n_x, rtol=1e-12)


def pin_pages_sinusoidal_table(fn):
    # Page "Tensor并行与算子拆分": PE[p, 2i] = sin(p * w_i), PE[p, 2i+1] = cos(p * w_i),
    # w_i = exp(2i * (-ln 10000 / d)). Rotating the unit odd feature of every pair
    # gives (-sin, cos) at those frequencies.
    d, P = 16, 50
    pos = np.arange(P)
    w = np.exp(np.arange(0, d, 2) * (-math.log(10000.0) / d))
    pe = np.zeros((P, d))
    pe[:, 0::2] = np.sin(pos[:, None] * w[None, :])
    pe[:, 1::2] = np.cos(pos[:, None] * w[None, :])
    x = np.zeros((P, 1, d))
    x[..., 1::2] = 1.0
    y = fn(x, pos)[:, 0, :]
    np.testing.assert_allclose(y[:, 0::2], -pe[:, 0::2], atol=1e-12)
    np.testing.assert_allclose(y[:, 1::2], pe[:, 1::2], atol=1e-12)


@pytest.mark.parametrize("D", [2, 8, 64, 128])
def test_rope_equals_complex_rotation(D):
    pin_complex_rotation(R.rope, D)


def test_rope_relative_position_identity():
    pin_relative_position(R.rope)


def test_rope_position_zero_and_norms():
    pin_position_zero_and_norms(R.rope)


def test_rope_matches_the_pages_sinusoidal_table():
    pin_pages_sinusoidal_table(R.rope)


def _rotate_half(x, pos, base=10000.0):
    # The other common pairing, (i, i + D/2): a plausible mix-up.
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    y = np.concatenate([x[..., 0::2], x[..., 1::2]], axis=-1)   # interleaved -> halves
    ang = np.asarray(pos, dtype=np.float64)[:, None] * R.theta(D, base)[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    a, b = y[..., :D // 2], y[..., D // 2:]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return np.concatenate([out[..., 0::2], out[..., 1::2]], axis=-1)


ROPE_MUTANTS = {
    "sin_sign_flipped": lambda x, pos: R.rope(x, -np.asarray(pos)),
    "base_1000": lambda x, pos: R.rope(x, pos, base=1000.0),
    "positions_off_by_one": lambda x, pos: R.rope(x, np.asarray(pos) + 1),
    "local_positions": lambda x, pos: R.rope(x, np.asarray(pos) % 4096),
    "rotate_half_pairing": _rotate_half,
}


def _fails(check):
    try:
        check()
    except AssertionError:
        return True
    return False


@pytest.mark.parametrize("name", sorted(ROPE_MUTANTS))
def test_rope_mutant_is_caught(name):
    fn = ROPE_MUTANTS[name]
    checks = [lambda: pin_complex_rotation(fn, 8), lambda: pin_complex_rotation(fn, 128),
              lambda: pin_relative_position(fn), lambda: pin_position_zero_and_norms(fn),
              lambda: pin_pages_sinusoidal_table(fn)]
    assert any(_fails(c) for c in checks), name
