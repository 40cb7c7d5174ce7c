"""Pins for the oracle's rotary position encoding (oracle.rope).

The pages name the rotation of Q and K but give no formula; the oracle takes
the standard rotary form.  The pins check it against numpy's complex
exponential (each pair is a complex number multiplied by exp(i p theta)), the
property the form exists for (the score of two rotated vectors depends only
on their distance; position 0 is the identity; norms are kept), and the
restart of positions at every packed sequence.
"""

import numpy as np

import oracle


def test_rope_is_complex_rotation():
    """Each pair is multiplied by exp(i p theta_i), computed by numpy's complex exp."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal((2, 9, 3, 8))
    y = oracle.rope(x, base=500.0)
    z = x[..., 0::2] + 1j * x[..., 1::2]
    theta = 500.0 ** (-np.arange(4) * 2 / 8)
    w = z * np.exp(1j * np.arange(9)[None, :, None, None] * theta)
    np.testing.assert_allclose(y[..., 0::2], w.real, rtol=0, atol=1e-13)
    np.testing.assert_allclose(y[..., 1::2], w.imag, rtol=0, atol=1e-13)


def test_rope_relative_positions():
    """<R_n q, R_m k> depends only on n - m, and position 0 is the identity."""
    rng = np.random.default_rng(8)
    d = 16
    q = rng.standard_normal(d)
    k = rng.standard_normal(d)
    x = np.zeros((1, 40, 2, d))
    x[0, :, 0] = q
    x[0, :, 1] = k
    y = oracle.rope(x)
    np.testing.assert_array_equal(y[0, 0], x[0, 0])
    for n, m in [(5, 2), (30, 27), (13, 10)]:          # the same distance 3
        assert abs(np.dot(y[0, n, 0], y[0, m, 1]) - np.dot(y[0, 3, 0], y[0, 0, 1])) < 1e-12
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)


def test_rope_packed_positions_restart():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((1, 12, 1, 4))
    cu = [0, 5, 5, 12]
    y = oracle.rope(x, cu_seqlens=cu)
    np.testing.assert_allclose(y[:, 0:5], oracle.rope(x[:, 0:5]), rtol=0, atol=0)
    np.testing.assert_allclose(y[:, 5:12], oracle.rope(x[:, 5:12]), rtol=0, atol=0)
