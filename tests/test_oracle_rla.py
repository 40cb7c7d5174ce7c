"""Pins for the oracle's residual linear attention (oracle.rla).

RLA (RAttention page, "Residual Linear Attention (RLA) 수식") reads a
decay-free linear-attention state w tokens late.  Pins: the double sum of the
definition on tiny inputs, the feature map against scipy's softmax, the
no-delay case against the retention oracle at gamma = 1 (a different route:
the parallel form), windows past the sequence length, and the restart at every
packed sequence.
"""

import numpy as np
import pytest
from scipy.special import softmax

import oracle


def _inputs(rng, B, T, H, dk, dv):
    return (rng.standard_normal((B, T, H, dk)), rng.standard_normal((B, T, H, dk)),
            rng.standard_normal((B, T, H, dv)))


def test_feature_map_is_softmax():
    x = np.random.default_rng(0).standard_normal((3, 5, 2, 7)) * 4
    np.testing.assert_allclose(oracle.softmax_features(x), softmax(x, axis=-1), rtol=1e-13)


@pytest.mark.parametrize("window", [0, 1, 3])
def test_rla_double_sum(window):
    rng = np.random.default_rng(1 + window)
    q, k, v = _inputs(rng, 1, 9, 2, 3, 4)
    o = oracle.rla(q, k, v, window)
    fq, fk = softmax(q, axis=-1), softmax(k, axis=-1)
    ref = np.zeros_like(o)
    for t in range(9):
        for m in range(t - window):                    # m <= t - window - 1
            for h in range(2):
                ref[0, t, h] += np.dot(fq[0, t, h], fk[0, m, h]) * v[0, m, h]
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-14)


def test_rla_without_delay_is_undecayed_retention_shifted_by_one():
    """window = -1 would read S_t; window = 0 reads S_(t-1): the gamma = 1
    parallel form on the features with keys and values shifted by one token."""
    rng = np.random.default_rng(5)
    q, k, v = _inputs(rng, 2, 12, 1, 4, 3)
    o = oracle.rla(q, k, v, 0)
    fq, fk = oracle.softmax_features(q), oracle.softmax_features(k)
    ks = np.zeros_like(fk)
    vs = np.zeros_like(v)
    ks[:, 1:], vs[:, 1:] = fk[:, :-1], v[:, :-1]
    np.testing.assert_allclose(o, oracle.msr_parallel(fq, ks, vs, [1.0]), rtol=1e-12, atol=1e-14)


def test_rla_window_past_the_sequence_is_zero():
    rng = np.random.default_rng(6)
    q, k, v = _inputs(rng, 1, 6, 1, 2, 2)
    assert np.all(oracle.rla(q, k, v, 5) == 0.0)
    assert np.any(oracle.rla(q, k, v, 4) != 0.0)


def test_rla_packed_sequences_restart():
    rng = np.random.default_rng(7)
    q, k, v = _inputs(rng, 1, 13, 2, 3, 2)
    cu = [0, 6, 6, 13]
    o = oracle.rla(q, k, v, 1, cu_seqlens=cu)
    np.testing.assert_allclose(o[:, 0:6], oracle.rla(q[:, 0:6], k[:, 0:6], v[:, 0:6], 1), rtol=0, atol=0)
    np.testing.assert_allclose(o[:, 6:13], oracle.rla(q[:, 6:13], k[:, 6:13], v[:, 6:13], 1), rtol=0, atol=0)
