"""Pins of the oracle for the steps before and after the rule (oracle/mixer_io.py):
checks that do not retype its formulas -- a library convolution, closed forms, special
cases and invariants.  CPU only."""

import numpy as np
import pytest

from oracle import mixer_io as mio

RNG = np.random.default_rng(2024)


def _x(B=2, T=11, C=5):
    return RNG.standard_normal((B, T, C))


def test_silu_values():
    # SiLU(0) = 0, SiLU(1) = sigmoid(1), and SiLU(x) - SiLU(-x) = x for every x
    assert mio.silu(0.0) == 0.0
    assert abs(mio.silu(1.0) - 1.0 / (1.0 + np.exp(-1.0))) < 1e-15
    x = np.linspace(-30, 30, 121)
    assert np.allclose(mio.silu(x) - mio.silu(-x), x, rtol=0, atol=1e-12)
    assert np.all(np.isfinite(mio.silu(np.array([-1e4, 1e4]))))


def test_conv_identity_on_the_newest_tap():
    x = _x()
    w = np.zeros((5, 4))
    w[:, 3] = 1.0
    y, _ = mio.short_conv_silu(x, w, state=RNG.standard_normal((2, 5, 3)))
    assert np.allclose(y, mio.silu(x), rtol=0, atol=1e-14)


def test_conv_oldest_tap_shifts_by_three_through_the_state():
    x = _x()
    st = RNG.standard_normal((2, 5, 3))
    w = np.zeros((5, 4))
    w[:, 0] = 1.0
    y, _ = mio.short_conv_silu(x, w, state=st)
    # y_t = SiLU(x_{t-3}); x_{-3..-1} are the state, oldest first
    prev = np.concatenate([np.swapaxes(st, 1, 2), x], axis=1)
    assert np.allclose(y, mio.silu(prev[:, :11]), rtol=0, atol=1e-14)


def test_conv_matches_a_library_convolution():
    x = _x(B=1, T=17, C=3)
    w = RNG.standard_normal((3, 4))
    b = RNG.standard_normal(3)
    y, _ = mio.short_conv_silu(x, w, b)
    for c in range(3):
        # causal full convolution with the taps reversed: np.convolve(x, w[::-1])[t]
        # = sum_i w[3 - i] x[t - i]
        pre = np.convolve(x[0, :, c], w[c, ::-1])[:17] + b[c]
        assert np.allclose(y[0, :, c], mio.silu(pre), rtol=0, atol=1e-12)


def test_conv_bias_only():
    x = _x()
    b = RNG.standard_normal(5)
    y, _ = mio.short_conv_silu(x, np.zeros((5, 4)), b)
    assert np.allclose(y, np.broadcast_to(mio.silu(b), y.shape), rtol=0, atol=1e-15)


def test_conv_streaming_equals_one_pass():
    x = _x(T=23)
    w = RNG.standard_normal((5, 4))
    b = RNG.standard_normal(5)
    st0 = RNG.standard_normal((2, 5, 3))
    y_all, s_all = mio.short_conv_silu(x, w, b, st0)
    y1, s1 = mio.short_conv_silu(x[:, :9], w, b, st0)
    y2, s2 = mio.short_conv_silu(x[:, 9:10], w, b, s1)   # a one-token call, like decode
    y3, s3 = mio.short_conv_silu(x[:, 10:], w, b, s2)
    assert np.array_equal(np.concatenate([y1, y2, y3], axis=1), y_all)
    assert np.array_equal(s3, s_all)
    # the state after a call is the last three inputs
    assert np.array_equal(s_all, np.swapaxes(x[:, -3:], 1, 2))


@pytest.mark.parametrize("d", [32, 128])
def test_rmsnorm_normalised_rows_have_unit_rms(d):
    o = RNG.standard_normal((7, d)) * 3.0
    z = RNG.standard_normal((7, d))
    w = RNG.uniform(0.5, 2.0, d)
    y = mio.gated_rmsnorm(o, z, w, eps=0.0)
    n = y / (w * mio.silu(z))
    assert np.allclose(np.sqrt(np.mean(n * n, axis=-1)), 1.0, rtol=1e-13)
    # and n is a positive multiple of o row by row
    ratio = n / o
    assert np.all(ratio > 0) and np.allclose(ratio, ratio[:, :1], rtol=1e-12)


def test_rmsnorm_constant_rows_and_scale():
    d = 64
    z = RNG.standard_normal((3, d))
    w = RNG.uniform(0.5, 2.0, d)
    o = np.array([2.0, -0.5, 7.0])[:, None] * np.ones((3, d))
    eps = 1e-6
    y = mio.gated_rmsnorm(o, z, w, eps)
    c = o[:, :1]
    expect = c / np.sqrt(c * c + eps) * w * mio.silu(z)
    assert np.allclose(y, expect, rtol=1e-14)
    # scale invariance without eps; a zero gate zeroes the output
    o2 = RNG.standard_normal((3, d))
    assert np.allclose(mio.gated_rmsnorm(5.0 * o2, z, w, 0.0), mio.gated_rmsnorm(o2, z, w, 0.0),
                       rtol=1e-13)
    assert np.all(mio.gated_rmsnorm(o2, np.zeros_like(z), w) == 0.0)
