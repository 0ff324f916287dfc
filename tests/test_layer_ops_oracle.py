"""Pins for the fp64 reference of the operations around the recurrence (oracle/layer_ops.py).

Each check follows from the definition the pages give, or from the mathematics, not
from re-typing the oracle's formula: unit length after L2 normalisation, the values
of the activations at fixed points and their symmetries, RMSNorm of a constant
vector, the gate halving at a zero pre-activation, the convolution's impulse response
and its restart at sequence boundaries.
"""

from __future__ import annotations

import math

import numpy as np
import pytest

from oracle import layer_ops as L


def test_l2_normalize_gives_unit_rows_along_the_same_direction():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, 3, 128))
    y = L.l2_normalize(x)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, rtol=1e-12)
    # same direction: y is a positive multiple of x
    ratio = y / x
    np.testing.assert_allclose(ratio, np.broadcast_to(ratio[..., :1], ratio.shape), rtol=1e-10)
    assert np.all(ratio > 0)
    # scale invariance
    np.testing.assert_allclose(L.l2_normalize(5.5 * x), y, rtol=1e-12)
    # a zero row stays zero (the epsilon only guards the division)
    assert np.all(L.l2_normalize(np.zeros(128)) == 0.0)


def test_activations_at_fixed_points_and_symmetries():
    assert L.sigmoid(0.0) == 0.5
    x = np.linspace(-30, 30, 121)
    np.testing.assert_allclose(L.sigmoid(-x), 1.0 - L.sigmoid(x), rtol=0, atol=1e-15)
    # logsigmoid is log of sigmoid, never positive, -log 2 at 0, ~x for very negative x,
    # ~ -e^{-x} for large x
    np.testing.assert_allclose(L.logsigmoid(x[np.abs(x) < 20]),
                               np.log(L.sigmoid(x[np.abs(x) < 20])), rtol=1e-12, atol=1e-15)
    assert np.all(L.logsigmoid(x) <= 0.0)
    assert L.logsigmoid(0.0) == pytest.approx(-math.log(2.0), rel=1e-15)
    assert L.logsigmoid(-50.0) == pytest.approx(-50.0, rel=1e-15)
    assert L.logsigmoid(40.0) == pytest.approx(-math.exp(-40.0), rel=1e-12)
    # Swish: 0 at 0, x sigma(x), -> x for large x, odd part x/2
    assert L.swish(0.0) == 0.0
    assert L.swish(40.0) == pytest.approx(40.0, rel=1e-12)
    np.testing.assert_allclose(L.swish(x) - L.swish(-x), x, rtol=0, atol=1e-12)


def test_rms_norm_of_constant_and_scaled_vectors():
    w = np.linspace(0.5, 1.5, 128)
    for c in (3.0, -0.25):
        y = L.rms_norm(np.full(128, c), w)
        # mean of squares is c^2, so the result is sign(c) w (up to the epsilon)
        np.testing.assert_allclose(y, np.sign(c) * w, rtol=1e-6 / c ** 2 + 1e-12)
    rng = np.random.default_rng(2)
    o = rng.standard_normal((5, 4, 128))
    y = L.rms_norm(o, np.ones(128))
    np.testing.assert_allclose(np.mean(y * y, axis=-1), 1.0, rtol=1e-5)
    # (equal up to the epsilon, which matters ~eps / (2 mean o^2) ~ 5e-7 here)
    np.testing.assert_allclose(L.rms_norm(100.0 * o, np.ones(128)), y, rtol=5e-6)


def test_output_gate_halves_at_zero_and_closes_and_opens():
    rng = np.random.default_rng(3)
    o = rng.standard_normal((6, 128))
    w = rng.random(128) + 0.5
    base = L.rms_norm(o, w)
    np.testing.assert_allclose(L.output_gate(o, w, np.zeros((6, 128))), 0.5 * base, rtol=1e-15)
    assert np.all(np.abs(L.output_gate(o, w, np.full((6, 128), -60.0))) < 1e-20)
    np.testing.assert_allclose(L.output_gate(o, w, np.full((6, 128), 60.0)), base, rtol=1e-12)


def test_short_conv_impulse_response_and_identity():
    C = 5
    rng = np.random.default_rng(4)
    w = rng.standard_normal((C, 4))
    x = np.zeros((9, C))
    x[2] = 1.0
    y = L.short_conv(x, w)
    # the impulse at token 2 reaches tokens 2..5 through taps 3, 2, 1, 0
    for t in range(9):
        expect = w[:, 3 - (t - 2)] if 2 <= t <= 5 else np.zeros(C)
        np.testing.assert_array_equal(y[t], expect)
    # the filter [0, 0, 0, 1] is the identity
    ident = np.zeros((C, 4))
    ident[:, 3] = 1.0
    z = rng.standard_normal((11, C))
    np.testing.assert_array_equal(L.short_conv(z, ident), z)
    # the filter [1, 0, 0, 0] shifts by three tokens
    shift = np.zeros((C, 4))
    shift[:, 0] = 1.0
    np.testing.assert_array_equal(L.short_conv(z, shift)[3:], z[:-3])
    np.testing.assert_array_equal(L.short_conv(z, shift)[:3], 0.0)


def test_short_conv_restarts_at_each_sequence():
    rng = np.random.default_rng(5)
    C = 3
    w = rng.standard_normal((C, 4))
    a, b = rng.standard_normal((6, C)), rng.standard_normal((4, C))
    packed = L.short_conv(np.concatenate([a, b]), w, cu_seqlens=[0, 6, 10])
    np.testing.assert_array_equal(packed[:6], L.short_conv(a, w))
    np.testing.assert_array_equal(packed[6:], L.short_conv(b, w))
    # and Swish after it
    np.testing.assert_array_equal(L.short_conv_swish(b, w), L.swish(L.short_conv(b, w)))


def test_fused_layer_reduces_to_the_recurrence():
    """With inputs already of unit length, pre-activations whose activations give back
    fixed gates, a unit norm weight and an open output gate, the composed function is
    RMSNorm of the plain recurrence; with the identity filter the convolution + Swish
    step is Swish alone."""
    import oracle
    rng = np.random.default_rng(6)
    T, H, d = 20, 2, 128
    q = rng.standard_normal((T, H, d))
    k = rng.standard_normal((T, H, d))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, d))
    x = rng.standard_normal((T, H, d)) + 3.0
    b = rng.standard_normal((T, H))
    o_f, h_f = L.fused_layer_forward(q, k, v, x, b, np.full((T, H, d), 60.0), np.ones(d))
    o_r, h_r = oracle.oracle_forward(q, k, v, L.logsigmoid(x), L.sigmoid(b))
    np.testing.assert_allclose(h_f, h_r, rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(o_f, L.rms_norm(o_r, np.ones(d)), rtol=1e-5, atol=1e-8)
    ident = np.zeros((H * d, 4))
    ident[:, 3] = 1.0
    o_c, _ = L.fused_layer_forward(q, k, v, x, b, np.zeros((T, H, d)), np.ones(d),
                                   conv_w={"q": ident, "k": ident, "v": ident})
    o_s, _ = oracle.oracle_forward(L.l2_normalize(L.swish(q)), L.l2_normalize(L.swish(k)),
                                   L.swish(v), L.logsigmoid(x), L.sigmoid(b))
    np.testing.assert_allclose(o_c, 0.5 * L.rms_norm(o_s, np.ones(d)), rtol=1e-5, atol=1e-8)
