"""Pins of the layer-step oracle (oracle/layer.py) against what the definitions
fix: a delta filter is the identity or a shift, the convolution equals numpy's
own full convolution per channel, a packed batch equals separate sequences,
Swish matches scipy's logistic function, normalised vectors have unit length
and the RMSNorm is scale invariant."""
import numpy as np
import pytest
from scipy.special import expit

from oracle import layer


def _rng(seed):
    return np.random.default_rng(seed)


def test_delta_filter_at_current_tap_is_identity():
    x = _rng(1).normal(size=(9, 2, 4))
    w = np.zeros((8, 4))
    w[:, 3] = 1.0
    np.testing.assert_allclose(layer.causal_conv4(x, w), x, rtol=0, atol=0)


def test_delta_filter_one_tap_back_is_a_shift_within_each_sequence():
    x = _rng(2).normal(size=(10, 1, 3))
    w = np.zeros((3, 4))
    w[:, 2] = 1.0
    cu = [0, 4, 10]
    y = layer.causal_conv4(x, w, cu)
    for s0, s1 in ((0, 4), (4, 10)):
        np.testing.assert_array_equal(y[s0], 0.0)           # nothing before a sequence
        np.testing.assert_array_equal(y[s0 + 1:s1], x[s0:s1 - 1])


def test_conv_equals_numpy_convolution_per_channel():
    T, H, d = 23, 2, 5
    x = _rng(3).normal(size=(T, H, d))
    w = _rng(4).normal(size=(H * d, 4))
    y = layer.causal_conv4(x, w)
    for h in range(H):
        for c in range(d):
            # np.convolve flips its second argument: tap 3 (current) first
            ref = np.convolve(x[:, h, c], w[h * d + c, ::-1])[:T]
            np.testing.assert_allclose(y[:, h, c], ref, rtol=1e-13, atol=1e-13)


def test_packed_batch_equals_separate_sequences():
    lens = [5, 1, 0, 8]
    cu = np.concatenate([[0], np.cumsum(lens)])
    x = _rng(5).normal(size=(cu[-1], 3, 4))
    w = _rng(6).normal(size=(12, 4))
    y = layer.causal_conv4(x, w, cu)
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        if b > a:
            np.testing.assert_allclose(y[a:b], layer.causal_conv4(x[a:b], w), rtol=0, atol=0)


def test_swish_matches_logistic_and_limits():
    x = np.linspace(-30, 30, 121)
    np.testing.assert_allclose(layer.swish(x), x * expit(x), rtol=1e-14, atol=1e-300)
    assert layer.swish(np.array([0.0]))[0] == 0.0
    assert abs(layer.swish(np.array([40.0]))[0] - 40.0) < 1e-12
    assert abs(layer.swish(np.array([-40.0]))[0]) < 1e-15


def test_l2_normalize_unit_length_and_direction():
    x = _rng(7).normal(size=(6, 3, 16))
    y = layer.l2_normalize(x, eps=0.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, rtol=1e-14)
    cos = (x * y).sum(-1) / np.linalg.norm(x, axis=-1)
    np.testing.assert_allclose(cos, 1.0, rtol=1e-14)
    # eps only matters for tiny vectors
    assert np.all(layer.l2_normalize(np.zeros((1, 1, 4)), eps=1e-6) == 0.0)


def test_output_norm_gate_properties():
    o = _rng(8).normal(size=(5, 2, 32))
    ones = np.ones(32)
    open_gate = np.full_like(o, 50.0)            # sigmoid = 1 to double precision
    y = layer.output_norm_gate(o, open_gate, ones, eps=0.0)
    np.testing.assert_allclose(np.sqrt((y * y).mean(-1)), 1.0, rtol=1e-14)
    # scale invariance of the RMSNorm, gate 0 halves, the weight scales channels
    np.testing.assert_allclose(layer.output_norm_gate(3.5 * o, open_gate, ones, eps=0.0), y,
                               rtol=1e-13)
    half = layer.output_norm_gate(o, np.zeros_like(o), ones, eps=0.0)
    np.testing.assert_allclose(half, 0.5 * y, rtol=1e-14)
    w = np.arange(32, dtype=np.float64)
    np.testing.assert_allclose(layer.output_norm_gate(o, open_gate, w, eps=0.0), y * w,
                               rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("eps", [1e-6])
def test_qkv_conv_norm_composes_the_steps(eps):
    T, H, d = 12, 2, 8
    r = _rng(9)
    xq, xk, xv = (r.normal(size=(T, H, d)) for _ in range(3))
    wq, wk, wv = (r.normal(size=(H * d, 4)) for _ in range(3))
    q, k, v = layer.qkv_conv_norm(xq, xk, xv, wq, wk, wv, eps=eps)
    sq = layer.swish(layer.causal_conv4(xq, wq))
    np.testing.assert_allclose(q, sq / np.sqrt((sq ** 2).sum(-1, keepdims=True) + eps))
    np.testing.assert_allclose(v, layer.swish(layer.causal_conv4(xv, wv)))
    assert np.all(np.linalg.norm(k, axis=-1) <= 1.0)
