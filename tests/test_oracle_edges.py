"""Pins of the oracle's layer-edge functions (oracle.layer_edges, oracle.rms_norm) against facts
that hold independently of their formulas."""
import numpy as np

import oracle


def test_sigmoid_and_decay_identities(rng):
    x = rng.normal(scale=4.0, size=1000)
    s = oracle.sigmoid(x)
    assert oracle.sigmoid(np.array([0.0]))[0] == 0.5
    np.testing.assert_allclose(s + oracle.sigmoid(-x), 1.0, atol=1e-15)
    np.testing.assert_allclose(s, 1.0 / (1.0 + np.exp(-x)), rtol=1e-9, atol=1e-16)
    # exp(-softplus(a)) = 1 / (1 + e^a) = sigmoid(-a): the decay lies in (0, 1)
    _, _, alpha, _, _ = oracle.layer_edges(x[:4], x[:4], x, x, x)
    np.testing.assert_allclose(alpha, 1.0 / (1.0 + np.exp(x)), rtol=1e-9, atol=1e-16)
    assert np.all((alpha > 0) & (alpha < 1))


def test_l2_normalize(rng):
    x = rng.normal(size=(50, 128))
    y = oracle.l2_normalize(x)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(y * np.linalg.norm(x, axis=-1, keepdims=True), x, rtol=1e-13)
    # below eps the vector is divided by eps, not blown up
    tiny = np.full((1, 128), 1e-9)
    np.testing.assert_allclose(oracle.l2_normalize(tiny), tiny / 1e-6)


def test_rms_norm(rng):
    o = rng.normal(scale=3.0, size=(20, 128))
    ones = np.ones(128)
    y = oracle.rms_norm(o, ones)
    ms = np.mean(o * o, axis=-1)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), ms / (ms + oracle.RMS_EPS), rtol=1e-13)
    w = rng.normal(size=128)
    np.testing.assert_allclose(oracle.rms_norm(o, w), y * w, rtol=1e-13)
    # scale invariance (up to eps)
    np.testing.assert_allclose(oracle.rms_norm(10.0 * o, ones), y, rtol=1e-6)
