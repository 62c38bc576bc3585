"""Pins of the oracle's layer-edge functions (oracle.layer_edges, oracle.rms_norm) against facts
that hold independently of their formulas."""
import numpy as np
import pytest

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


def test_known_values():
    """Exact values at ln 3 (e^x = 3) and 0, independent of how the maps are written."""
    l3 = np.log(3.0)
    np.testing.assert_allclose(oracle.sigmoid(np.array([l3, -l3])), [0.75, 0.25], rtol=1e-15)
    np.testing.assert_allclose(oracle.softplus(np.array([0.0, l3, -l3])), [np.log(2.0), np.log(4.0), np.log(4.0 / 3.0)],
                               rtol=1e-15)
    _, _, alpha, b, w = oracle.layer_edges(np.ones((1, 4)), np.ones((1, 4)), np.array([l3]), np.array([l3]),
                                           np.array([-l3]))
    np.testing.assert_allclose([alpha[0], b[0], w[0]], [0.25, 0.75, 0.25], rtol=1e-15)


def test_derivatives(rng):
    """sigmoid' = sigmoid (1 - sigmoid) and softplus' = sigmoid, by central differences."""
    x = rng.normal(scale=3.0, size=200)
    h = 1e-5
    s = oracle.sigmoid(x)
    np.testing.assert_allclose((oracle.sigmoid(x + h) - oracle.sigmoid(x - h)) / (2 * h), s * (1 - s), atol=1e-9)
    np.testing.assert_allclose((oracle.softplus(x + h) - oracle.softplus(x - h)) / (2 * h), s, atol=1e-9)
    # softplus(x) - softplus(-x) = x
    np.testing.assert_allclose(oracle.softplus(x) - oracle.softplus(-x), x, atol=1e-12)


def test_layer_edges_route_each_input(rng):
    """Distinct raw inputs: each output depends on its own input only, through its own map."""
    T, K, V = 9, 16, 8
    qr, kr = rng.normal(size=(T, K)), 5.0 * rng.normal(size=(T, K))
    a, bl, wl = rng.normal(size=(T, K)), rng.normal(size=(T, K)), rng.normal(size=(T, V))
    q, k, alpha, b, w = oracle.layer_edges(qr, kr, a, bl, wl)
    for y, x in ((q, qr), (k, kr)):
        np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, rtol=1e-14)
        np.testing.assert_allclose(np.sum(y * x, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    # alpha = sigmoid(-a) = 1 - sigmoid(a);  gates are sigmoids of their own logits
    np.testing.assert_allclose(alpha + oracle.sigmoid(a), 1.0, atol=1e-15)
    np.testing.assert_allclose(b + oracle.sigmoid(-bl), 1.0, atol=1e-15)
    np.testing.assert_allclose(w + oracle.sigmoid(-wl), 1.0, atol=1e-15)
    assert b.shape == (T, K) and w.shape == (T, V)


PIN_TESTS = ("test_sigmoid_and_decay_identities", "test_l2_normalize", "test_rms_norm", "test_known_values",
             "test_derivatives", "test_layer_edges_route_each_input")

_sig, _sp, _l2, _rms, _edges = (oracle.sigmoid, oracle.softplus, oracle.l2_normalize, oracle.rms_norm,
                                oracle.layer_edges)
EDGE_MUTANTS = {
    "sigmoid_scale": ("sigmoid", lambda x: 0.5 * (1.0 + np.tanh(np.asarray(x, dtype=np.float64)))),
    "sigmoid_sign": ("sigmoid", lambda x: 0.5 * (1.0 - np.tanh(0.5 * np.asarray(x, dtype=np.float64)))),
    "softplus_sign": ("softplus", lambda x: np.logaddexp(0.0, -np.asarray(x, dtype=np.float64))),
    "softplus_no_log": ("softplus", lambda x: np.maximum(np.asarray(x, dtype=np.float64), 0.0)),
    "l2_squared": ("l2_normalize",
                   lambda x, eps=oracle.NORM_EPS: x / np.maximum(np.sum(x * x, axis=-1, keepdims=True), eps)),
    "l2_eps_added": ("l2_normalize",
                     lambda x, eps=oracle.NORM_EPS: x / (np.linalg.norm(x, axis=-1, keepdims=True) + eps)),
    "l2_wrong_axis": ("l2_normalize",
                      lambda x, eps=oracle.NORM_EPS: x / np.maximum(np.linalg.norm(x, axis=0, keepdims=True), eps)),
    "rms_sum": ("rms_norm", lambda o, wt, eps=oracle.RMS_EPS: o / np.sqrt(np.sum(o * o, axis=-1, keepdims=True) + eps)
                * wt),
    "rms_eps_outside": ("rms_norm", lambda o, wt, eps=oracle.RMS_EPS: o / (np.sqrt(np.mean(o * o, axis=-1,
                                                                                             keepdims=True)) + eps) * wt),
    "rms_no_weight": ("rms_norm", lambda o, wt, eps=oracle.RMS_EPS: _rms(o, np.ones_like(wt), eps)),
    "decay_sign": ("layer_edges", lambda qr, kr, a, bl, wl: (_l2(qr), _l2(kr), np.exp(-_sp(-np.asarray(a))),
                                                             _sig(bl), _sig(wl))),
    "gates_swapped": ("layer_edges", lambda qr, kr, a, bl, wl: (_l2(qr), _l2(kr), np.exp(-_sp(a)), _sig(wl[..., :1])
                                                                * np.ones_like(bl), _sig(wl))),
    "q_not_normalised": ("layer_edges", lambda qr, kr, a, bl, wl: (np.asarray(qr, dtype=np.float64), _l2(kr),
                                                                   np.exp(-_sp(a)), _sig(bl), _sig(wl))),
}


@pytest.mark.parametrize("name", sorted(EDGE_MUTANTS))
def test_edge_pins_catch_mutant(monkeypatch, rng, name):
    """Each planted mistake in an edge map fails at least one of the pins above."""
    attr, fn = EDGE_MUTANTS[name]
    monkeypatch.setattr(oracle, attr, fn)
    caught = []
    for t in PIN_TESTS:
        f = globals()[t]
        try:
            f(rng) if f.__code__.co_argcount else f()
        except AssertionError:
            caught.append(t)
    assert caught, f"mutant {name} passes every edge pin"
