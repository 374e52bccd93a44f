"""Pins of the oracle's AdamW (vector-valued parameters; CPU).

The MONA page assigns embeddings and biases to standard AdamW without
formulas; the reading (bias-corrected Adam, decoupled weight decay) is pinned
by a two-step hand-worked example, the sign-like first step (bias correction
makes m_hat = g and v_hat = g^2 whatever the betas), pure decay at zero
gradient, and the beta = 0 case.
"""
import numpy as np
import pytest

import oracle
from conftest import load_golden


def test_adamw_hand_example_two_steps():
    g = load_golden("adamw_hand_2.txt")
    hp = dict(lr=g["lr"], beta1=g["beta1"], beta2=g["beta2"], eps=g["eps"], weight_decay=g["weight_decay"])
    W, m, v = oracle.adamw(g["W0"], g["G1"], np.zeros(2), np.zeros(2), step=1, **hp)
    assert np.allclose(m, g["m1"], rtol=0, atol=1e-15) and np.allclose(v, g["v1"], rtol=0, atol=1e-15)
    assert np.allclose(W, g["W1"], rtol=0, atol=1e-15)
    W, m, v = oracle.adamw(W, g["G2"], m, v, step=2, **hp)
    assert np.allclose(m, g["m2"], rtol=0, atol=1e-15) and np.allclose(v, g["v2"], rtol=0, atol=1e-15)
    assert np.allclose(W, g["W2"], rtol=0, atol=1e-14)


@pytest.mark.parametrize("b1,b2", [(0.9, 0.999), (0.5, 0.5), (0.0, 0.0)])
def test_adamw_first_step_is_sign_like(b1, b2):
    rng = np.random.default_rng(2)
    G = rng.standard_normal(50) * 10.0 ** rng.integers(-3, 3, 50)
    W0 = rng.standard_normal(50)
    W, m, v = oracle.adamw(W0, G, np.zeros(50), np.zeros(50), lr=0.01, beta1=b1, beta2=b2, eps=0.0,
                           weight_decay=0.0, step=1)
    assert np.allclose(W, W0 - 0.01 * np.sign(G), rtol=0, atol=1e-15)


def test_adamw_zero_gradient_is_pure_decay():
    W0 = np.array([1.0, -3.0, 0.25])
    W, m, v = oracle.adamw(W0, np.zeros(3), np.zeros(3), np.zeros(3), lr=0.1, beta1=0.9, beta2=0.99, eps=1e-8,
                           weight_decay=0.2, step=5)
    assert np.allclose(W, W0 * (1 - 0.1 * 0.2), rtol=0, atol=1e-15)
    assert np.all(m == 0) and np.all(v == 0)


def test_adamw_no_momentum_case():
    # beta1 = beta2 = 0: m = g, v = g^2, no bias correction left: update g / (|g| + eps)
    rng = np.random.default_rng(4)
    G, W0, m0, v0 = (rng.standard_normal(20) for _ in range(4))
    W, m, v = oracle.adamw(W0, G, m0, np.abs(v0), lr=0.05, beta1=0.0, beta2=0.0, eps=0.1, weight_decay=0.0,
                           step=3)
    assert np.allclose(m, G, rtol=0, atol=0) and np.allclose(v, G * G, rtol=1e-15, atol=0)
    assert np.allclose(W, W0 - 0.05 * G / (np.abs(G) + 0.1), rtol=0, atol=1e-15)
