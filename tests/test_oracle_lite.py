"""Pins of the oracle's MONA-Lite functions (CPU).

MONA-Lite (MONA page, section "Efficientie en Implementatie") keeps one
auxiliary buffer B = beta_a A - (1 - beta_a) G of the previous step, in
bfloat16, instead of G_prev and A.  Unrounded, it is MONA rewritten: the
momentum sequence must be the same.  Pinned by hand-worked values, the
algebraic identity over several steps and parameter sets, the bfloat16
storage of B, and the composition of the full step.
"""
import numpy as np
import pytest

import oracle
from conftest import load_golden

QUINTIC = (3.4445, -4.7750, 2.0315)


def test_mona_lite_hand_example():
    g = load_golden("mona_lite_hand_2x2.txt")
    B, M = oracle.mona_lite(g["G"], g["B"], g["M"], g["beta_a"], g["alpha"], g["mu"], round_b=True)
    assert np.array_equal(M.ravel(), g["M_new"])
    assert np.array_equal(B.ravel(), g["B_new"])


def test_mona_lite_reproduces_the_mona_hand_example():
    lite = load_golden("mona_lite_hand_2x2.txt")
    mona = load_golden("mona_hand_2x2.txt")
    # the one-buffer form of the MONA example's state
    B0 = mona["beta_a"] * mona["A"] - (1 - mona["beta_a"]) * mona["G_prev"]
    assert np.allclose(B0, lite["B_of_mona_example"], rtol=0, atol=1e-15)
    B, M = oracle.mona_lite(mona["G"], B0, mona["M"], mona["beta_a"], mona["alpha"], mona["mu"], round_b=False)
    assert np.allclose(M.ravel(), mona["M_new"], rtol=0, atol=1e-14)
    # and B' is the one-buffer form of the MONA example's new state
    expect_B = mona["beta_a"] * mona["A_new"] - (1 - mona["beta_a"]) * mona["G"]
    assert np.allclose(B.ravel(), expect_B, rtol=0, atol=1e-14)


@pytest.mark.parametrize("beta_a,alpha,mu", [(0.9, 0.5, 0.95), (0.0, 1.0, 0.9), (1.0, 0.3, 0.5),
                                             (0.5, 0.0, 0.95), (0.7, 2.0, 0.0)])
def test_mona_lite_equals_mona_without_rounding(beta_a, alpha, mu):
    rng = np.random.default_rng(11)
    shape = (7, 13)
    Gp, A, M = np.zeros(shape), np.zeros(shape), np.zeros(shape)
    B, Ml = np.zeros(shape), np.zeros(shape)
    for k in range(6):
        G = rng.standard_normal(shape) * (1 + k)
        Gp, A, M = oracle.mona(G, Gp, A, M, beta_a, alpha, mu)
        B, Ml = oracle.mona_lite(G, B, Ml, beta_a, alpha, mu, round_b=False)
        scale = max(1.0, np.abs(M).max())
        assert np.abs(Ml - M).max() <= 1e-13 * scale, k
        assert np.abs(B - (beta_a * A - (1 - beta_a) * G)).max() <= 1e-13 * scale, k


def test_mona_lite_stores_b_in_bfloat16():
    rng = np.random.default_rng(3)
    G, B, M = (rng.standard_normal((9, 9)) for _ in range(3))
    B = oracle.round_bf16(B)
    Br, Mr = oracle.mona_lite(G, B, M, 0.9, 0.5, 0.95, round_b=True)
    Bx, Mx = oracle.mona_lite(G, B, M, 0.9, 0.5, 0.95, round_b=False)
    assert np.array_equal(Br, oracle.round_bf16(Bx))      # B stored rounded (RNE) ...
    assert np.array_equal(Mr, Mx)                         # ... M of this step unaffected
    # next step: M sees the rounded B through A_k only
    G2 = rng.standard_normal((9, 9))
    _, M2r = oracle.mona_lite(G2, Br, Mr, 0.9, 0.5, 0.95, round_b=True)
    _, M2x = oracle.mona_lite(G2, Bx, Mx, 0.9, 0.5, 0.95, round_b=False)
    assert np.allclose(M2r - M2x, 0.5 * (Br - Bx), rtol=0, atol=1e-14)   # alpha * (B rounding error)


def test_muon_lite_step_composition():
    rng = np.random.default_rng(5)
    W, G, B, M = (rng.standard_normal((12, 20)) for _ in range(4))
    B = oracle.round_bf16(B)
    hp = dict(mu=0.95, eta=0.02, lam=0.1, gamma=1.0, beta_a=0.9, alpha=0.5)
    out = oracle.muon_lite_step(W, G, B, M, coeffs=[QUINTIC] * 5, **hp)
    B2, M2 = oracle.mona_lite(G, B, M, hp["beta_a"], hp["alpha"], hp["mu"])
    O = oracle.orthogonalise(M2, [QUINTIC] * 5)
    W2 = oracle.weight_update(W, O, hp["eta"], hp["gamma"], hp["lam"])
    assert np.array_equal(out["B"], B2) and np.array_equal(out["M"], M2)
    assert np.array_equal(out["O"], O) and np.array_equal(out["W"], W2)
