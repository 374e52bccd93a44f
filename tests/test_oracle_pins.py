"""Pins of the fp64 CPU oracle to facts outside itself (no GPU needed).

Each check ties one oracle function to something the pages or mathematics fix:
hand-worked examples of the MONA equations (MONA page, section 2, steps 1-4),
closed forms of the polar factor (quant_prune_distill post 677, opening
paragraph: polar(X) = U V^T), the action of a matrix polynomial iteration on
singular values, invariants of the polar decomposition, and LAPACK's SVD
(numpy) on small inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import load_golden, rel_fro

QUINTIC = (3.4445, -4.7750, 2.0315)


def _rng(seed):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------- rounding

def test_round_bf16_matches_torch_on_float32_values():
    # values exactly representable in float32, so torch rounds once (RNE)
    rng = _rng(1)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-40, 38, 20000),
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, -3.4e38, 1e-40, -1e-45]),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_round_fp16_matches_numpy():
    rng = _rng(2)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 6, 20000),
        np.array([0.0, 65504.0, 65519.99, 6e-8, 3e-8, 2.98e-8, 1.0 + 2 ** -11]),
    ])
    ref = x.astype(np.float16).astype(np.float64)
    got = oracle.round_fp16(x)
    np.testing.assert_array_equal(got, ref)


def test_round_fp32_matches_numpy():
    rng = _rng(3)
    x = rng.standard_normal(20000) * 10.0 ** rng.integers(-45, 38, 20000)
    ref = x.astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(oracle.round_fp32(x), ref)


# ----------------------------------------------------------------- MONA

def test_mona_hand_example():
    g = load_golden("mona_hand_2x2.txt")
    Gp, A, M = oracle.mona(g["G"], g["G_prev"], g["A"], g["M"], g["beta_a"], g["alpha"], g["mu"])
    np.testing.assert_allclose(A, g["A_new"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(M, g["M_new"], rtol=0, atol=1e-14)
    np.testing.assert_array_equal(Gp, g["G_prev_new"])


def test_weight_update_hand_example():
    g = load_golden("weight_update_hand_2x2.txt")
    W = oracle.weight_update(g["W"], g["O"], g["eta"], g["gamma"], g["lambda"])
    np.testing.assert_allclose(W, g["W_new"], rtol=0, atol=1e-15)


def test_mona_special_cases():
    rng = _rng(4)
    G, Gp, A, M = (rng.standard_normal(257) for _ in range(4))
    # alpha = 0: plain heavy-ball Muon momentum
    _, _, Mn = oracle.mona(G, Gp, A, M, 0.9, 0.0, 0.95)
    np.testing.assert_allclose(Mn, 0.95 * M + G, rtol=0, atol=1e-14)
    # mu = 0: M' = G + alpha*A'
    _, An, Mn = oracle.mona(G, Gp, A, M, 0.9, 0.5, 0.0)
    np.testing.assert_allclose(Mn, G + 0.5 * An, rtol=0, atol=1e-14)
    # beta_a = 1: acceleration buffer unchanged
    _, An, _ = oracle.mona(G, Gp, A, M, 1.0, 0.5, 0.9)
    np.testing.assert_array_equal(An, A)
    # beta_a = 0: A' is the raw difference
    _, An, _ = oracle.mona(G, Gp, A, M, 0.0, 0.5, 0.9)
    np.testing.assert_allclose(An, G - Gp, rtol=0, atol=1e-15)
    # equal consecutive gradients and zero buffers: D = 0 => A' = 0, M' = G
    _, An, Mn = oracle.mona(G, G, 0 * A, 0 * M, 0.9, 0.5, 0.95)
    np.testing.assert_array_equal(An, 0 * A)
    np.testing.assert_array_equal(Mn, G)


def test_weight_update_special_cases():
    rng = _rng(5)
    W, O = rng.standard_normal(100), rng.standard_normal(100)
    np.testing.assert_array_equal(oracle.weight_update(W, O, 0.0, 1.0, 0.1), W)
    np.testing.assert_allclose(oracle.weight_update(W, O, 0.02, 1.0, 0.0), W - 0.02 * O,
                               rtol=0, atol=1e-16)


# ----------------------------------------------------------------- polar factor

def _check_polar_invariants(X, P, tol=1e-12):
    rows, cols = X.shape
    if rows >= cols:      # tall: P^T P = I, H = P^T X symmetric PSD, X = P H
        np.testing.assert_allclose(P.T @ P, np.eye(cols), atol=tol)
        H = P.T @ X
    else:                 # wide: P P^T = I, H = X P^T symmetric PSD, X = H P
        np.testing.assert_allclose(P @ P.T, np.eye(rows), atol=tol)
        H = X @ P.T
    np.testing.assert_allclose(H, H.T, atol=tol * np.abs(X).max() * max(rows, cols))
    assert np.linalg.eigvalsh((H + H.T) / 2).min() > -tol * np.abs(X).max()
    Xr = P @ H if rows >= cols else H @ P
    np.testing.assert_allclose(Xr, X, atol=tol * np.abs(X).max() * max(rows, cols))


@pytest.mark.parametrize("shape", [(16, 32), (32, 32), (32, 16), (1, 7), (7, 1), (33, 65)])
def test_polar_matches_lapack_svd(shape):
    X = _rng(6).standard_normal(shape)
    P = oracle.polar(X)
    U, _, Vt = np.linalg.svd(X, full_matrices=False)
    np.testing.assert_allclose(P, U @ Vt, atol=1e-12)
    _check_polar_invariants(X, P)


def test_polar_invariants_ill_conditioned():
    rng = _rng(7)
    s, l = 24, 40
    U, _ = np.linalg.qr(rng.standard_normal((s, s)))
    V, _ = np.linalg.qr(rng.standard_normal((l, s)))
    sig = np.logspace(0, -3, s)
    X = U @ np.diag(sig) @ V.T
    P = oracle.polar(X)
    np.testing.assert_allclose(P, U @ V.T, atol=1e-11)
    _check_polar_invariants(X, P, tol=1e-11)


def test_polar_closed_forms():
    g = load_golden("polar_hand.txt")
    np.testing.assert_allclose(oracle.polar(np.diag(g["diag"])), np.diag(g["diag_polar"]),
                               atol=1e-15)
    np.testing.assert_allclose(oracle.polar(g["X_rot"].reshape(2, 2)),
                               g["X_rot_polar"].reshape(2, 2), atol=1e-15)
    np.testing.assert_allclose(oracle.polar(g["row"].reshape(1, 3)), g["row_polar"].reshape(1, 3),
                               atol=1e-15)
    np.testing.assert_allclose(oracle.polar(g["row"].reshape(3, 1)), g["row_polar"].reshape(3, 1),
                               atol=1e-15)


def test_polar_of_orthogonal_and_scaling():
    rng = _rng(8)
    Q, _ = np.linalg.qr(rng.standard_normal((20, 20)))
    np.testing.assert_allclose(oracle.polar(Q), Q, atol=1e-13)
    X = rng.standard_normal((12, 30))
    P = oracle.polar(X)
    for c in (1e-6, 0.37, 1e5):
        np.testing.assert_allclose(oracle.polar(c * X), P, atol=1e-12)
    # transpose equivariance: polar(X^T) = polar(X)^T
    np.testing.assert_allclose(oracle.polar(X.T), P.T, atol=1e-12)


def test_polar_rank_deficient_is_partial_isometry():
    rng = _rng(9)
    B = rng.standard_normal((10, 3)) @ rng.standard_normal((3, 25))   # rank 3
    P = oracle.polar(B)
    U, S, Vt = np.linalg.svd(B, full_matrices=False)
    np.testing.assert_allclose(P, U[:, :3] @ Vt[:3], atol=1e-10)


# ----------------------------------------------------------------- Newton-Schulz

def _phi(sig, coeffs):
    """Scalar polynomial applied to singular values (closed form of the iteration)."""
    s = np.array(sig, dtype=np.float64)
    for a, b, c in coeffs:
        s = a * s + b * s ** 3 + c * s ** 5
    return s


@pytest.mark.parametrize("shape", [(8, 8), (16, 40), (31, 64), (1, 5)])
def test_ns_poly_closed_form_through_svd(shape):
    # A matrix polynomial iteration X <- p(X X^T) X acts on the singular values
    # only: NS(X) = U phi(S) V^T.  Any transposed operand, wrong side or dropped
    # term in the matrix products breaks this identity.
    rng = _rng(10)
    X = rng.standard_normal(shape)
    X /= np.linalg.norm(X) * 1.01
    coeffs = [QUINTIC] * 5
    Y = oracle.ns_poly(X, coeffs)
    U, S, Vt = np.linalg.svd(X, full_matrices=False)
    np.testing.assert_allclose(Y, U @ np.diag(_phi(S, coeffs)) @ Vt, atol=1e-12)


def test_ns_poly_mixed_schedule_and_prescale():
    rng = _rng(11)
    X = rng.standard_normal((12, 20))
    X /= np.linalg.norm(X)
    coeffs = [QUINTIC] * 3 + [(1.5, -0.5, 0.0)] * 4
    pre = np.ones(7)
    pre[3] = 1 / 1.05
    Y = oracle.ns_poly(X, coeffs, prescale=pre)
    U, S, Vt = np.linalg.svd(X, full_matrices=False)
    s = _phi(S, coeffs[:3]) / 1.05
    s = _phi(s, coeffs[3:])
    np.testing.assert_allclose(Y, U @ np.diag(s) @ Vt, atol=1e-12)


def test_ns_on_orthogonal_input_scales_by_coefficient_sum():
    # sigma = 1 everywhere: one quintic step multiplies by a + b + c = 0.701
    rng = _rng(12)
    Q, _ = np.linalg.qr(rng.standard_normal((16, 16)))
    Y = oracle.ns_poly(Q, [QUINTIC])
    np.testing.assert_allclose(Y, 0.701 * Q, atol=1e-13)


def test_orthogonalise_orientation_and_scale():
    rng = _rng(13)
    M = rng.standard_normal((40, 16))          # tall: iterates on M^T
    O = oracle.orthogonalise(M, [QUINTIC] * 5)
    Ot = oracle.orthogonalise(M.T.copy(), [QUINTIC] * 5)
    np.testing.assert_allclose(O, Ot.T, atol=1e-14)
    # normalisation by the Frobenius norm: positive scaling changes nothing
    O2 = oracle.orthogonalise(1e3 * M, [QUINTIC] * 5)
    np.testing.assert_allclose(O2, O, atol=1e-7)   # eps = 1e-7 shifts the scale by ~eps/|M|
    # same singular vectors as the exact polar factor (closed form again)
    U, S, Vt = np.linalg.svd(M, full_matrices=False)
    s = _phi(S / (np.linalg.norm(M) + 1e-7), [QUINTIC] * 5)
    np.testing.assert_allclose(O, U @ np.diag(s) @ Vt, atol=1e-12)


def test_orthogonalise_zero_matrix_is_zero():
    O = oracle.orthogonalise(np.zeros((8, 12)), [QUINTIC] * 5)
    np.testing.assert_array_equal(O, np.zeros((8, 12)))


def test_five_quintic_steps_are_not_the_polar_factor():
    # The fixed coefficients sum to 0.701, so the iteration leaves singular
    # values spread around 1 instead of converging: tolerances for the
    # 5-step path are taken against the same iteration, not against polar(M).
    rng = _rng(14)
    M = rng.standard_normal((64, 128))
    O = oracle.orthogonalise(M, [QUINTIC] * 5)
    assert rel_fro(O, oracle.polar(M)) > 0.05
    sv = np.linalg.svd(O, compute_uv=False)
    assert 0.6 < sv.min() and sv.max() < 1.2


# ----------------------------------------------------------------- Gram route

CONVERGED = [QUINTIC] * 8 + [(1.5, -0.5, 0.0)] * 6


@pytest.mark.parametrize("restarts,sched", [((), "converged"), ((0, 9), "converged"),
                                             ((0, 3, 9, 12), "converged"),
                                             ((0, 2, 4), "quintic6")])
def test_gram_route_equals_direct_route_in_exact_arithmetic(restarts, sched):
    # X_{k+1} = h_k(X_k X_k^T) X_k whichever way it is evaluated; with
    # restarts the Gram route divides by f exactly where the direct route
    # gets a pre-scale of 1/f.  The 6-step quintic schedule does not converge,
    # so a missing division at a restart cannot wash out.
    coeffs = CONVERGED if sched == "converged" else [QUINTIC] * 6
    rng = _rng(15)
    f = 1.05
    X = rng.standard_normal((20, 48))
    X /= np.linalg.norm(X) * f
    G = oracle.gram_poly(X, coeffs, restarts=restarts, f=f)
    pre = np.ones(len(coeffs))
    for k in restarts:
        if k > 0:
            pre[k] = 1 / f
    D = oracle.ns_poly(X, coeffs, prescale=pre)
    np.testing.assert_allclose(G, D, atol=1e-10)


@pytest.mark.parametrize("kappa", [1e1, 1e2, 1e3])
def test_converged_schedule_reaches_polar(kappa):
    rng = _rng(16)
    s, l = 48, 96
    U, _ = np.linalg.qr(rng.standard_normal((s, s)))
    V, _ = np.linalg.qr(rng.standard_normal((l, s)))
    M = U @ np.diag(np.logspace(0, -np.log10(kappa), s)) @ V.T
    P = oracle.polar(M)
    for route in ("direct", "gram"):
        O = oracle.orthogonalise(M, CONVERGED, route=route, restarts=(0, 9), f=1.05)
        assert rel_fro(O, P) < 1e-9, route


# ----------------------------------------------------------------- full step

def test_muon_step_is_the_composition_of_its_parts():
    # MONA page, section 2: pre-pass (steps 1-4), O = NS(M'), then the update.
    rng = _rng(17)
    rows, cols = 24, 10
    W, G, Gp, A, M = (rng.standard_normal((rows, cols)) for _ in range(5))
    hp = dict(mu=0.95, eta=0.02, lam=0.1, gamma=1.3, beta_a=0.9, alpha=0.5)
    out = oracle.muon_step(W, G, Gp, A, M, coeffs=[QUINTIC] * 5, **hp)
    Gp2, A2, M2 = oracle.mona(G, Gp, A, M, hp["beta_a"], hp["alpha"], hp["mu"])
    O = oracle.orthogonalise(M2, [QUINTIC] * 5)
    W2 = oracle.weight_update(W, O, hp["eta"], hp["gamma"], hp["lam"])
    for k, v in (("G_prev", Gp2), ("A", A2), ("M", M2), ("O", O), ("W", W2)):
        np.testing.assert_array_equal(out[k], v, err_msg=k)
    # the rounded-start variant rounds the (wide view of the) momentum before
    # normalising by the unrounded norm
    outb = oracle.muon_step(W, G, Gp, A, M, coeffs=[QUINTIC] * 5, round_to=oracle.ROUND_BF16, **hp)
    Xr = oracle.round_bf16(M2.T) / (np.linalg.norm(M2) + 1e-7)
    Ob = oracle.ns_poly(Xr, [QUINTIC] * 5).T
    np.testing.assert_allclose(outb["O"], Ob, atol=1e-12)


def test_ns_poly_scalar_table():
    """Singular values 1 and 0.1 follow the composed scalar quintic step by step
    (tests/golden/quintic_scalar_table.txt); a 1 x 1 input x gives sign(x) phi_5(1)."""
    g = load_golden("quintic_scalar_table.txt")
    X = np.diag([1.0, 0.1])
    for k in range(1, 6):
        Y = oracle.ns_poly(X, [QUINTIC] * k)
        assert abs(Y[0, 0] - g["sigma1"][k - 1]) <= 1e-9, k
        assert abs(Y[1, 1] - g["sigma01"][k - 1]) <= 1e-9, k
        assert abs(Y[0, 1]) == 0.0 and abs(Y[1, 0]) == 0.0
    for x in (2.5, -0.3):
        O = oracle.orthogonalise(np.array([[x]]), [QUINTIC] * 5, eps=0.0)
        assert abs(O[0, 0] - np.sign(x) * g["sigma1"][4]) <= 1e-9
