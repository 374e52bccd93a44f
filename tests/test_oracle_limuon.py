"""Pins of the LiMuon oracle (CPU).

LiMuon (LiMuon page, section "Метод") updates with a randomized SVD of the
momentum, read as O = U_r V_r^T of the Halko-Martinsson-Tropp randomized SVD
(Y = M Omega, Q = orth(Y), B = Q^T M = U~ S V^T, U = Q U~).  The oracle is
pinned by:
  * hand-worked cases (tests/golden/limuon_hand.txt);
  * whenever range(M Omega) holds range(M), the exact rank-r factor of M's own
    SVD: built from a planted SVD (no library SVD involved), and for r at least
    the rank, the independent one-sided Jacobi polar factor of the C oracle;
  * invariances any correct O obeys: O(c M) = O(M) for c > 0 (down to tiny c),
    O(P M) = P O(M) for orthogonal P, O(M P; P^T Omega) = O(M; Omega) P;
  * properties of any sketch: O is a partial isometry with r unit singular
    values and its columns lie in range(M Omega);
  * planted mistakes (at the end) that these pins reject.
"""
import types

import numpy as np
import pytest

import oracle
from conftest import load_golden
from oracle import limuon as lim


def _orth(n, seed):
    q, r = np.linalg.qr(np.random.default_rng(seed).standard_normal((n, n)))
    return q * np.sign(np.diag(r))


def _planted(rows, cols, s, seed):
    """M = U diag(s) V^T with orthonormal U (rows x len(s)) and V (cols x len(s))."""
    U = _orth(rows, seed)[:, :len(s)]
    V = _orth(cols, seed + 1)[:, :len(s)]
    return U @ np.diag(s) @ V.T, U, V


def _omega(cols, k, seed):
    return np.random.default_rng(seed).standard_normal((cols, k))


def test_hand_examples(mod=lim):
    g = load_golden("limuon_hand.txt")
    Md = g["M_diag"].reshape(3, 4)
    Od = g["Omega_diag"].reshape(4, 3)
    for r in (1, 2, 3):
        assert np.allclose(mod.rsvd_orthogonal(Md, Od, r), g[f"O_diag_r{r}"].reshape(3, 4), rtol=0, atol=1e-14)
    Ms = g["M_signs"].reshape(3, 2)
    I2 = g["Omega_I2"].reshape(2, 2)
    for r in (1, 2):
        assert np.allclose(mod.rsvd_orthogonal(Ms, I2, r), g[f"O_signs_r{r}"].reshape(3, 2), rtol=0, atol=1e-14)
    assert np.allclose(mod.rsvd_orthogonal(g["M_rank1"].reshape(2, 2), I2, 2), g["O_rank1_r2"].reshape(2, 2),
                       rtol=0, atol=1e-14)
    # one test column: the sketch keeps only range(M Omega), so O is not M's own top factor
    assert np.allclose(mod.rsvd_orthogonal(g["M_k1"].reshape(2, 3), g["Omega_k1"].reshape(3, 1), 1),
                       g["O_k1_r1"].reshape(2, 3), rtol=0, atol=1e-14)


def test_step_hand_example(mod=lim):
    g = load_golden("limuon_hand.txt")
    out = mod.limuon_step(g["step_W"].reshape(3, 4), g["M_diag"].reshape(3, 4), np.zeros((3, 4)),
                          g["Omega_diag"].reshape(4, 3), mu=g["step_mu"], eta=g["step_eta"],
                          lam=g["step_lambda"], gamma=g["step_gamma"], rank=2)
    assert np.array_equal(out["M"], g["M_diag"].reshape(3, 4))
    assert np.allclose(out["O"], g["O_diag_r2"].reshape(3, 4), rtol=0, atol=1e-14)
    assert np.allclose(out["W"], g["step_W_new"].reshape(3, 4), rtol=0, atol=1e-14)


def test_momentum_closed_form(mod=lim):
    rng = np.random.default_rng(5)
    M, G = rng.standard_normal((4, 6)), rng.standard_normal((4, 6))
    for mu in (0.0, 0.5, 0.95):
        out = mod.momentum(M, G, mu)
        for i in range(4):
            for j in range(6):
                assert out[i, j] == mu * M[i, j] + G[i, j]


@pytest.mark.parametrize("rows,cols,rank,k", [(12, 30, 4, 10), (30, 12, 4, 10), (16, 16, 7, 9),
                                              (20, 48, 12, 12)])
def test_truncation_equals_planted_svd(rows, cols, rank, k, mod=lim):
    # distinct planted singular values; M has rank 12 (or min side), k >= rank(M)
    n = min(rows, cols, 12)
    s = np.linspace(3.0, 0.5, n)
    M, U, V = _planted(rows, cols, s, seed=rows * 100 + cols)
    O = mod.rsvd_orthogonal(M, _omega(cols, max(k, n), seed=7), rank)
    assert np.allclose(O, U[:, :rank] @ V[:, :rank].T, rtol=0, atol=1e-10)


@pytest.mark.parametrize("rows,cols,rho,k,r", [(16, 40, 16, 20, 16), (40, 16, 16, 16, 16),
                                               (12, 30, 5, 8, 8), (25, 9, 3, 6, 5)])
def test_full_rank_request_equals_jacobi_polar(rows, cols, rho, k, r, mod=lim):
    rng = np.random.default_rng(rows + cols + rho)
    M = rng.standard_normal((rows, rho)) @ rng.standard_normal((rho, cols))
    O = mod.rsvd_orthogonal(M, _omega(cols, k, seed=11), r)
    assert np.allclose(O, oracle.polar(M), rtol=0, atol=1e-9)


def test_zero_momentum_gives_zero(mod=lim):
    assert np.array_equal(mod.rsvd_orthogonal(np.zeros((5, 7)), _omega(7, 4, 1), 3), np.zeros((5, 7)))


@pytest.mark.parametrize("c", [1e-9, 1e-3, 7.5, 1e6])
def test_scale_invariance(c, mod=lim):
    rng = np.random.default_rng(3)
    M = rng.standard_normal((14, 33))
    Om = _omega(33, 10, 4)
    assert np.allclose(mod.rsvd_orthogonal(c * M, Om, 6), mod.rsvd_orthogonal(M, Om, 6), rtol=0, atol=1e-10)


def test_orthogonal_invariance(mod=lim):
    rng = np.random.default_rng(8)
    M = rng.standard_normal((14, 33))
    Om = _omega(33, 10, 9)
    O = mod.rsvd_orthogonal(M, Om, 6)
    P = _orth(14, 10)
    assert np.allclose(mod.rsvd_orthogonal(P @ M, Om, 6), P @ O, rtol=0, atol=1e-10)
    R = _orth(33, 12)
    assert np.allclose(mod.rsvd_orthogonal(M @ R, R.T @ Om, 6), O @ R, rtol=0, atol=1e-10)


@pytest.mark.parametrize("rows,cols,k,r", [(30, 50, 12, 8), (50, 30, 12, 12), (64, 64, 20, 3)])
def test_sketch_properties(rows, cols, k, r, mod=lim):
    # rank(M) > k: O approximates, but is always a rank-r partial isometry inside range(M Omega)
    rng = np.random.default_rng(rows * cols)
    M = rng.standard_normal((rows, cols))
    Om = _omega(cols, k, 13)
    O = mod.rsvd_orthogonal(M, Om, r)
    sv = np.linalg.svd(O, compute_uv=False)
    assert np.allclose(sv[:r], 1.0, atol=1e-12) and np.all(sv[r:] < 1e-12)
    Y = M @ Om
    resid = O - Y @ np.linalg.lstsq(Y, O, rcond=None)[0]
    assert np.linalg.norm(resid) < 1e-10 * np.linalg.norm(O)
    # with k = min(rows, cols) the sketch holds the whole range and O is exact
    kk = min(rows, cols)
    s = np.linalg.svd(M, compute_uv=False)
    O_full = mod.rsvd_orthogonal(M, _omega(cols, kk, 14), r)
    assert abs(np.sum(O_full * M) - np.sum(s[:r])) < 1e-9 * np.sum(s[:r])


def test_rank_validated(mod=lim):
    with pytest.raises(ValueError):
        mod.rsvd_orthogonal(np.ones((3, 4)), np.ones((4, 2)), 3)
    with pytest.raises(ValueError):
        mod.rsvd_orthogonal(np.ones((3, 4)), np.ones((3, 2)), 1)


# --- planted mistakes -------------------------------------------------------

MUTATIONS = [
    # (name, original text, planted text, pins that must fail)
    ("keeps_singular_values", "return U @ Vt[keep, :]", "return U @ np.diag(S[keep]) @ Vt[keep, :]",
     [test_hand_examples]),
    ("smallest_r", "keep = [i for i in range(min(rank, S.size))",
     "keep = [i for i in range(S.size - min(rank, S.size), S.size)", [test_hand_examples]),
    ("left_factor_not_rotated", "U = Q @ Ub[:, keep]", "U = Q[:, keep]", [test_hand_examples]),
    ("momentum_sign", "return mu * np.asarray(M, np.float64) + np.asarray(G, np.float64)",
     "return mu * np.asarray(M, np.float64) - np.asarray(G, np.float64)", [test_momentum_closed_form]),
    ("decay_sign", "return W - eta * (gamma * O + lam * W)", "return W - eta * (gamma * O - lam * W)",
     [test_step_hand_example]),
    ("absolute_threshold", "if S[i] > TAU * S[0]]", "if S[i] > TAU]",
     [lambda mod: test_scale_invariance(1e-9, mod)]),
    ("no_orthonormalisation", "Q, _ = np.linalg.qr(Y, mode=\"reduced\")", "Q = Y",
     [lambda mod: test_truncation_equals_planted_svd(12, 30, 4, 10, mod)]),
]


def _mutant(orig, planted):
    src = open(lim.__file__).read()
    assert src.count(orig) == 1, orig
    mod = types.ModuleType("limuon_mutant")
    exec(compile(src.replace(orig, planted), "limuon_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,orig,planted,pins", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(name, orig, planted, pins):
    mod = _mutant(orig, planted)
    for pin in pins:
        with pytest.raises(Exception):
            pin(mod)
