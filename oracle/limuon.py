"""fp64 CPU oracle of the LiMuon step: momentum, then a randomized truncated SVD
in place of the Newton-Schulz orthogonalisation.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module; the product path never does.  It
shares no code with the CUDA library.

Source: the LiMuon page (arxiv.sitesynth.xyz digest 2509.14562v1, "LiMuon:
Light and Fast Muon Optimizer for Large Models"), section "Метод" (method):
LiMuon keeps Muon's momentum and computes the update from a randomized SVD of
the momentum.  The page gives no formulas; the reading followed here:

  1. M <- mu M + G: the heavy-ball momentum of the Muon update (MONA page,
     section 2, step 4, with alpha = 0).
  2. The basic randomized SVD of Halko, Martinsson and Tropp ("Finding
     structure with randomness", 2011, the two-stage prototype): a Gaussian
     test matrix Omega (cols x k, k = r + p with p oversampling columns) is an
     input; Y = M Omega; Q = an orthonormal basis of range(Y) (thin QR).
  3. B = Q^T M (k x cols) and its SVD B = U~ S V^T; U = Q U~.
  4. O = U_r V_r^T over the r largest singular values: the orthogonal factor
     of the rank-r approximation, as the polar factor U V^T is Muon's.
     Singular values at or below TAU * s_1 count as zero and are left out, so
     a rank-deficient M gives a partial isometry and a zero M gives O = 0.
  5. W <- W - eta (gamma O + lambda W) (MONA page, section 2, step 4).

numpy's QR and SVD serve as library steps; everything is fp64.
"""
import numpy as np

# singular values at or below TAU * (largest) count as zero
TAU = 1e-5


def momentum(M, G, mu):
    """Step 1: M' = mu M + G, elementwise in fp64."""
    return mu * np.asarray(M, np.float64) + np.asarray(G, np.float64)


def range_basis(M, Omega):
    """Step 2: Q, an orthonormal basis of range(M Omega) (rows x k)."""
    Y = np.asarray(M, np.float64) @ np.asarray(Omega, np.float64)
    Q, _ = np.linalg.qr(Y, mode="reduced")
    return Q


def rsvd_orthogonal(M, Omega, rank):
    """Steps 2-4: O = U_r V_r^T of the randomized SVD of M (rows x cols) with
    the test matrix Omega (cols x k); rank r <= k."""
    M = np.asarray(M, np.float64)
    Omega = np.asarray(Omega, np.float64)
    if Omega.shape[0] != M.shape[1] or not 1 <= rank <= Omega.shape[1]:
        raise ValueError("Omega must be cols x k with 1 <= rank <= k")
    Q = range_basis(M, Omega)
    B = Q.T @ M
    Ub, S, Vt = np.linalg.svd(B, full_matrices=False)
    if S.size == 0 or S[0] == 0.0:
        return np.zeros_like(M)
    keep = [i for i in range(min(rank, S.size)) if S[i] > TAU * S[0]]
    U = Q @ Ub[:, keep]
    return U @ Vt[keep, :]


def weight_update(W, O, eta, gamma, lam):
    """Step 5: W' = W - eta (gamma O + lambda W)."""
    W = np.asarray(W, np.float64)
    return W - eta * (gamma * O + lam * W)


def limuon_step(W, G, M, Omega, *, mu, eta, lam, gamma, rank):
    """One LiMuon step on one matrix; returns dict(W, M, O) in fp64."""
    Mn = momentum(M, G, mu)
    O = rsvd_orthogonal(Mn, Omega, rank)
    return dict(W=weight_update(W, O, eta, gamma, lam), M=Mn, O=O)
