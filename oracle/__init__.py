"""fp64 CPU oracle for the Muon / MONA optimizer step (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package; the product path never does.  The
arithmetic lives in ``muon_oracle.c`` (plain C, IEEE double); this module only
marshals numpy arrays.  It shares no code with the CUDA library.

Sources followed (see the C file for the step-by-step citations):
  * MONA page (gist.science, paper 2605.26842), section 2 "Methodologie: MONA",
    steps 1-4 -- the elementwise pre-pass and the weight update.
  * quant_prune_distill post 677 (tgviewer.app) -- polar factor, Newton-Schulz,
    the Gram route X (X^T X)^{-1/2} with restarts and division by 1.02-1.05.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

# coefficients of the quintic step fixed for this optimizer: (a, b, c)
QUINTIC = (3.4445, -4.7750, 2.0315)
# textbook cubic Newton-Schulz for the polar factor (converges for 0 < sigma < sqrt(3))
CUBIC = (1.5, -0.5, 0.0)

ROUND_NONE, ROUND_BF16, ROUND_FP16, ROUND_FP32 = 0, 1, 2, 3

_D = ctypes.POINTER(ctypes.c_double)
_I = ctypes.POINTER(ctypes.c_int)


def configure(L):
    """Declare the C signatures on a loaded oracle library and return it."""
    L.oracle_round_bf16.restype = ctypes.c_double
    L.oracle_round_bf16.argtypes = [ctypes.c_double]
    L.oracle_round_fp16.restype = ctypes.c_double
    L.oracle_round_fp16.argtypes = [ctypes.c_double]
    L.oracle_round_fp32.restype = ctypes.c_double
    L.oracle_round_fp32.argtypes = [ctypes.c_double]
    L.oracle_round_array.argtypes = [_D, ctypes.c_longlong, ctypes.c_int]
    L.oracle_num_threads.restype = ctypes.c_int
    L.oracle_set_num_threads.argtypes = [ctypes.c_int]
    L.oracle_frobenius.restype = ctypes.c_double
    L.oracle_frobenius.argtypes = [_D, ctypes.c_longlong]
    L.oracle_mona.argtypes = [ctypes.c_longlong, _D, _D, _D, _D,
                              ctypes.c_double, ctypes.c_double, ctypes.c_double]
    L.oracle_weight_update.argtypes = [ctypes.c_longlong, _D, _D,
                                       ctypes.c_double, ctypes.c_double, ctypes.c_double]
    L.oracle_ns_poly.argtypes = [_D, ctypes.c_int, ctypes.c_int, ctypes.c_int, _D, _D]
    L.oracle_gram_poly.argtypes = [_D, ctypes.c_int, ctypes.c_int, ctypes.c_int, _D,
                                   _I, ctypes.c_int, ctypes.c_double]
    L.oracle_polar_jacobi.restype = ctypes.c_int
    L.oracle_polar_jacobi.argtypes = [_D, ctypes.c_int, ctypes.c_int, _D]
    L.oracle_polar.restype = ctypes.c_int
    L.oracle_polar.argtypes = [_D, ctypes.c_int, ctypes.c_int, _D]
    L.oracle_orthogonalise.argtypes = [_D, ctypes.c_int, ctypes.c_int, _D, ctypes.c_int,
                                       ctypes.c_int, _D, _I, ctypes.c_int,
                                       ctypes.c_double, ctypes.c_double, ctypes.c_int]
    L.oracle_muon_step.argtypes = [ctypes.c_int, ctypes.c_int, _D, _D, _D, _D, _D, _D,
                                   ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                   ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                   ctypes.c_int, _D, ctypes.c_double, ctypes.c_double,
                                   ctypes.c_int]
    L.oracle_adamw.argtypes = [ctypes.c_longlong, _D, _D, _D, _D, ctypes.c_double, ctypes.c_double,
                               ctypes.c_double, ctypes.c_double, ctypes.c_double, ctypes.c_int]
    L.oracle_mona_lite.argtypes = [ctypes.c_longlong, _D, _D, _D, ctypes.c_double, ctypes.c_double,
                                   ctypes.c_double, ctypes.c_int]
    L.oracle_muon_lite_step.argtypes = [ctypes.c_int, ctypes.c_int, _D, _D, _D, _D, _D,
                                        ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                        ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                        ctypes.c_int, _D, ctypes.c_double, ctypes.c_double,
                                        ctypes.c_int, ctypes.c_int]
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = configure(ctypes.CDLL(_build.build()))
    return _lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a):
    return a.ctypes.data_as(_D)


def _coeffs(coeffs):
    c = _f64(coeffs).reshape(-1, 3)
    return np.ascontiguousarray(c.reshape(-1)), c.shape[0]


def schedule(n_steps, coeff=QUINTIC):
    """A schedule of ``n_steps`` identical (a, b, c) triples."""
    return np.array([coeff] * n_steps, dtype=np.float64)


def num_threads():
    return lib().oracle_num_threads()


def set_num_threads(n):
    lib().oracle_set_num_threads(int(n))


def round_bf16(x):
    a = _f64(x).copy()
    lib().oracle_round_array(_p(a), a.size, ROUND_BF16)
    return a


def round_fp16(x):
    a = _f64(x).copy()
    lib().oracle_round_array(_p(a), a.size, ROUND_FP16)
    return a


def round_fp32(x):
    a = _f64(x).copy()
    lib().oracle_round_array(_p(a), a.size, ROUND_FP32)
    return a


def round_kind(x, kind):
    a = _f64(x).copy()
    lib().oracle_round_array(_p(a), a.size, int(kind))
    return a


def frobenius(x):
    a = _f64(x)
    return lib().oracle_frobenius(_p(a), a.size)


def mona(G, Gp, A, M, beta_a, alpha, mu):
    """MONA pre-pass; returns (Gp', A', M') as new arrays."""
    G = _f64(G)
    Gp, A, M = _f64(Gp).copy(), _f64(A).copy(), _f64(M).copy()
    assert G.shape == Gp.shape == A.shape == M.shape
    lib().oracle_mona(G.size, _p(G), _p(Gp), _p(A), _p(M), beta_a, alpha, mu)
    return Gp, A, M


def weight_update(W, O, eta, gamma, lam):
    W = _f64(W).copy()
    O = _f64(O)
    lib().oracle_weight_update(W.size, _p(W), _p(O), eta, gamma, lam)
    return W


def ns_poly(X, coeffs, prescale=None):
    """Quintic (or any (a,b,c)) iteration on a wide X (s <= l); no normalisation."""
    X = _f64(X).copy()
    s, l = X.shape
    assert s <= l
    c, n = _coeffs(coeffs)
    pre = None if prescale is None else _f64(prescale)
    lib().oracle_ns_poly(_p(X), s, l, n, _p(c), None if pre is None else _p(pre))
    return X


def gram_poly(X, coeffs, restarts=(), f=1.0):
    """Gram route on a wide, already normalised X; restarts at steps k > 0."""
    X = _f64(X).copy()
    s, l = X.shape
    assert s <= l
    c, n = _coeffs(coeffs)
    r = np.ascontiguousarray(np.asarray(list(restarts) or [0], dtype=np.int32))
    lib().oracle_gram_poly(_p(X), s, l, n, _p(c), r.ctypes.data_as(_I), len(restarts), f)
    return X


def polar(X):
    """Exact polar factor U V^T by one-sided Jacobi (any orientation)."""
    X = _f64(X)
    rows, cols = X.shape
    P = np.empty_like(X)
    sweeps = lib().oracle_polar(_p(X), rows, cols, _p(P))
    if sweeps < 0:
        raise RuntimeError("Jacobi did not converge")
    return P


def orthogonalise(M, coeffs, route="direct", restarts=(), f=1.0, eps=1e-7, round_to=ROUND_NONE):
    """Normalise M (and round its start to ``round_to``), then iterate."""
    M = _f64(M)
    rows, cols = M.shape
    O = np.empty_like(M)
    c, n = _coeffs(coeffs)
    r = np.ascontiguousarray(np.asarray(list(restarts) or [0], dtype=np.int32))
    lib().oracle_orthogonalise(_p(M), rows, cols, _p(O), 0 if route == "direct" else 1,
                               n, _p(c), r.ctypes.data_as(_I), len(restarts), f, eps,
                               int(round_to))
    return O


def muon_step(W, G, Gp, A, M, *, mu, eta, lam, gamma, beta_a, alpha,
              coeffs, eps=1e-7, f=1.0, round_to=ROUND_NONE):
    """One MONA/Muon step for one matrix; returns dict of new W, Gp, A, M and O."""
    W, Gp, A, M = (_f64(v).copy() for v in (W, Gp, A, M))
    G = _f64(G)
    rows, cols = W.shape
    O = np.empty_like(W)
    c, n = _coeffs(coeffs)
    lib().oracle_muon_step(rows, cols, _p(W), _p(G), _p(Gp), _p(A), _p(M), _p(O),
                           mu, eta, lam, gamma, beta_a, alpha, n, _p(c), eps, f,
                           int(round_to))
    return {"W": W, "G_prev": Gp, "A": A, "M": M, "O": O}


def mona_lite(G, B, M, beta_a, alpha, mu, round_b=True):
    """MONA-Lite elementwise pass (one buffer B instead of G_prev and A, B in
    bfloat16 when round_b); returns (B', M') as new arrays."""
    G = _f64(G)
    B, M = _f64(B).copy(), _f64(M).copy()
    assert G.shape == B.shape == M.shape
    lib().oracle_mona_lite(G.size, _p(G), _p(B), _p(M), beta_a, alpha, mu, 1 if round_b else 0)
    return B, M


def muon_lite_step(W, G, B, M, *, mu, eta, lam, gamma, beta_a, alpha,
                   coeffs, eps=1e-7, f=1.0, round_to=ROUND_NONE, round_b=True):
    """One MONA-Lite step for one matrix; returns dict of new W, B, M and O."""
    W, B, M = (_f64(v).copy() for v in (W, B, M))
    G = _f64(G)
    rows, cols = W.shape
    O = np.empty_like(W)
    c, n = _coeffs(coeffs)
    lib().oracle_muon_lite_step(rows, cols, _p(W), _p(G), _p(B), _p(M), _p(O),
                                mu, eta, lam, gamma, beta_a, alpha, n, _p(c), eps, f,
                                int(round_to), 1 if round_b else 0)
    return {"W": W, "B": B, "M": M, "O": O}


def adamw(W, G, m, v, *, lr, beta1, beta2, eps, weight_decay, step):
    """AdamW (bias-corrected, decoupled decay) on flat arrays; returns (W', m', v')."""
    W, m, v = _f64(W).copy(), _f64(m).copy(), _f64(v).copy()
    G = _f64(G)
    assert W.shape == G.shape == m.shape == v.shape
    lib().oracle_adamw(W.size, _p(W), _p(G), _p(m), _p(v), lr, beta1, beta2, eps, weight_decay, int(step))
    return W, m, v
