"""GPU parity of limuon_step_batched against the fp64 oracle.

Inputs: gradients with a planted spectrum (1/(1+i) for the first r singular
values, a tail below 0.01, random singular vectors), so that the rank-r factor
is well separated; a Gaussian test matrix Omega (cols x k) per parameter.
Every step both sides start from the same state (the GPU's fp32 M and W);
the oracle takes the GPU's fp32 values exactly, and the fp32 values of the
hyper-parameters the GPU computes with.  Tolerances:
  M      elementwise |gpu - ref| <= 2^-24 |ref|: one fp32 rounding of mu M + G
  O      relative Frobenius 2e-4 against the oracle's O from the GPU's own M:
         fp32 sums over up to l terms (about sqrt(l) 2^-24 = 4e-6 relative at
         l = 3072) in the three products, amplified by the conditioning of
         the rank-r factor (s_1 / s_r <= 16 here) -- a float32 emulation of the
         GPU's rounding points reaches 1e-6 to 2e-5 on these inputs
  W      bf16: relative Frobenius 2^-8 against the oracle; elementwise within
         one bf16 rounding (plus fp32 evaluation) of W - eta (gamma O + lambda W)
         evaluated in fp64 with the O the GPU stored; fp32: the update W - W0
         within O's tolerance
Plus: k = 48 (64-column kernels), r above the rank (partial isometry), a zero
momentum (O = 0), a non-finite gradient element, 130 parameters (two launches),
matrices taller than one projection segment (1024 rows; ragged segments and
column blocks), and the 72-matrix GPT-2-small set at full size, one matrix per
shape group.
"""
import numpy as np
import pytest
import torch

import muon_family_optimizer_b200 as mo
from conftest import rel_fro
from muon_family_optimizer_b200 import synthetic as syn
from oracle import limuon as lim

pytestmark = pytest.mark.gpu

SHAPES = [(256, 256), (192, 520), (520, 192), (100, 36), (1, 48), (130, 2), (768, 3072), (300, 7)]
TOL_O = 2e-4


def f64(t):
    return t.detach().to(torch.float32).cpu().double().numpy()


def _planted(rows, cols, r, seed):
    g = torch.Generator().manual_seed(seed)
    n = min(rows, cols)
    U = torch.linalg.qr(torch.randn(rows, n, generator=g, dtype=torch.float64))[0]
    V = torch.linalg.qr(torch.randn(cols, n, generator=g, dtype=torch.float64))[0]
    s = torch.cat([1.0 / (1 + torch.arange(min(r, n), dtype=torch.float64)),
                   0.01 * torch.rand(max(0, n - r), generator=g, dtype=torch.float64)])
    return (U * s) @ V.T


def _omega(cols, k, seed):
    return torch.randn(cols, k, generator=torch.Generator().manual_seed(seed)).cuda()


def _params(shapes, w_dtype, k, r, seed=0, o_out=True):
    out = []
    for j, (rows, cols) in enumerate(shapes):
        W = (torch.randn(rows, cols, generator=torch.Generator().manual_seed(seed + 31 * j)) * 0.02).to(w_dtype)
        out.append(dict(W=W.cuda(), M=torch.zeros(rows, cols, device="cuda"), Omega=_omega(cols, k, seed + 7 * j),
                        O_out=torch.empty(rows, cols, device="cuda") if o_out else None,
                        seed=seed + 101 * j, r=r))
    return out


def _run(params, w_dtype, hp):
    ws = torch.empty(mo.limuon_workspace_size(params, hp), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mo.limuon_step_batched(params, mo._dtype_code(w_dtype), hp, ws, d_status=status)
    torch.cuda.synchronize()
    return int(status.item())


def _hp(r, p, lam=0.1):
    return dict(mu=0.95, eta=0.02, gamma=1.0, rank=r, oversample=p, **{"lambda": lam})


def _ulp(x, dt):
    if dt == torch.float32:
        return np.zeros_like(x)
    mant = 7 if dt == torch.bfloat16 else 10
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126 if dt == torch.bfloat16 else 2.0 ** -14)))
    return 2.0 ** (e - mant)


def _check_step(params, w_dtype, hp, t):
    # the oracle receives the fp32 values of the hyper-parameters the GPU uses
    h32 = {k: (float(np.float32(v)) if isinstance(v, float) else v) for k, v in hp.items()}
    for j, p in enumerate(params):
        rows, cols = p["W"].shape
        p["G"] = _planted(rows, cols, hp["rank"], p["seed"] + t).to(w_dtype).cuda()
    M0 = [f64(p["M"]) for p in params]
    W0 = [f64(p["W"]) for p in params]
    assert _run(params, w_dtype, hp) == 0
    for j, p in enumerate(params):
        G = f64(p["G"])
        Mg = f64(p["M"])
        Mref = lim.momentum(M0[j], G, h32["mu"])
        assert np.all(np.abs(Mg - Mref) <= 2.0 ** -24 * np.abs(Mref)), (t, j)
        Og = f64(p["O_out"])
        Oref = lim.rsvd_orthogonal(Mg, f64(p["Omega"]), hp["rank"])
        assert rel_fro(Og, Oref) <= TOL_O, (t, j, rel_fro(Og, Oref))
        Wg = f64(p["W"])
        Wref = lim.weight_update(W0[j], Oref, h32["eta"], h32["gamma"], h32["lambda"])
        if w_dtype == torch.float32:
            assert rel_fro(Wg - W0[j], Wref - W0[j]) <= TOL_O, (t, j)
        else:
            assert rel_fro(Wg, Wref) <= 2.0 ** -8, (t, j)
            own = lim.weight_update(W0[j], Og, h32["eta"], h32["gamma"], h32["lambda"])
            bnd = 0.5 * _ulp(own, w_dtype) * 1.001 + 2.0 ** -22 * (np.abs(W0[j]) + hp["eta"] * np.abs(Og))
            assert np.all(np.abs(Wg - own) <= bnd), (t, j, float(np.max(np.abs(Wg - own) - bnd)))


@pytest.mark.parametrize("w_dtype", [torch.bfloat16, torch.float32, torch.float16])
def test_limuon_two_steps_vs_oracle(w_dtype):
    hp = _hp(16, 16)
    params = _params(SHAPES, w_dtype, 32, 16)
    for t in range(2):
        _check_step(params, w_dtype, hp, t)


TALL = [(2100, 136), (1500, 36), (1025, 64)]


@pytest.mark.parametrize("w_dtype", [torch.bfloat16, torch.float32])
def test_limuon_tall_matrices_segmented_projection(w_dtype):
    # more than 1024 rows: the projection runs each 128-column block as row
    # segments whose partial B^T are added by the segment that finishes last
    hp = _hp(16, 16)
    params = _params(TALL, w_dtype, 32, 16, seed=11)
    for t in range(2):
        _check_step(params, w_dtype, hp, t)


def test_limuon_wide_sketch_64_columns():
    hp = _hp(40, 8)
    params = _params(SHAPES, torch.bfloat16, 48, 40, seed=5)
    _check_step(params, torch.bfloat16, hp, 0)


def test_limuon_rank_above_matrix_rank_is_polar():
    # r = 16 on matrices of rank 1 and 2: O is the (partial-isometry) polar factor
    hp = _hp(16, 4, lam=0.0)
    params = _params([(1, 48), (130, 2), (9, 5)], torch.float32, 20, 16, seed=9)
    _check_step(params, torch.float32, hp, 0)
    for p in params:
        O = f64(p["O_out"])
        n = min(O.shape)
        assert np.allclose(np.linalg.svd(O, compute_uv=False)[:n], 1.0, atol=1e-5)


def test_limuon_zero_momentum_gives_zero_update():
    hp = _hp(8, 8)
    params = _params([(64, 96), (33, 17)], torch.float32, 16, 8)
    for p in params:
        p["G"] = torch.zeros_like(p["W"])
    W0 = [p["W"].clone() for p in params]
    assert _run(params, torch.float32, hp) == 0
    for p, w0 in zip(params, W0):
        assert torch.count_nonzero(p["O_out"]) == 0
        expect = w0 - hp["eta"] * (hp["lambda"] * w0)
        assert torch.allclose(p["W"], expect, rtol=2 ** -22, atol=0)


def test_limuon_nonfinite_keeps_weights():
    hp = _hp(8, 8)
    params = _params([(64, 96), (40, 40)], torch.bfloat16, 16, 8)
    for p in params:
        rows, cols = p["W"].shape
        p["G"] = _planted(rows, cols, 8, p["seed"]).to(torch.bfloat16).cuda()
    params[1]["G"][3, 5] = float("inf")
    W0, W1 = params[0]["W"].clone(), params[1]["W"].clone()
    st = _run(params, torch.bfloat16, hp)
    assert st & mo.FLAG_NONFINITE
    assert torch.equal(params[1]["W"], W1)
    assert not torch.equal(params[0]["W"], W0)


def test_limuon_overflow_in_the_sketch_keeps_weights():
    # a finite momentum whose sketch Y = M Omega overflows fp32 (entries of
    # 2.85e38 times Gaussian weights, summed over 200 columns): the k x k Gram
    # of Y is not finite, the matrix is marked, its W kept and the flag raised;
    # the other matrix steps
    hp = _hp(8, 8)
    params = _params([(64, 96), (48, 200)], torch.float32, 16, 8)
    for p in params:
        rows, cols = p["W"].shape
        p["G"] = _planted(rows, cols, 8, p["seed"]).to(torch.float32).cuda()
    params[1]["G"].zero_()
    params[1]["M"].fill_(3e38)          # mu M + 0 stays finite; the sums over 200 columns do not
    W0, W1 = params[0]["W"].clone(), params[1]["W"].clone()
    st = _run(params, torch.float32, hp)
    assert st & mo.FLAG_NONFINITE
    assert torch.isfinite(params[1]["M"]).all()
    assert torch.equal(params[1]["W"], W1)
    assert not torch.equal(params[0]["W"], W0)


def test_limuon_many_parameters_two_launches():
    shapes = [(24 + (i % 5) * 8, 40 + (i % 7) * 4) for i in range(130)]
    hp = _hp(4, 4)
    params = _params(shapes, torch.bfloat16, 8, 4, seed=3)
    _check_step(params, torch.bfloat16, hp, 0)


def test_limuon_gpt2_small_full_size():
    """All 72 matrices in one call (the benchmark's configuration: r = 16, p = 16,
    bf16 W and G); one matrix per shape group checked against the oracle."""
    wl = syn.WORKLOADS["gpt2_small"]
    hp = dict(mu=0.95, eta=0.02, gamma=1.0, rank=16, oversample=16, **{"lambda": 0.0})
    params, omegas = [], {}
    for j, (rows, cols) in enumerate(wl["shapes"]):
        if cols not in omegas:
            omegas[cols] = _omega(cols, 32, cols)
        G = syn.gradient("gpt2_small", j, 0, rows, cols, device="cuda").to(torch.bfloat16)
        params.append(dict(W=syn.initial_weight("gpt2_small", j, rows, cols).to(torch.bfloat16).cuda(), G=G,
                           M=torch.zeros(rows, cols, device="cuda"), Omega=omegas[cols],
                           O_out=torch.empty(rows, cols, device="cuda")))
    W0 = [p["W"].clone() for p in params]
    assert _run(params, torch.bfloat16, hp) == 0
    seen = set()
    for j, p in enumerate(params):
        if p["W"].shape in seen:
            continue
        seen.add(p["W"].shape)
        Mg = f64(p["M"])
        assert np.array_equal(Mg, f64(p["G"]))           # first step from zero: M = G exactly
        Oref = lim.rsvd_orthogonal(Mg, f64(p["Omega"]), 16)
        assert rel_fro(f64(p["O_out"]), Oref) <= TOL_O, (j, rel_fro(f64(p["O_out"]), Oref))
        Wref = lim.weight_update(f64(W0[j]), Oref, hp["eta"], hp["gamma"], hp["lambda"])
        assert rel_fro(f64(p["W"]), Wref) <= 2.0 ** -8, j
    assert len(seen) == len(set(wl["shapes"]))      # 768 x 768, 768 x 3072, 3072 x 768
