"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle.

Tolerances (relative Frobenius error unless stated):
  16-bit Newton-Schulz vs the oracle run from the same 16-bit input   3e-2
  fp32 Newton-Schulz vs the oracle                                     1e-4
  fp32 elementwise state (A, M; fp32 W)                                 1e-6
  G_prev                                                               bit-exact copy of G
  bf16 W                                                               1 bf16 ulp per element
  converged schedule and Gram route vs the exact polar factor          2e-2 (condition number <= 1e3)
"""
import math

import numpy as np
import pytest
import torch

import muon_family_optimizer_b200 as mo
import oracle
from conftest import rel_fro
from muon_family_optimizer_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

QUINTIC = (3.4445, -4.7750, 2.0315)
CUBIC = (1.5, -0.5, 0.0)
CONVERGED = [QUINTIC] * 8 + [CUBIC] * 6
RESTARTS = (3, 5, 7)     # restarts of the converged schedule (see mo.converged_schedule)
DT = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}
ROUND = {"bf16": oracle.ROUND_BF16, "fp16": oracle.ROUND_FP16, "fp32": oracle.ROUND_NONE}


def f64(t):
    return t.detach().to(torch.float32).cpu().double().numpy()


def run_polar(route, X, coeffs, restarts=(), f=1.0, eps=1e-7):
    sched = mo.make_schedule(coeffs, eps=eps, restarts=restarts, scale_f=f)
    b, r, c = (1, *X.shape) if X.dim() == 2 else X.shape
    size = (mo.ns_polar_workspace_size if route == "direct" else mo.gram_polar_workspace_size)(
        b, r, c, mo._dtype_code(X.dtype))
    ws = torch.empty(size, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(X)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    (mo.ns_polar if route == "direct" else mo.gram_polar)(X, out, sched, ws, d_status=status)
    torch.cuda.synchronize()
    return out, int(status.item())


# ----------------------------------------------------------------- ns_polar

def test_ns_polar_fp32_tiny():
    X = syn.tiny_sequence()[1].cuda()
    out, st = run_polar("direct", X, [QUINTIC] * 5)
    assert st == 0
    ref = oracle.orthogonalise(f64(X), [QUINTIC] * 5)
    assert rel_fro(f64(out), ref) <= 1e-4


@pytest.mark.parametrize("dt", ["bf16", "fp16"])
@pytest.mark.parametrize("shape", [(128, 256), (200, 328), (328, 200), (256, 256), (37, 1000),
                                   (1, 64), (64, 1), (3, 5), (130, 130), (1100, 1300), (1300, 1100)])
def test_ns_polar_16bit_vs_oracle(dt, shape):
    X = syn.gaussian(shape, 11 + shape[0], "cpu").to(DT[dt]).cuda()
    out, st = run_polar("direct", X, [QUINTIC] * 5)
    assert st == 0
    ref = oracle.orthogonalise(f64(X), [QUINTIC] * 5)
    assert rel_fro(f64(out), ref) <= 3e-2


@pytest.mark.parametrize("shape", [(200, 456), (1100, 1300), (1300, 1100)])
@pytest.mark.parametrize("coeff", [(1.0, 0.0, 0.0), (0.0, 1.0, 0.0), (0.0, 0.0, 1e4), (0.5, -0.25, 1250.0)])
def test_single_step_products(coeff, shape):
    # isolates the three products of one step: (1,0,0) the copy and scaling,
    # (0,1,0) X X^T X, (0,0,c) (X X^T)^2 X; s >= 1024 takes the 256 x 512
    # tiles for the symmetric products too, with ragged edges.  A bfloat16
    # input is iterated in fp16: with c = 1 the entries of B' = (X X^T)^2 of a
    # normalised 1100 x 1300 matrix are below 2e-6, in fp16's subnormal range,
    # where the fp16-rounded computation itself is 12% off; c = 1e4 keeps B' in
    # the normal range (fp16-rounded computation: 5e-4 off).
    X = syn.gaussian(shape, 5, "cpu").to(torch.bfloat16).cuda()
    out, st = run_polar("direct", X, [coeff])
    assert st == 0
    ref = oracle.orthogonalise(f64(X), [coeff])
    assert rel_fro(f64(out), ref) <= 1e-2


def test_ns_polar_batched_and_in_place():
    X = torch.stack([syn.gaussian((96, 320), 40 + i) for i in range(5)]).to(torch.bfloat16).cuda()
    X0 = X.clone()
    sched = mo.quintic_schedule(5)
    ws = torch.empty(mo.ns_polar_workspace_size(5, 96, 320, mo.BF16), dtype=torch.uint8, device="cuda")
    mo.ns_polar(X, X, sched, ws)   # in place
    torch.cuda.synchronize()
    for i in range(5):
        ref = oracle.orthogonalise(f64(X0[i]), [QUINTIC] * 5)
        assert rel_fro(f64(X[i]), ref) <= 3e-2


def test_ns_polar_zero_matrix_is_zero():
    X = torch.zeros(64, 96, dtype=torch.bfloat16, device="cuda")
    out, st = run_polar("direct", X, [QUINTIC] * 5)
    assert st == 0
    assert torch.count_nonzero(out).item() == 0


def test_ns_polar_nonfinite_flag():
    X = syn.gaussian((64, 96), 3).to(torch.bfloat16).cuda()
    X[3, 7] = float("nan")
    out, st = run_polar("direct", X, [QUINTIC] * 5)
    assert st & mo.FLAG_NONFINITE


# ----------------------------------------------------------------- converged / Gram route

@pytest.mark.parametrize("route", ["direct", "gram"])
@pytest.mark.parametrize("dt,kappa", [("fp16", 1e1), ("fp16", 1e2), ("fp16", 1e3), ("bf16", 1e1), ("bf16", 1e2),
                                      ("bf16", 1e3)])
@pytest.mark.parametrize("shape", [(256, 640), (640, 256), (384, 384)])
def test_converged_vs_exact_polar(route, dt, kappa, shape):
    # a bfloat16 input is iterated in fp16 after normalisation (include/muon.h)
    M = syn.log_spectrum(*shape, kappa, 77).to(DT[dt])
    out, st = run_polar(route, M.cuda(), CONVERGED, restarts=RESTARTS, f=1.05)
    assert st == 0
    P = oracle.polar(f64(M))     # exact polar factor of the same 16-bit input
    assert rel_fro(f64(out), P) <= 2e-2


@pytest.mark.parametrize("dt", ["fp16", "bf16"])
def test_gram_route_matches_oracle_gram_route(dt):
    M = syn.log_spectrum(192, 448, 1e2, 78).to(DT[dt])
    sched = [QUINTIC] * 6
    out, st = run_polar("gram", M.cuda(), sched, restarts=(0, 3), f=1.05)
    assert st == 0
    ref = oracle.orthogonalise(f64(M), sched, route="gram", restarts=(0, 3), f=1.05)
    assert rel_fro(f64(out), ref) <= 3e-2


def test_gram_route_fp32_and_tall():
    M = syn.log_spectrum(300, 120, 1e2, 79)   # tall
    out, st = run_polar("gram", M.cuda(), CONVERGED, restarts=RESTARTS, f=1.05)
    assert st == 0
    ref = oracle.orthogonalise(f64(M), CONVERGED, route="gram", restarts=RESTARTS, f=1.05)
    assert rel_fro(f64(out), ref) <= 1e-4


# ----------------------------------------------------------------- full optimizer step

def _state(shapes, w_dtype, workload, t=0, device="cuda"):
    params = []
    for j, (r, c) in enumerate(shapes):
        W = syn.initial_weight(workload, j, r, c).to(w_dtype)
        G = syn.gradient(workload, j, t, r, c).to(w_dtype)
        Gp = syn.gradient(workload, j, t + 8, r, c).to(w_dtype)
        A = syn.gaussian((r, c), 500 + j, std=1e-3)
        M = syn.gaussian((r, c), 600 + j, std=1e-3)
        params.append({k: v.to(device).contiguous() for k, v in
                       dict(W=W, G=G, G_prev=Gp, A=A, M=M).items()})
    return params


def _step(params, w_dtype, ns_dtype, hp, coeffs, with_O=True, sched=None):
    for p in params:
        if with_O:
            p["O_out"] = torch.empty(p["W"].shape, dtype=torch.float32, device="cuda")
    sched = sched if sched is not None else mo.make_schedule(coeffs)
    ws = torch.empty(mo.muon_workspace_size(params, mo._dtype_code(ns_dtype), sched), dtype=torch.uint8,
                     device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mo.muon_step_batched(params, mo._dtype_code(w_dtype), mo._dtype_code(ns_dtype), hp, sched, ws,
                         d_status=status)
    torch.cuda.synchronize()
    return int(status.item())


def _ulp_bf16(x):
    x = np.abs(x)
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def _check_step(before, after, hp, ns_dt, w_dt):
    for b, a in zip(before, after):
        # a short side below 16 is iterated in fp32 whatever the iteration type
        narrow = min(b["W"].shape) < 16
        it_dt = "fp32" if narrow else ns_dt
        ref = oracle.muon_step(f64(b["W"]), f64(b["G"]), f64(b["G_prev"]), f64(b["A"]), f64(b["M"]),
                               mu=hp["mu"], eta=hp["eta"], lam=hp["lambda"], gamma=hp["gamma"],
                               beta_a=hp["beta_a"], alpha=hp["alpha"], coeffs=[QUINTIC] * 5,
                               round_to=ROUND[it_dt])
        assert rel_fro(f64(a["A"]), ref["A"]) <= 1e-6
        assert rel_fro(f64(a["M"]), ref["M"]) <= 1e-6
        assert torch.equal(a["G_prev"].cpu(), b["G"].cpu())
        tol = 1e-4 if it_dt == "fp32" else 3e-2
        assert rel_fro(f64(a["O_out"]), ref["O"]) <= tol
        if w_dt == "fp32":
            assert rel_fro(f64(a["W"]), ref["W"]) <= 1e-6
        else:
            # against the oracle: one bf16 rounding (2^-9 relative) plus the update's error
            assert rel_fro(f64(a["W"]), ref["W"]) <= 2.0 ** -8
            # consistency of the fused epilogue: the stored W is the rounded update
            # W - eta (gamma O + lambda W) of the O it stored (one rounding, <= 1 ulp)
            W0, O = f64(b["W"]), f64(a["O_out"])
            Wexp = W0 - hp["eta"] * (hp["gamma"] * O + hp["lambda"] * W0)
            assert np.all(np.abs(f64(a["W"]) - Wexp) <= _ulp_bf16(Wexp) + 1e-30)


def test_muon_step_tiny_three_steps_fp32():
    w = syn.WORKLOADS["tiny"]
    hp = w["hp"]
    W0, G0, G1, G2 = syn.tiny_sequence()
    p = dict(W=W0.clone(), G=G0.clone(), G_prev=torch.zeros_like(W0), A=torch.zeros_like(W0),
             M=torch.zeros_like(W0))
    ref = {k: f64(v) for k, v in p.items()}
    gpu = [{k: v.cuda() for k, v in p.items()}]
    for t, G in enumerate([G0, G1, G2]):
        gpu[0]["G"] = G.cuda().contiguous()
        ref["G"] = f64(G)
        assert _step(gpu, torch.float32, torch.float32, hp, [QUINTIC] * 5) == 0
        out = oracle.muon_step(ref["W"], ref["G"], ref["G_prev"], ref["A"], ref["M"], mu=hp["mu"],
                               eta=hp["eta"], lam=hp["lambda"], gamma=hp["gamma"], beta_a=hp["beta_a"],
                               alpha=hp["alpha"], coeffs=[QUINTIC] * 5)
        ref.update(W=out["W"], G_prev=out["G_prev"], A=out["A"], M=out["M"])
        assert rel_fro(f64(gpu[0]["O_out"]), out["O"]) <= 1e-4, t
        for k in ("W", "M", "A"):
            assert rel_fro(f64(gpu[0][k]), ref[k]) <= 1e-6, (t, k)


@pytest.mark.parametrize("ns_dt", ["bf16", "fp16", "fp32"])
def test_muon_step_mixed_shapes(ns_dt):
    shapes = [(256, 256), (192, 520), (520, 192), (100, 36), (1, 48), (130, 2)]
    hp = dict(mu=0.95, eta=0.02, gamma=1.0, beta_a=0.9, alpha=0.5, **{"lambda": 0.1})
    before = _state(shapes, torch.bfloat16, "gpt2_small")
    after = [{k: v.clone() for k, v in p.items()} for p in before]
    assert _step(after, torch.bfloat16, DT[ns_dt], hp, [QUINTIC] * 5) == 0
    _check_step(before, after, hp, ns_dt, "bf16")


@pytest.mark.parametrize("ns_dt", ["bf16", "fp16"])
def test_muon_step_gram_route_on_elongated_groups(ns_dt):
    # the Gram route inside the step ([POLAR]: iterate on the small Gram matrix),
    # one restart before step 3, on groups whose long side is >= 2x the short
    # side; in exact arithmetic it is the direct iteration, so the oracle's
    # direct step is the reference.  (200, 200) and (300, 520) stay direct.
    shapes = [(192, 520), (520, 192), (128, 1024), (200, 200), (300, 520), (64, 2048), (130, 2)]
    hp = dict(mu=0.95, eta=0.02, gamma=1.0, beta_a=0.9, alpha=0.5, **{"lambda": 0.1})
    sched = mo.quintic_gram_schedule(5, gram_aspect=2.0)
    for workload in ("gpt2_small", "llama_430m"):   # rank-16 plus noise; power-law spectra
        before = _state(shapes, torch.bfloat16, workload)
        after = [{k: v.clone() for k, v in p.items()} for p in before]
        assert _step(after, torch.bfloat16, DT[ns_dt], hp, None, sched=sched) == 0
        _check_step(before, after, hp, ns_dt, "bf16")


def test_muon_step_gram_route_matches_oracle_gram_route():
    # against the oracle's own Gram route with the same restart: the two
    # evaluation orders agree in fp64, so this isolates the GPU's products
    shapes = [(160, 640), (640, 160)]
    hp = dict(mu=0.9, eta=0.02, gamma=1.0, beta_a=0.9, alpha=0.5, **{"lambda": 0.0})
    before = _state(shapes, torch.bfloat16, "gpt2_small")
    after = [{k: v.clone() for k, v in p.items()} for p in before]
    sched = mo.quintic_gram_schedule(5, gram_aspect=3.0)
    assert _step(after, torch.bfloat16, torch.bfloat16, hp, None, sched=sched) == 0
    for b, a in zip(before, after):
        ref = oracle.muon_step(f64(b["W"]), f64(b["G"]), f64(b["G_prev"]), f64(b["A"]), f64(b["M"]),
                               mu=hp["mu"], eta=hp["eta"], lam=hp["lambda"], gamma=hp["gamma"],
                               beta_a=hp["beta_a"], alpha=hp["alpha"], coeffs=[QUINTIC] * 5,
                               round_to=oracle.ROUND_BF16)
        O_gram = oracle.orthogonalise(ref["M"], [QUINTIC] * 5, route="gram", restarts=mo.GRAM_STEP_RESTARTS,
                                      f=1.0, round_to=oracle.ROUND_BF16)
        assert rel_fro(O_gram, ref["O"]) <= 1e-9            # the two routes, in fp64
        assert rel_fro(f64(a["O_out"]), O_gram) <= 3e-2


def test_muon_step_fp32_weights_bf16_iteration():
    shapes = [(64, 128), (300, 90)]
    hp = dict(mu=0.9, eta=0.05, gamma=0.7, beta_a=0.8, alpha=1.0, **{"lambda": 0.01})
    before = _state(shapes, torch.float32, "gpt2_small")
    after = [{k: v.clone() for k, v in p.items()} for p in before]
    assert _step(after, torch.float32, torch.bfloat16, hp, [QUINTIC] * 5) == 0
    for b, a in zip(before, after):
        ref = oracle.muon_step(f64(b["W"]), f64(b["G"]), f64(b["G_prev"]), f64(b["A"]), f64(b["M"]),
                               mu=hp["mu"], eta=hp["eta"], lam=hp["lambda"], gamma=hp["gamma"],
                               beta_a=hp["beta_a"], alpha=hp["alpha"], coeffs=[QUINTIC] * 5,
                               round_to=oracle.ROUND_BF16)
        assert rel_fro(f64(a["O_out"]), ref["O"]) <= 3e-2
        # W - W0 is eta*(gamma O + lambda W): compare the update itself
        dW = f64(a["W"]) - f64(b["W"])
        assert rel_fro(dW, ref["W"] - f64(b["W"])) <= 3e-2


def test_muon_step_nonfinite_keeps_weights():
    shapes = [(64, 96), (64, 96)]
    hp = dict(mu=0.95, eta=0.02, gamma=1.0, beta_a=0.9, alpha=0.5, **{"lambda": 0.1})
    params = _state(shapes, torch.bfloat16, "gpt2_small")
    params[1]["G"][5, 5] = float("inf")
    W1 = params[1]["W"].clone()
    W0 = params[0]["W"].clone()
    st = _step(params, torch.bfloat16, torch.bfloat16, hp, [QUINTIC] * 5)
    assert st & mo.FLAG_NONFINITE
    assert torch.equal(params[1]["W"], W1)
    assert not torch.equal(params[0]["W"], W0)


def test_gpt2_small_full_step_sampled():
    # The full GPT-2-small layer set in one call; every matrix's cheap state is
    # checked, the orthogonalised update on one matrix of each shape.
    w = syn.WORKLOADS["gpt2_small"]
    before = _state(w["shapes"], torch.bfloat16, "gpt2_small")
    after = [{k: v.clone() for k, v in p.items()} for p in before]
    assert _step(after, torch.bfloat16, torch.bfloat16, w["hp"], [QUINTIC] * 5) == 0
    sample = {0, 4, 5}     # 768x768, 768x3072, 3072x768
    _check_step([before[i] for i in sorted(sample)], [after[i] for i in sorted(sample)], w["hp"], "bf16", "bf16")
    for b, a in zip(before, after):
        assert torch.equal(a["G_prev"], b["G"])
