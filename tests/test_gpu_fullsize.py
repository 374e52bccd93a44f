"""Parity at the full workload sizes, in the launch configuration bench.py times
(one muon_step_batched call over every matrix, or one gram_polar call per batch).

The fp64 oracle computes whole-matrix results on one matrix per shape group
where it finishes in seconds, and single elements of the elementwise pass
anywhere.  For matrices too large for it, properties that hold at any size are
checked instead:
  * spectrum: the iteration is a matrix polynomial in X0 X0^T acting on X0, so
    the singular values of O are phi(sigma_i(X0)) with phi the composed scalar
    quintic (MONA page, section 2 step 4; the quintic form as configured);
  * polar-factor invariants: for a full-rank wide M, P = polar(M) has P P^T = I
    and M P^T symmetric (positive definite) -- checked on the converged Gram
    route with bounds that follow from its tolerance against P.
"""
import numpy as np
import pytest
import torch

import muon_family_optimizer_b200 as mo
import oracle
from conftest import rel_fro
from muon_family_optimizer_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

QUINTIC = (3.4445, -4.7750, 2.0315)


def f64(t):
    return t.detach().to(torch.float32).cpu().double().numpy()


def phi5(s):
    s = np.asarray(s, dtype=np.float64)
    for _ in range(5):
        a, b, c = QUINTIC
        s = a * s + b * s ** 3 + c * s ** 5
    return s


def build_state(workload, dev, o_out_for=()):
    """Full-size state; gradients share one spectrum draw per shape (random column
    signs per matrix) so that building 6.98 G elements stays quick."""
    w = syn.WORKLOADS[workload]
    params, cache = [], {}
    for j, (r, c) in enumerate(w["shapes"]):
        if (r, c) not in cache:
            cache[(r, c)] = [syn.gradient(workload, j, t, r, c, device=dev) for t in (0, 8)]
        g, gp = cache[(r, c)]
        sign = (torch.randint(0, 2, (1, c), device=dev, generator=torch.Generator(dev).manual_seed(j)) * 2 - 1)
        p = dict(W=syn.initial_weight(workload, j, r, c, device=dev).to(w["w_dtype"]),
                 G=(g * sign).to(w["w_dtype"]), G_prev=(gp * sign.flip(1)).to(w["w_dtype"]),
                 A=(gp * 1e-2).contiguous(), M=(g * 1e-1 * sign).contiguous())
        if j in o_out_for:
            p["O_out"] = torch.empty(r, c, dtype=torch.float32, device=dev)
        params.append(p)
    return w, params


def sampled_mona_check(before, after, hp, n=4096, seed=0):
    """A, M, G_prev on sampled elements against the oracle's elementwise pass."""
    g = torch.Generator().manual_seed(seed)
    numel = before["G"].numel()
    idx = torch.randint(0, numel, (n,), generator=g).to(before["G"].device)
    take = lambda t: t.reshape(-1)[idx].double().cpu().numpy()
    Gp, A, M = oracle.mona(take(before["G"]), take(before["G_prev"]), take(before["A"]), take(before["M"]),
                           hp["beta_a"], hp["alpha"], hp["mu"])
    assert rel_fro(take(after["A"]), A) <= 1e-6
    assert rel_fro(take(after["M"]), M) <= 1e-6
    assert np.array_equal(take(after["G_prev"]), Gp)


def run_step(params, w, sched=None):
    sched = sched if sched is not None else mo.quintic_schedule(5)
    arr = mo.make_params(params)
    ws = torch.empty(mo.muon_workspace_size(arr, mo._dtype_code(w["ns_dtype"]), sched), dtype=torch.uint8,
                     device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mo.muon_step_batched(arr, mo._dtype_code(w["w_dtype"]), mo._dtype_code(w["ns_dtype"]), w["hp"], sched, ws,
                         d_status=status)
    torch.cuda.synchronize()
    del ws
    return int(status.item())


def oracle_full_check(before, after, hp):
    """Whole-matrix parity of one parameter against the oracle's full step."""
    ref = oracle.muon_step(f64(before["W"]), f64(before["G"]), f64(before["G_prev"]), f64(before["A"]),
                           f64(before["M"]), mu=hp["mu"], eta=hp["eta"], lam=hp["lambda"], gamma=hp["gamma"],
                           beta_a=hp["beta_a"], alpha=hp["alpha"], coeffs=[QUINTIC] * 5,
                           round_to=oracle.ROUND_BF16)
    assert rel_fro(f64(after["A"]), ref["A"]) <= 1e-6
    assert rel_fro(f64(after["M"]), ref["M"]) <= 1e-6
    assert rel_fro(f64(after["O_out"]), ref["O"]) <= 3e-2
    assert rel_fro(f64(after["W"]), ref["W"]) <= 2.0 ** -8


def spectrum_check(after_M, O):
    """Singular values of O against phi applied to those of the bf16-rounded,
    normalised momentum (fp32 SVD on the GPU)."""
    M = after_M
    X0 = M.to(torch.bfloat16).float() / (torch.linalg.norm(M.double()).float() + 1e-7)
    s_in = torch.linalg.svdvals(X0 if X0.shape[0] <= X0.shape[1] else X0.T).double().cpu().numpy()
    s_out = torch.linalg.svdvals(O if O.shape[0] <= O.shape[1] else O.T).double().cpu().numpy()
    expect = np.sort(phi5(s_in))
    got = np.sort(s_out)
    assert np.linalg.norm(got - expect) / np.linalg.norm(expect) <= 3e-2


def weight_consistency(before, after, hp, n=4096):
    """Sampled W against the update of the stored O (one bf16 rounding)."""
    g = torch.Generator().manual_seed(1)
    idx = torch.randint(0, before["W"].numel(), (n,), generator=g).to(before["W"].device)
    W0 = before["W"].reshape(-1)[idx].double().cpu().numpy()
    O = after["O_out"].reshape(-1)[idx].double().cpu().numpy()
    W1 = after["W"].reshape(-1)[idx].double().cpu().numpy()
    Wexp = W0 - hp["eta"] * (hp["gamma"] * O + hp["lambda"] * W0)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(Wexp), 2.0 ** -126))) - 7)
    assert np.all(np.abs(W1 - Wexp) <= ulp)


def test_llama_430m_full_step():
    dev = torch.device("cuda")
    shapes = syn.WORKLOADS["llama_430m"]["shapes"]
    firsts = {}
    for j, sh in enumerate(shapes):
        firsts.setdefault(sh, j)
    w, params = build_state("llama_430m", dev, o_out_for=set(firsts.values()))
    before = [{k: v.clone() for k, v in p.items() if k != "O_out"} for p in params]
    assert run_step(params, w) == 0
    for j in firsts.values():
        oracle_full_check(before[j], params[j], w["hp"])
    for j in range(0, len(params), 7):
        sampled_mona_check(before[j], params[j], w["hp"], seed=j)
    del params, before
    torch.cuda.empty_cache()


def test_llama3_8b_full_step():
    dev = torch.device("cuda")
    torch.cuda.empty_cache()
    free, _ = torch.cuda.mem_get_info()
    if free < 150 * 2 ** 30:
        pytest.skip(f"needs ~150 GiB of free device memory, {free / 2 ** 30:.0f} GiB free")
    shapes = syn.WORKLOADS["llama3_8b"]["shapes"]
    firsts = {}
    for j, sh in enumerate(shapes):
        firsts.setdefault(sh, j)
    w, params = build_state("llama3_8b", dev, o_out_for=set(firsts.values()))
    small, square = firsts[(1024, 4096)], firsts[(4096, 4096)]
    keep = set(firsts.values()) | set(range(0, len(params), 23))
    before = {j: {k: v.clone() for k, v in params[j].items() if k != "O_out"} for j in keep}
    assert run_step(params, w) == 0
    # whole-matrix parity where the fp64 oracle takes at most a minute or two:
    # the 1024 x 4096 and one 4096 x 4096 matrix, element by element
    oracle_full_check(before[small], params[small], w["hp"])
    oracle_full_check(before[square], params[square], w["hp"])
    for sh, j in firsts.items():
        weight_consistency(before[j], params[j], w["hp"])
        if sh not in ((1024, 4096), (4096, 4096)):
            spectrum_check(params[j]["M"], params[j]["O_out"])
    for j in keep:
        sampled_mona_check(before[j], params[j], w["hp"], seed=j)
        assert torch.equal(params[j]["G_prev"], before[j]["G"])
    del params, before
    torch.cuda.empty_cache()


@pytest.mark.parametrize("workload", ["gpt2_small", "llama_430m"])
def test_full_step_gram_route(workload):
    """The whole layer set in one call with the Gram route on the elongated
    groups (768 x 3072, 1024 x 4096 and their transposes: long side >= 2 x short
    side; one restart before step 3), the square groups direct.  One matrix per
    shape against the oracle's step (in exact arithmetic both routes give the
    same O), sampled elementwise state everywhere."""
    dev = torch.device("cuda")
    shapes = syn.WORKLOADS[workload]["shapes"]
    firsts = {}
    for j, sh in enumerate(shapes):
        firsts.setdefault(sh, j)
    w, params = build_state(workload, dev, o_out_for=set(firsts.values()))
    before = [{k: v.clone() for k, v in p.items() if k != "O_out"} for p in params]
    assert run_step(params, w, mo.quintic_gram_schedule(5, gram_aspect=2.0)) == 0
    for j in firsts.values():
        oracle_full_check(before[j], params[j], w["hp"])
        weight_consistency(before[j], params[j], w["hp"])
    for j in range(0, len(params), 5):
        sampled_mona_check(before[j], params[j], w["hp"], seed=j)
    del params, before
    torch.cuda.empty_cache()


@pytest.mark.parametrize("shape,batch", [((768, 2048), 64), ((2048, 768), 64), ((16384, 2048), 1)])
def test_moe_gram_route_full_size(shape, batch):
    """Configured MoE stress sizes, fp16, condition numbers 1e1..1e3 across the
    batch, Gram route with restarts and the 1.05 divisor.

    With delta = 2e-2 the converged tolerance against the exact polar factor P
    (||O - P||_F <= delta ||P||_F, ||P||_F = sqrt(s)), E = O - P gives
      ||O O^T - I||_F <= 2 ||E||_F + ||E||_F^2  ->  / sqrt(s): 2 delta + delta^2 sqrt(s)
      ||M O^T - O M^T||_F <= 2 ||M||_2 ||E||_F  ->  / (2 ||M||_2 sqrt(s)): delta
    (wide view; P P^T = I and M P^T = U Sigma U^T symmetric)."""
    dev = torch.device("cuda")
    delta = 2e-2
    kappas = [1e1, 1e2, 1e3]
    X = torch.stack([syn.log_spectrum(*shape, kappas[i % 3], 4000 + i, device=dev) for i in range(batch)])
    X = X.to(torch.float16).contiguous()
    out = torch.empty_like(X)
    ws = torch.empty(mo.gram_polar_workspace_size(batch, *shape, mo.FP16), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    mo.gram_polar(X, out, mo.converged_schedule(), ws, d_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for i in sorted(set(list(range(min(batch, 3))) + [batch - 1])):
        O = out[i].double()
        M = X[i].double()
        On, Mn = (O, M) if O.shape[0] <= O.shape[1] else (O.T, M.T)
        s = On.shape[0]
        orth = torch.linalg.norm(On @ On.T - torch.eye(s, device=dev, dtype=torch.float64)) / s ** 0.5
        H = Mn @ On.T
        m2 = torch.linalg.matrix_norm(Mn, ord=2)
        sym = torch.linalg.norm(H - H.T) / (2 * m2 * s ** 0.5)
        assert orth <= 2 * delta + delta ** 2 * s ** 0.5, (i, float(orth))
        assert sym <= delta, (i, float(sym))
    if shape[0] * shape[1] <= 2048 * 768:
        # one sample against the oracle's exact polar factor of the same fp16 input
        i = 2   # condition number 1e3
        assert rel_fro(f64(out[i]), oracle.polar(f64(X[i]))) <= delta
