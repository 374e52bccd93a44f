"""GPU parity of adamw_step_batched against the fp64 oracle.

Three steps; each starts both sides from the oracle's state rounded to the
storage types (W in its dtype, m and v in fp32), with the hyper-parameters the
GPU receives (fp32 values, given to the oracle exactly).  Per element:
  m      |gpu - ref| <= 2^-22 (b1 |m_prev| + (1 - b1) |g|): three fp32 roundings of
         the terms (the sum may cancel far below them)
  v      |gpu - ref| <= 2^-21 (b2 v_prev + (1 - b2) g^2): four
  W      |gpu - ref| <= 2^-20 (|W_prev| + |W_ref| + lr (|u| + wd |W_prev|))
                          + lr (dm / (1 - b1^t) / (sqrt(v_hat) + eps) + |u| dv / (2 v))
                          + (16-bit W: one rounding, ulp(W_ref)),
         u the normalised update: the fp32 evaluation of m_hat / (sqrt(v_hat) +
         eps) and of the final subtraction (whose operands W_prev and lr (u + wd
         W_prev) may cancel far below them), plus the m and v bounds dm, dv
         above carried through u to first order (m itself may cancel)
Plus: 130 parameters (two launches), unaligned views (element-wise path), and
a non-finite gradient element that keeps its state and raises the flag.
"""
import numpy as np
import pytest
import torch

import muon_family_optimizer_b200 as mo
import oracle

pytestmark = pytest.mark.gpu

HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.1)
HP32 = {k: float(np.float32(v)) for k, v in HP.items()}
SIZES = [1, 7, 768, 2304, 3072, 65541, 1024 * 768, (3, 5)]


def _ulp(x, dt):
    if dt == torch.float32:
        return np.zeros_like(x)
    mant = 7 if dt == torch.bfloat16 else 10
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126 if dt == torch.bfloat16 else 2.0 ** -14)))
    return 2.0 ** (e - mant)


def _round(x, dt):
    return torch.from_numpy(x).to(dt).double().numpy()


def _state(dt, sizes, seed=0, unaligned=False):
    g = torch.Generator().manual_seed(seed)
    out = []
    for sz in sizes:
        shape = sz if isinstance(sz, tuple) else (sz,)
        n = int(np.prod(shape))
        W = torch.randn(n + unaligned, generator=g)[unaligned:].reshape(shape) * 0.02
        out.append(dict(W=W.to(dt).double().numpy(), m=np.zeros(shape), v=np.zeros(shape)))
    return out


def _grad(shape, t, j, dt):
    g = torch.Generator().manual_seed(1000 + 16 * j + t)
    return (torch.randn(shape, generator=g) * 10.0 ** (-(j % 4))).to(dt)


def _to_gpu(a, dt, unaligned):
    if not unaligned:
        return torch.from_numpy(a).to(dt).cuda().contiguous()
    flat = torch.zeros(a.size + 1, dtype=dt, device="cuda")
    view = flat[1:].view(a.shape)
    view.copy_(torch.from_numpy(a).to(dt))
    return view


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32, torch.float16])
@pytest.mark.parametrize("unaligned", [False, True])
def test_adamw_three_steps_vs_oracle(dt, unaligned):
    state = _state(dt, SIZES, unaligned=unaligned)
    for t in range(1, 4):
        params, grads = [], []
        for j, S in enumerate(state):
            G = _grad(S["W"].shape, t, j, dt)
            grads.append(G.double().numpy())
            params.append(dict(W=_to_gpu(S["W"], dt, unaligned), G=_to_gpu(grads[-1], dt, unaligned),
                               m=_to_gpu(S["m"], torch.float32, unaligned), v=_to_gpu(S["v"], torch.float32, unaligned)))
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        mo.adamw_step_batched(params, mo._dtype_code(dt), HP32, t, d_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for j, (S, p) in enumerate(zip(state, params)):
            W, m, v = oracle.adamw(S["W"], grads[j], S["m"], S["v"], step=t, **HP32)
            mg, vg, Wg = (p[k].double().cpu().numpy() for k in ("m", "v", "W"))
            g = grads[j]
            b1, b2 = HP32["beta1"], HP32["beta2"]
            assert np.all(np.abs(mg - m) <= 2.0 ** -22 * (b1 * np.abs(S["m"]) + (1 - b1) * np.abs(g))), (t, j)
            assert np.all(np.abs(vg - v) <= 2.0 ** -21 * (b2 * S["v"] + (1 - b2) * g * g)), (t, j)
            c1 = 1 - HP32["beta1"] ** t
            c2 = 1 - HP32["beta2"] ** t
            u = (m / c1) / (np.sqrt(v / c2) + HP32["eps"])
            Wp = np.abs(S["W"])
            dm = 2.0 ** -22 * (b1 * np.abs(S["m"]) + (1 - b1) * np.abs(g))
            dv = 2.0 ** -21 * (b2 * S["v"] + (1 - b2) * g * g)
            du = dm / c1 / (np.sqrt(v / c2) + HP32["eps"]) + np.abs(u) * np.where(v > 0, dv / (2 * np.where(v > 0, v, 1)), 0)
            bnd = (2.0 ** -20 * (Wp + np.abs(W) + HP32["lr"] * (np.abs(u) + HP32["weight_decay"] * Wp))
                   + HP32["lr"] * du + _ulp(W, dt))
            assert np.all(np.abs(Wg - W) <= bnd), (t, j, float(np.max(np.abs(Wg - W) - bnd)))
            state[j] = dict(W=_round(W, dt), m=_round(m, torch.float32), v=_round(v, torch.float32))


def test_adamw_many_parameters_two_launches():
    dt = torch.bfloat16
    sizes = [17 + 3 * i for i in range(130)]
    state = _state(dt, sizes, seed=3)
    params, grads = [], []
    for j, S in enumerate(state):
        grads.append(_grad(S["W"].shape, 1, j, dt).double().numpy())
        params.append(dict(W=_to_gpu(S["W"], dt, False), G=_to_gpu(grads[-1], dt, False),
                           m=torch.zeros(S["W"].shape, device="cuda"), v=torch.zeros(S["W"].shape, device="cuda")))
    mo.adamw_step_batched(params, mo._dtype_code(dt), HP32, 1)
    torch.cuda.synchronize()
    for j, (S, p) in enumerate(zip(state, params)):
        W, m, v = oracle.adamw(S["W"], grads[j], S["m"], S["v"], step=1, **HP32)
        assert np.all(np.abs(p["m"].double().cpu().numpy() - m) <= 2.0 ** -22 * (1 - HP32["beta1"]) * np.abs(grads[j])), j
        Wg = p["W"].double().cpu().numpy()
        assert np.all(np.abs(Wg - W) <= _ulp(W, dt) + 2.0 ** -20 * (np.abs(S["W"]) + np.abs(W) + HP32["lr"] * 2)), j


def test_adamw_nonfinite_gradient_element_keeps_state():
    dt = torch.bfloat16
    W0 = (torch.randn(1000, generator=torch.Generator().manual_seed(9)) * 0.02).to(dt).cuda()
    G = torch.randn(1000, generator=torch.Generator().manual_seed(10)).to(dt).cuda()
    G[17] = float("inf")
    G[500] = float("nan")
    p = dict(W=W0.clone(), G=G, m=torch.full((1000,), 0.5, device="cuda"), v=torch.full((1000,), 0.25, device="cuda"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mo.adamw_step_batched([p], mo._dtype_code(dt), HP32, 2, d_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & mo.FLAG_NONFINITE
    for i in (17, 500):
        assert p["W"][i].item() == W0[i].item() and p["m"][i].item() == 0.5 and p["v"][i].item() == 0.25
    changed = (p["W"] != W0).sum().item()
    assert changed > 900


def test_model_step_fuses_adamw_into_the_step_launch():
    # muon_model_step: the matrices exactly as muon_step_batched and the vectors
    # exactly as adamw_step_batched (the same per-element arithmetic, as items of
    # the step's pre-pass launch): both compared bit for bit with the separate
    # calls, and the vectors against the oracle within this file's bounds
    from muon_family_optimizer_b200 import synthetic as syn
    hp = dict(mu=0.95, eta=0.02, gamma=1.0, beta_a=0.9, alpha=0.5, **{"lambda": 0.1})
    shapes = [(256, 384), (384, 256), (64, 96)]

    def mats():
        out = []
        for j, (r, c) in enumerate(shapes):
            out.append(dict(W=syn.initial_weight("gpt2_small", j, r, c).to(torch.bfloat16).cuda(),
                            G=syn.gradient("gpt2_small", j, 0, r, c).to(torch.bfloat16).cuda(),
                            G_prev=syn.gradient("gpt2_small", j, 8, r, c).to(torch.bfloat16).cuda(),
                            A=torch.zeros(r, c, device="cuda"), M=torch.zeros(r, c, device="cuda")))
        return out

    def vecs(state, t):
        out = []
        for j, st in enumerate(state):
            shape = st["W"].shape
            out.append(dict(W=torch.from_numpy(st["W"]).to(torch.bfloat16).cuda(),
                            G=_grad(shape, t, j, torch.bfloat16).cuda(),
                            m=torch.from_numpy(st["m"]).float().cuda(), v=torch.from_numpy(st["v"]).float().cuda()))
        return out

    sizes = [768, 2304, 65541, (3, 5)]
    state = _state(torch.bfloat16, sizes)
    sched = mo.quintic_schedule(5)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in (1, 2):
        A, B = mats(), mats()
        VA, VB = vecs(state, t), vecs(state, t)
        ws = torch.empty(mo.muon_workspace_size(A, mo.BF16, sched), dtype=torch.uint8, device="cuda")
        mo.muon_model_step(A, VA, mo.BF16, mo.BF16, hp, HP, t, sched, ws, d_status=status)
        mo.muon_step_batched(B, mo.BF16, mo.BF16, hp, sched, ws)
        mo.adamw_step_batched(VB, mo.BF16, HP, t)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for a, b in zip(A, B):
            for k in ("W", "G_prev", "A", "M"):
                assert torch.equal(a[k], b[k]), k
        for j, (a, b) in enumerate(zip(VA, VB)):
            for k in ("W", "m", "v"):
                assert torch.equal(a[k], b[k]), (j, k)
            st = state[j]
            g = a["G"].double().cpu().numpy()
            W_ref, m_ref, v_ref = oracle.adamw(st["W"], g, st["m"], st["v"], step=t, **HP32)
            # this file's per-element bounds on the moments (the same bits as adamw_step_batched)
            b1, b2 = HP32["beta1"], HP32["beta2"]
            mg, vg = a["m"].double().cpu().numpy(), a["v"].double().cpu().numpy()
            assert np.all(np.abs(mg - m_ref) <= 2.0 ** -22 * (b1 * np.abs(st["m"]) + (1 - b1) * np.abs(g)))
            assert np.all(np.abs(vg - v_ref) <= 2.0 ** -21 * (b2 * st["v"] + (1 - b2) * g * g))
            state[j] = dict(W=_round(W_ref, torch.bfloat16), m=_round(m_ref, torch.float32),
                            v=_round(v_ref, torch.float32))
    # a non-finite vector gradient: that element keeps its state, the flag is raised
    A, V = mats(), vecs(state, 3)
    V[1]["G"][7] = float("nan")
    w7 = V[1]["W"][7].clone()
    status.zero_()
    mo.muon_model_step(A, V, mo.BF16, mo.BF16, hp, HP, 3, sched, ws, d_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & mo.FLAG_NONFINITE
    assert torch.equal(V[1]["W"][7], w7)
