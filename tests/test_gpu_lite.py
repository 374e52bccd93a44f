"""GPU parity of MONA-Lite (muon_lite_step_batched) against the fp64 oracle.

Three steps from a zero state.  Every step starts both sides from the same
state: the oracle's state rounded to the storage types (W in its dtype, B in
bfloat16, M in fp32) is written into the GPU's buffers, both take one step
from it, and the results are compared.  Tolerances (relative Frobenius unless
stated):
  M (fp32)          1e-6
  B (bfloat16)      elementwise |B_gpu - B_ref| <= ulp(B_ref)
                              + 2^-21 (beta_a |A_k| + (1 - beta_a) |G_k|):
                    one bfloat16 rounding that may fall on the other side of a
                    tie, since the GPU forms B = beta_a A_k - (1 - beta_a) G_k in
                    fp32 with fp32 beta_a and 1 - beta_a (relative 2^-22 each,
                    doubled; B may cancel to far below its terms); and >= 99 %
                    of all elements identical
  O                 3e-2 against the oracle from the same rounded start; a
                    short side below 16 (the 130 x 2 and 1 x 48 cases) is
                    iterated in fp32 by the library, so there O is checked at
                    1e-4 against the oracle from the unrounded momentum
  W                 bf16: 2^-8; fp32: the update W - W0 within O's tolerance
                    (it is eta (gamma O + lambda W), dominated by O)
First step from zero: A_1 = (1 - beta_a) G in both forms, so M and W equal
muon_step_batched's bit for bit.
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
HP = dict(mu=0.95, eta=0.02, gamma=1.0, beta_a=0.9, alpha=0.5, **{"lambda": 0.1})
SHAPES = [(256, 256), (192, 520), (520, 192), (100, 36), (1, 48), (130, 2), (768, 3072)]


def f64(t):
    return t.detach().to(torch.float32).cpu().double().numpy()


def _ulp_bf16(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 7)


def _grads(shape, j, t):
    return syn.gradient("gpt2_small", j, t, *shape)


def _lite_state(w_dtype):
    out = []
    for j, (r, c) in enumerate(SHAPES):
        out.append(dict(W=syn.initial_weight("gpt2_small", j, r, c).to(w_dtype).cuda(),
                        B=torch.zeros(r, c, dtype=torch.bfloat16, device="cuda"),
                        M=torch.zeros(r, c, dtype=torch.float32, device="cuda"),
                        O_out=torch.empty(r, c, dtype=torch.float32, device="cuda")))
    return out


def _run(params, w_dtype, ns_dtype, lite=True):
    sched = mo.quintic_schedule(5)
    size = (mo.muon_lite_workspace_size if lite else mo.muon_workspace_size)(params, mo._dtype_code(ns_dtype), sched)
    ws = torch.empty(size, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    (mo.muon_lite_step_batched if lite else mo.muon_step_batched)(
        params, mo._dtype_code(w_dtype), mo._dtype_code(ns_dtype), HP, sched, ws, d_status=status)
    torch.cuda.synchronize()
    return int(status.item())


@pytest.mark.parametrize("w_dtype,ns_dtype", [(torch.bfloat16, torch.bfloat16), (torch.float32, torch.bfloat16),
                                              (torch.bfloat16, torch.float16)])
def test_lite_three_steps_vs_oracle(w_dtype, ns_dtype):
    gpu = _lite_state(w_dtype)
    round_w = oracle.round_bf16 if w_dtype == torch.bfloat16 else oracle.round_fp32
    state = [dict(W=f64(p["W"]), B=np.zeros(p["W"].shape), M=np.zeros(p["W"].shape)) for p in gpu]
    beta = HP["beta_a"]
    rnd = oracle.ROUND_BF16 if ns_dtype == torch.bfloat16 else oracle.ROUND_FP16
    for t in range(3):
        for j, p in enumerate(gpu):
            S = state[j]
            p["G"] = _grads(SHAPES[j], j, t).to(w_dtype).cuda().contiguous()
            p["W"].copy_(torch.from_numpy(S["W"]))
            p["B"].copy_(torch.from_numpy(S["B"]))
            p["M"].copy_(torch.from_numpy(S["M"]))
        assert _run(gpu, w_dtype, ns_dtype) == 0
        same, total = 0, 0
        for j, p in enumerate(gpu):
            S = state[j]
            G = f64(p["G"])
            A_k = S["B"] + (1 - beta) * G
            narrow = min(SHAPES[j]) < 16
            out = oracle.muon_lite_step(S["W"], G, S["B"], S["M"], mu=HP["mu"], eta=HP["eta"],
                                        lam=HP["lambda"], gamma=HP["gamma"], beta_a=beta,
                                        alpha=HP["alpha"], coeffs=[QUINTIC] * 5,
                                        round_to=oracle.ROUND_NONE if narrow else rnd, round_b=True)
            assert rel_fro(f64(p["M"]), out["M"]) <= 1e-6, (t, j)
            Bg = f64(p["B"])
            bnd = _ulp_bf16(out["B"]) + 2.0 ** -21 * (beta * np.abs(A_k) + (1 - beta) * np.abs(G))
            assert np.all(np.abs(Bg - out["B"]) <= bnd), (t, j, float(np.max(np.abs(Bg - out["B"]) - bnd)))
            same += int(np.sum(Bg == out["B"]))
            total += Bg.size
            tol_o = 1e-4 if narrow else 3e-2
            assert rel_fro(f64(p["O_out"]), out["O"]) <= tol_o, (t, j)
            if w_dtype == torch.float32:
                # the update eta (gamma O + lambda W) carries O's relative error
                assert rel_fro(f64(p["W"]) - S["W"], out["W"] - S["W"]) <= tol_o, (t, j)
            else:
                assert rel_fro(f64(p["W"]), out["W"]) <= 2.0 ** -8, (t, j)
            state[j] = dict(W=round_w(out["W"]), B=out["B"], M=oracle.round_fp32(out["M"]))
        assert same / total >= 0.99, t


def test_lite_first_step_equals_full_mona_step():
    lite = _lite_state(torch.bfloat16)
    full = []
    for j, p in enumerate(lite):
        p["G"] = _grads(SHAPES[j], j, 0).to(torch.bfloat16).cuda().contiguous()
        full.append(dict(W=p["W"].clone(), G=p["G"], G_prev=torch.zeros_like(p["G"]),
                         A=torch.zeros_like(p["M"]), M=torch.zeros_like(p["M"]),
                         O_out=torch.empty_like(p["M"])))
    assert _run(lite, torch.bfloat16, torch.bfloat16, lite=True) == 0
    assert _run(full, torch.bfloat16, torch.bfloat16, lite=False) == 0
    for a, b in zip(lite, full):
        assert torch.equal(a["M"], b["M"])
        assert torch.equal(a["W"], b["W"])
        # B_1 = beta_a A_1 - (1 - beta_a) G with A_1 = (1 - beta_a) G, rounded once
        expect = (HP["beta_a"] * b["A"] - (1 - HP["beta_a"]) * b["G"].float()).to(torch.bfloat16)
        diff = (a["B"].float() - expect.float()).abs()
        assert torch.all(diff <= torch.from_numpy(_ulp_bf16(f64(expect))).cuda().float())


def test_lite_nonfinite_keeps_weights():
    params = _lite_state(torch.bfloat16)[:2]
    for j, p in enumerate(params):
        p["G"] = _grads(SHAPES[j], j, 0).to(torch.bfloat16).cuda().contiguous()
    params[1]["G"][3, 3] = float("nan")
    W0, W1 = params[0]["W"].clone(), params[1]["W"].clone()
    st = _run(params, torch.bfloat16, torch.bfloat16)
    assert st & mo.FLAG_NONFINITE
    assert torch.equal(params[1]["W"], W1)
    assert not torch.equal(params[0]["W"], W0)
