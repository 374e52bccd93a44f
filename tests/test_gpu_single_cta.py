"""The one-CTA-per-tile kernels (MUON_CTA_PAIRS=0) against the oracle.

By default the library runs every tensor-core product on CTA pairs; the
environment switch selects the one-CTA kernels for the whole process, so this
test runs the parity cases in a child process."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, %r)
import numpy as np, torch
import muon_family_optimizer_b200 as mo, oracle
from muon_family_optimizer_b200 import synthetic as syn
Q = (3.4445, -4.7750, 2.0315)
def f64(t): return t.detach().float().cpu().double().numpy()
def rel(a, b): return np.linalg.norm(a - b) / np.linalg.norm(b)
worst = 0.0
for shape, b, dt in [((200, 328), 2, torch.bfloat16), ((768, 3072), 1, torch.bfloat16),
                     ((300, 130), 2, torch.float16), ((520, 520), 1, torch.bfloat16)]:
    X = torch.stack([syn.gaussian(shape, 7 + i) for i in range(b)]).to(dt).cuda()
    out = torch.empty_like(X)
    ws = torch.empty(mo.ns_polar_workspace_size(b, *shape, mo._dtype_code(dt)), dtype=torch.uint8, device="cuda")
    mo.ns_polar(X, out, mo.quintic_schedule(5), ws)
    torch.cuda.synchronize()
    for i in range(b):
        worst = max(worst, rel(f64(out[i]), oracle.orthogonalise(f64(X[i]), [Q] * 5)))
M = syn.log_spectrum(256, 640, 1e3, 77).to(torch.float16).cuda()
out = torch.empty_like(M)
ws = torch.empty(mo.gram_polar_workspace_size(1, 256, 640, mo.FP16), dtype=torch.uint8, device="cuda")
mo.gram_polar(M, out, mo.converged_schedule(), ws)
torch.cuda.synchronize()
gram = rel(f64(out), oracle.polar(f64(M)))
print(worst, gram)
""" % ROOT


def test_single_cta_kernels_match_oracle():
    env = dict(os.environ, MUON_CTA_PAIRS="0")
    out = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    worst, gram = map(float, out.stdout.split()[-2:])
    assert worst <= 3e-2
    assert gram <= 2e-2
