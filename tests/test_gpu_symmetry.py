"""Exact symmetry of the stored symmetric products (white-box).

The symmetric results A = X X^T and B' = aI + bA + cA^2 are stored as their
128 x 128 blocks on and above the diagonal; consumers read a block left of the
diagonal as the transpose of its mirror.  So every stored diagonal block must be
exactly (bitwise) symmetric, and where a CTA pair consumes the result the first
block below the diagonal must be the exact transpose of its mirror.  Products of
one operand with itself get this from the tensor cores (entries (i, j) and
(j, i) are sums of the same products in the same order); this test checks it
on the stored bits, for the CTA-pair kernels in this process and for the
one-CTA kernels (MUON_CTA_PAIRS=0) in a child process.

The workspace layout read here is the library's internal one for ns_polar
(status word, fp64 norms, two s x l buffers, then the s x s buffers), with rows
padded to 8 elements and every region aligned to 1024 bytes.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))

import muon_family_optimizer_b200 as mo  # noqa: E402
from muon_family_optimizer_b200 import synthetic as syn  # noqa: E402

pytestmark = pytest.mark.gpu

CASES = [(768, 768), (768, 3072), (700, 1000), (3072, 768), (1100, 1100), (1100, 2600), (2600, 1100)]


def _align(x, a=1024):
    return (x + a - 1) // a * a


def _pad8(x):
    return (x + 7) // 8 * 8


def symmetric_buffers(rows, cols, dtype, batch=3):
    """Run one quintic step; return the stored X X^T and B' (int16 bit patterns)."""
    X = torch.stack([syn.power_law(rows, cols, 91 + i, device="cuda") for i in range(batch)]).to(dtype)
    X = X.contiguous()
    out = torch.empty_like(X)
    ws = torch.zeros(mo.ns_polar_workspace_size(batch, rows, cols, mo._dtype_code(dtype)), dtype=torch.uint8,
                     device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mo.ns_polar(X, out, mo.quintic_schedule(1), ws, d_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    s, l = min(rows, cols), max(rows, cols)
    ldl, lds = _pad8(l), _pad8(s)
    off = _align(_align(256) + 8 * batch)
    off = _align(off + batch * s * ldl * 2)          # x[0]
    off = _align(off + batch * s * ldl * 2)          # x[1]
    bufs = []
    for _ in range(2):                                # X X^T, then B'
        b = ws[off:off + batch * s * lds * 2].view(torch.int16).view(batch, s, lds)[:, :, :s]
        bufs.append(b.cpu().numpy())
        off = _align(off + batch * s * lds * 2)
    return bufs


def check(pairs):
    failures = []
    for dtype in (torch.bfloat16, torch.float16):
        for rows, cols in CASES:
            for name, buf in zip(("XX^T", "B'"), symmetric_buffers(rows, cols, dtype)):
                s = buf.shape[1]
                nb = (s + 127) // 128
                for bi in range(nb):
                    a0, a1 = 128 * bi, min(s, 128 * bi + 128)
                    d = buf[:, a0:a1, a0:a1]
                    if not np.array_equal(d, d.transpose(0, 2, 1)):
                        failures.append((str(dtype), rows, cols, name, "diagonal", bi))
                    if pairs and bi + 1 < nb:
                        b0, b1 = a1, min(s, a1 + 128)
                        if not np.array_equal(buf[:, b0:b1, a0:a1], buf[:, a0:a1, b0:b1].transpose(0, 2, 1)):
                            failures.append((str(dtype), rows, cols, name, "band", bi))
    return failures


def test_symmetric_storage_exact_cta_pairs():
    assert check(pairs=True) == []


def test_symmetric_storage_exact_one_cta():
    env = dict(os.environ, MUON_CTA_PAIRS="0")
    code = (f"import sys; sys.path.insert(0, {HERE!r}); import test_gpu_symmetry as t; "
            "f = t.check(pairs=False); print('FAILURES', f); sys.exit(1 if f else 0)")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
