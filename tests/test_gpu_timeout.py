"""The bounded waits end in a status word, not a hung GPU.

muon_wait_selftest runs the kernels' own wait helper on a barrier nothing
completes, with a 50 ms limit: MUON_FLAG_TIMEOUT must reach the status word,
the launch must finish, and the context must stay usable for the next call.
"""
import time

import pytest
import torch

import muon_family_optimizer_b200 as mo

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_reports_timeout():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    mo.muon_wait_selftest(50, status)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(status.item()) & mo.FLAG_TIMEOUT
    assert 0.04 <= elapsed < 2.0
    # the context is still usable: a normal call afterwards succeeds
    X = torch.randn(128, 256, device="cuda").to(torch.bfloat16)
    out = torch.empty_like(X)
    ws = torch.empty(mo.ns_polar_workspace_size(1, 128, 256, mo.BF16), dtype=torch.uint8, device="cuda")
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    mo.ns_polar(X, out, mo.quintic_schedule(5), ws, d_status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0 and torch.isfinite(out.float()).all()


def test_selftest_argument_checks():
    L = mo.lib()
    assert L.muon_wait_selftest(50, None, None) == mo.ERR_INVALID_ARG
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert L.muon_wait_selftest(0, status.data_ptr(), None) == mo.ERR_INVALID_ARG
    assert L.muon_wait_selftest(5000, status.data_ptr(), None) == mo.ERR_INVALID_ARG
