"""ns_polar_noalloc: the entry point for callers that cannot allocate a
workspace (graph capture, restricted allocators, plugins handed only their
buffers).  It must give the same result as ns_polar with a caller workspace,
call after call, although both calls share the library's fixed scratch.

This file is collected last so that a failure here leaves every other test
already run."""
import pytest
import torch

import muon_family_optimizer_b200 as mo
from conftest import rel_fro

pytestmark = pytest.mark.gpu


def _reference(X, sched):
    ws = torch.empty(mo.ns_polar_workspace_size(*X.shape, mo._dtype_code(X.dtype)), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty_like(X)
    mo.ns_polar(X, out, sched, ws)
    return out


def test_noalloc_matches_workspace_entry_point_twice():
    from muon_family_optimizer_b200 import synthetic as syn
    sched = mo.quintic_schedule(5)
    cases = [syn.gaussian((3, 200, 456), 21).to(torch.bfloat16).cuda(),
             syn.gaussian((2, 520, 130), 22).to(torch.float16).cuda()]
    for X in cases:
        ref = _reference(X, sched)
        for _ in range(2):                      # two calls in a row on the shared scratch
            out = torch.full_like(X, float("nan"))
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
            mo.ns_polar_noalloc(X, out, sched, d_status=status)
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            for b in range(X.shape[0]):
                assert rel_fro(out[b].float().cpu().numpy(), ref[b].float().cpu().numpy()) <= 3e-2


def test_noalloc_rejects_requests_beyond_its_scratch():
    cap = mo.ns_polar_noalloc_capacity()
    assert cap == 32 << 20
    X = torch.zeros(1, 8, 8, dtype=torch.bfloat16, device="cuda")
    sched = mo.quintic_schedule(5)
    big = 4096
    assert mo.ns_polar_workspace_size(1, big, big, mo.BF16) > cap
    with pytest.raises(mo.MuonError) as err:
        # sizes are checked before any pointer is used or anything is enqueued
        mo.lib()
        st = mo.lib().ns_polar_noalloc(mo._ptr(X), mo._ptr(X), 1, big, big, big * big, mo.BF16,
                                       mo.ctypes.byref(sched), None, mo._stream_ptr(None))
        mo._check(st, "ns_polar_noalloc")
    assert err.value.status == mo.ERR_WORKSPACE
