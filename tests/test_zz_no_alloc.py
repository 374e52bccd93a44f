"""ns_polar_noalloc: the entry point for callers that cannot allocate a
workspace (code running under CUDA graph capture, runtimes whose allocators
forbid outside allocations, plugins handed only their buffers).  It runs the
ns_polar kernels on the library's fixed scratch instead of a caller
workspace, so on the same input it must give exactly ns_polar's result, call
after call, although every call shares (and leaves its data in) that scratch.

This file is collected last so that a failure here leaves every other test
already run."""
import pytest
import torch

import muon_family_optimizer_b200 as mo
import oracle
from conftest import rel_fro

pytestmark = pytest.mark.gpu

QUINTIC = (3.4445, -4.7750, 2.0315)


def _reference(X, sched):
    ws = torch.empty(mo.ns_polar_workspace_size(*X.shape, mo._dtype_code(X.dtype)), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty_like(X)
    mo.ns_polar(X, out, sched, ws)
    return out


def test_noalloc_matches_workspace_entry_point_twice():
    from muon_family_optimizer_b200 import synthetic as syn
    sched = mo.quintic_schedule(5)
    # the larger request runs first, so stale data it leaves in the scratch
    # (e.g. in the padded rows of the smaller call's s x s buffers) would show
    cases = [syn.gaussian((3, 200, 456), 21).to(torch.bfloat16).cuda(),
             syn.gaussian((2, 520, 130), 22).to(torch.float16).cuda()]
    for X in cases:
        ref = _reference(X, sched)
        torch.cuda.synchronize()
        for _ in range(2):                      # two calls in a row on the shared scratch
            out = torch.full_like(X, float("nan"))
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
            mo.ns_polar_noalloc(X, out, sched, d_status=status)
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            # same kernels, same input: the same bits as with a caller workspace
            assert torch.equal(out, ref)
            for b in range(X.shape[0]):
                # and the iteration itself, against the fp64 oracle from the same 16-bit input
                x = X[b].double().cpu().numpy()
                expect = oracle.orthogonalise(x, [QUINTIC] * 5)
                assert rel_fro(out[b].double().cpu().numpy(), expect) <= 3e-2


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
