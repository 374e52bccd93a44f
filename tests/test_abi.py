"""The C ABI library loads, exports every entry point include/muon.h declares,
and its host-side checks behave -- no GPU needed (no compute is launched).

The ctypes structures of the Python binding are checked against the C
header's layout by compiling a probe with gcc that prints sizeof/offsetof.
"""
import ctypes
import os
import re
import subprocess

import pytest

import muon_family_optimizer_b200 as mo
from muon_family_optimizer_b200 import build as mbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "muon.h")


@pytest.fixture(scope="module")
def lib():
    mbuild.build()
    return mo.lib()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"MUON_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) >= {"muon_step_batched", "ns_polar", "gram_polar", "muon_workspace_size",
                          "muon_status_string"}
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", mo.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(names) <= exported


def test_library_links_no_cuda_runtime_dynamically(lib):
    out = subprocess.run(["ldd", mo.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcudart" not in out and "libtorch" not in out


PROBE = r"""
#include <stdio.h>
#include <stddef.h>
#include "muon.h"
#define P(T, f) printf(#T "." #f " %zu\n", offsetof(T, f));
int main(void) {
  printf("muon_param %zu\n", sizeof(muon_param));
  printf("muon_schedule %zu\n", sizeof(muon_schedule));
  printf("muon_hparams %zu\n", sizeof(muon_hparams));
  printf("muon_ns_coeff %zu\n", sizeof(muon_ns_coeff));
  printf("muon_lite_param %zu\n", sizeof(muon_lite_param));
  printf("muon_vec_param %zu\n", sizeof(muon_vec_param));
  printf("muon_adamw_hparams %zu\n", sizeof(muon_adamw_hparams));
  printf("muon_rsvd_param %zu\n", sizeof(muon_rsvd_param));
  printf("muon_rsvd_hparams %zu\n", sizeof(muon_rsvd_hparams));
  P(muon_rsvd_param, rows) P(muon_rsvd_param, cols) P(muon_rsvd_param, W) P(muon_rsvd_param, G)
  P(muon_rsvd_param, M) P(muon_rsvd_param, Omega) P(muon_rsvd_param, gamma) P(muon_rsvd_param, O_out)
  P(muon_rsvd_hparams, mu) P(muon_rsvd_hparams, eta) P(muon_rsvd_hparams, lambda) P(muon_rsvd_hparams, gamma)
  P(muon_rsvd_hparams, rank) P(muon_rsvd_hparams, oversample)
  P(muon_vec_param, n) P(muon_vec_param, W) P(muon_vec_param, G) P(muon_vec_param, m) P(muon_vec_param, v)
  P(muon_adamw_hparams, lr) P(muon_adamw_hparams, beta1) P(muon_adamw_hparams, beta2) P(muon_adamw_hparams, eps)
  P(muon_adamw_hparams, weight_decay)
  P(muon_lite_param, rows) P(muon_lite_param, cols) P(muon_lite_param, W) P(muon_lite_param, G)
  P(muon_lite_param, B) P(muon_lite_param, M) P(muon_lite_param, gamma) P(muon_lite_param, O_out)
  P(muon_param, rows) P(muon_param, cols) P(muon_param, W) P(muon_param, G) P(muon_param, G_prev)
  P(muon_param, A) P(muon_param, M) P(muon_param, gamma) P(muon_param, O_out)
  P(muon_schedule, n_steps) P(muon_schedule, coeffs) P(muon_schedule, eps)
  P(muon_schedule, restarts) P(muon_schedule, n_restarts) P(muon_schedule, scale_f)
  P(muon_schedule, gram_aspect)
  P(muon_hparams, mu) P(muon_hparams, eta) P(muon_hparams, lambda) P(muon_hparams, gamma)
  P(muon_hparams, beta_a) P(muon_hparams, alpha)
  return 0;
}
"""


def test_binding_struct_layout_matches_header(tmp_path):
    src = tmp_path / "probe.c"
    src.write_text(PROBE)
    exe = tmp_path / "probe"
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)])
    got = dict(line.rsplit(" ", 1) for line in subprocess.check_output([str(exe)], text=True).splitlines())
    assert int(got["muon_param"]) == ctypes.sizeof(mo.Param)
    assert int(got["muon_schedule"]) == ctypes.sizeof(mo.Schedule)
    assert int(got["muon_hparams"]) == ctypes.sizeof(mo.HParams)
    assert int(got["muon_ns_coeff"]) == ctypes.sizeof(mo.NsCoeff)
    assert int(got["muon_lite_param"]) == ctypes.sizeof(mo.LiteParam)
    assert int(got["muon_vec_param"]) == ctypes.sizeof(mo.VecParam)
    assert int(got["muon_adamw_hparams"]) == ctypes.sizeof(mo.AdamWHParams)
    assert int(got["muon_rsvd_param"]) == ctypes.sizeof(mo.RsvdParam)
    assert int(got["muon_rsvd_hparams"]) == ctypes.sizeof(mo.RsvdHParams)
    py = {"muon_param": mo.Param, "muon_schedule": mo.Schedule, "muon_hparams": mo.HParams,
          "muon_lite_param": mo.LiteParam, "muon_vec_param": mo.VecParam,
          "muon_adamw_hparams": mo.AdamWHParams, "muon_rsvd_param": mo.RsvdParam,
          "muon_rsvd_hparams": mo.RsvdHParams}
    for key, val in got.items():
        if "." not in key:
            continue
        struct, field = key.split(".")
        field = "lambda_" if field == "lambda" else field
        assert getattr(py[struct], field).offset == int(val), key


def test_status_strings(lib):
    for code in range(7):
        s = mo.muon_status_string(code)
        assert s and s != "unknown status"
    assert mo.muon_status_string(99) == "unknown status"


def test_workspace_size_queries_are_host_only(lib):
    arr = (mo.Param * 3)()
    for i, (r, c) in enumerate([(768, 768), (768, 3072), (3072, 768)]):
        arr[i].rows, arr[i].cols = r, c
    n16 = mo.muon_workspace_size(arr, mo.BF16)
    n32 = mo.muon_workspace_size(arr, mo.FP32)
    assert n16 > 0 and n32 > n16
    # the two 768x3072 orientations share a group: 2 X buffers of 2 x 768 x 3072,
    # 2 square buffers of 2 x 768 x 768, plus 768x768 group -- in bf16
    lower = 2 * (2 * 768 * 3072 * 2) + 2 * (2 * 768 * 768 * 2) + 4 * (768 * 768 * 2)
    assert lower <= n16 <= lower + 64 * 1024
    assert mo.ns_polar_workspace_size(4, 100, 300, mo.BF16) < mo.gram_polar_workspace_size(4, 100, 300, mo.BF16)
    # a schedule with the Gram route on elongated groups: the 768x3072 group takes
    # four more 768x768 buffers, the square group stays direct
    gram = mo.quintic_gram_schedule(5, gram_aspect=2.0)
    assert mo.muon_workspace_size(arr, mo.BF16, gram) - n16 in range(4 * 2 * 768 * 768 * 2,
                                                                     4 * 2 * 768 * 768 * 2 + 8 * 1024)
    assert mo.muon_workspace_size(arr, mo.BF16, mo.quintic_schedule(5)) == n16
    assert mo.muon_workspace_size(arr, mo.BF16, mo.quintic_gram_schedule(5, gram_aspect=5.0)) == n16


def test_narrow_groups_take_fp32_buffers(lib):
    # a short side below 16 is iterated in fp32 whatever the iteration type:
    # its buffers are sized in 4-byte elements
    arr = (mo.Param * 1)()
    arr[0].rows, arr[0].cols = 15, 1000
    n16 = mo.muon_workspace_size(arr, mo.BF16)
    assert n16 == mo.muon_workspace_size(arr, mo.FP32)
    arr[0].rows = 16
    assert mo.muon_workspace_size(arr, mo.BF16) < mo.muon_workspace_size(arr, mo.FP32)


def test_schedule_gram_aspect_is_validated(lib):
    arr = (mo.Param * 1)()
    arr[0].rows, arr[0].cols = 64, 256
    sz = ctypes.c_size_t(0)
    for bad in (-1.0, float("nan"), float("inf")):
        sched = mo.make_schedule([mo.QUINTIC] * 5, gram_aspect=bad)
        assert lib.muon_workspace_size(arr, 1, mo.BF16, ctypes.byref(sched), ctypes.byref(sz)) == mo.ERR_INVALID_ARG


def test_invalid_arguments_are_rejected_before_any_launch(lib):
    L = lib
    sched = mo.quintic_schedule(5)
    bad = mo.make_schedule([(1, 0, 0)], restarts=[5])        # restart beyond n_steps
    sz = ctypes.c_size_t(0)
    assert L.ns_polar_workspace_size(0, 4, 4, mo.BF16, ctypes.byref(sz)) == mo.ERR_INVALID_ARG
    assert L.ns_polar_workspace_size(1, 4, 4, 7, ctypes.byref(sz)) == mo.ERR_INVALID_ARG
    assert L.ns_polar(None, None, 1, 4, 4, 16, mo.BF16, ctypes.byref(sched), None, 0, None, None) == \
        mo.ERR_INVALID_ARG
    buf = ctypes.create_string_buffer(64)
    p = ctypes.cast(buf, ctypes.c_void_p)
    assert L.ns_polar(p, p, 1, 4, 4, 16, mo.BF16, ctypes.byref(bad), p, 64, None, None) == mo.ERR_INVALID_ARG
    # workspace too small is reported as such (still before any device call)
    assert L.ns_polar(p, p, 1, 4, 4, 16, mo.BF16, ctypes.byref(sched), p, 1, None, None) == mo.ERR_WORKSPACE
    nan_sched = mo.make_schedule([(float("nan"), 0, 0)])
    assert L.gram_polar(p, p, 1, 4, 4, 16, mo.BF16, ctypes.byref(nan_sched), p, 1 << 20, None, None) == \
        mo.ERR_INVALID_ARG
    arr = (mo.Param * 1)()
    arr[0].rows, arr[0].cols = 4, 4
    hp = mo.HParams(0.9, 0.02, 0.0, 1.0, 0.9, 0.5)
    # W/G/... NULL
    assert L.muon_step_batched(arr, 1, mo.BF16, mo.BF16, ctypes.byref(hp), ctypes.byref(sched), p, 1 << 20,
                               None, None) == mo.ERR_INVALID_ARG


def test_lite_entry_points_host_checks(lib):
    L = lib
    shapes = [(768, 768), (768, 3072), (3072, 768)]
    arr = (mo.Param * 3)()
    lite = (mo.LiteParam * 3)()
    for i, (r, c) in enumerate(shapes):
        arr[i].rows, arr[i].cols = r, c
        lite[i].rows, lite[i].cols = r, c
    # same iteration workspace as the full step
    assert mo.muon_lite_workspace_size(lite, mo.BF16) == mo.muon_workspace_size(arr, mo.BF16)
    sz = ctypes.c_size_t(0)
    assert L.muon_lite_workspace_size(None, 1, mo.BF16, None, ctypes.byref(sz)) == mo.ERR_INVALID_ARG
    assert L.muon_lite_workspace_size(lite, 0, mo.BF16, None, ctypes.byref(sz)) == mo.ERR_INVALID_ARG
    sched = mo.quintic_schedule(5)
    hp = mo.HParams(0.9, 0.02, 0.0, 1.0, 0.9, 0.5)
    buf = ctypes.create_string_buffer(64)
    p = ctypes.cast(buf, ctypes.c_void_p)
    # NULL W / G / B / M
    assert L.muon_lite_step_batched(lite, 1, mo.BF16, mo.BF16, ctypes.byref(hp), ctypes.byref(sched), p,
                                    1 << 20, None, None) == mo.ERR_INVALID_ARG
    one = (mo.LiteParam * 1)()
    one[0] = mo.LiteParam(4, 4, p.value, p.value, None, p.value, float("nan"), None)
    assert L.muon_lite_step_batched(one, 1, mo.BF16, mo.BF16, ctypes.byref(hp), ctypes.byref(sched), p,
                                    1 << 20, None, None) == mo.ERR_INVALID_ARG


def test_adamw_argument_checks(lib):
    L = lib
    buf = ctypes.create_string_buffer(64)
    p = ctypes.cast(buf, ctypes.c_void_p).value
    good = mo.AdamWHParams(1e-3, 0.9, 0.999, 1e-8, 0.01)
    one = (mo.VecParam * 1)(mo.VecParam(4, p, p, p, p))
    assert L.adamw_step_batched(None, 1, mo.BF16, ctypes.byref(good), 1, None, None) == mo.ERR_INVALID_ARG
    assert L.adamw_step_batched(one, 0, mo.BF16, ctypes.byref(good), 1, None, None) == mo.ERR_INVALID_ARG
    assert L.adamw_step_batched(one, 1, mo.BF16, ctypes.byref(good), 0, None, None) == mo.ERR_INVALID_ARG
    assert L.adamw_step_batched(one, 1, 9, ctypes.byref(good), 1, None, None) == mo.ERR_INVALID_ARG
    for bad in (mo.AdamWHParams(1e-3, 1.0, 0.999, 1e-8, 0.0), mo.AdamWHParams(1e-3, 0.9, -0.1, 1e-8, 0.0),
                mo.AdamWHParams(float("nan"), 0.9, 0.999, 1e-8, 0.0), mo.AdamWHParams(1e-3, 0.9, 0.999, -1.0, 0.0)):
        assert L.adamw_step_batched(one, 1, mo.BF16, ctypes.byref(bad), 1, None, None) == mo.ERR_INVALID_ARG
    nul = (mo.VecParam * 1)(mo.VecParam(4, p, None, p, p))
    assert L.adamw_step_batched(nul, 1, mo.BF16, ctypes.byref(good), 1, None, None) == mo.ERR_INVALID_ARG
    empty = (mo.VecParam * 1)(mo.VecParam(0, p, p, p, p))
    assert L.adamw_step_batched(empty, 1, mo.BF16, ctypes.byref(good), 1, None, None) == mo.ERR_INVALID_ARG


def test_limuon_argument_checks(lib):
    L = lib
    buf = ctypes.create_string_buffer(4096)
    p = ctypes.cast(buf, ctypes.c_void_p).value
    ws = (p + 255) & ~255
    good = mo.RsvdHParams(0.95, 0.02, 0.0, 1.0, 16, 16)
    one = (mo.RsvdParam * 1)(mo.RsvdParam(4, 8, p, p, p, p, float("nan"), None))
    size = ctypes.c_size_t(0)
    assert L.limuon_workspace_size(one, 1, ctypes.byref(good), ctypes.byref(size)) == mo.OK
    # the per-matrix flag, three k x k fp64 matrices (Y^T Y, B B^T, the factor) on 32 columns,
    # then Y and its low parts (4 x 32 floats each) and B^T and its low parts (8 x 32 floats
    # each), each region 256-byte aligned
    assert size.value == 256 + 3 * 32 * 32 * 8 + 2 * 512 + 2 * 1024
    big = mo.RsvdHParams(0.95, 0.02, 0.0, 1.0, 40, 8)
    assert L.limuon_workspace_size(one, 1, ctypes.byref(big), ctypes.byref(size)) == mo.OK
    assert size.value == 256 + 3 * 64 * 64 * 8 + 2 * 1024 + 2 * 2048   # k = 48 runs on 64 columns
    # 2500 rows: three projection segments of at most 1024 rows, so one segment counter for the
    # single 128-column block and the three partial B^T (3 x 8 x 32 floats)
    tall = (mo.RsvdParam * 1)(mo.RsvdParam(2500, 8, p, p, p, p, float("nan"), None))
    assert L.limuon_workspace_size(tall, 1, ctypes.byref(good), ctypes.byref(size)) == mo.OK
    assert size.value == 256 + 256 + 3 * 32 * 32 * 8 + 2 * 2500 * 32 * 4 + 2 * 1024 + 3 * 1024
    too_big = mo.RsvdHParams(0.95, 0.02, 0.0, 1.0, 60, 5)
    assert L.limuon_workspace_size(one, 1, ctypes.byref(too_big), ctypes.byref(size)) == mo.ERR_UNSUPPORTED
    for bad in (mo.RsvdHParams(0.95, 0.02, 0.0, 1.0, 0, 4), mo.RsvdHParams(0.95, 0.02, 0.0, 1.0, 4, -1),
                mo.RsvdHParams(float("nan"), 0.02, 0.0, 1.0, 4, 4), mo.RsvdHParams(0.95, float("inf"), 0.0, 1.0, 4, 4)):
        assert L.limuon_workspace_size(one, 1, ctypes.byref(bad), ctypes.byref(size)) == mo.ERR_INVALID_ARG
        assert L.limuon_step_batched(one, 1, mo.BF16, ctypes.byref(bad), ws, 2048, None, None) == mo.ERR_INVALID_ARG
    assert L.limuon_step_batched(one, 0, mo.BF16, ctypes.byref(good), ws, 2048, None, None) == mo.ERR_INVALID_ARG
    assert L.limuon_step_batched(one, 1, 7, ctypes.byref(good), ws, 2048, None, None) == mo.ERR_INVALID_ARG
    assert L.limuon_step_batched(one, 1, mo.BF16, ctypes.byref(good), ws, 1000, None, None) == mo.ERR_WORKSPACE
    assert L.limuon_step_batched(one, 1, mo.BF16, ctypes.byref(good), None, 4096, None, None) == mo.ERR_WORKSPACE
    assert L.limuon_step_batched(one, 1, mo.BF16, ctypes.byref(good), ws + 16, 1 << 20, None, None) == \
        mo.ERR_INVALID_ARG
    nul = (mo.RsvdParam * 1)(mo.RsvdParam(4, 8, p, p, p, None, float("nan"), None))
    assert L.limuon_step_batched(nul, 1, mo.BF16, ctypes.byref(good), ws, 2048, None, None) == mo.ERR_INVALID_ARG
    empty = (mo.RsvdParam * 1)(mo.RsvdParam(0, 8, p, p, p, p, float("nan"), None))
    assert L.limuon_workspace_size(empty, 1, ctypes.byref(good), ctypes.byref(size)) == mo.ERR_INVALID_ARG


def test_limuon_binding_validates_tensors():
    import torch
    W = torch.zeros(4, 8, dtype=torch.bfloat16)
    ok = dict(W=W, G=torch.zeros(4, 8, dtype=torch.bfloat16), M=torch.zeros(4, 8), Omega=torch.zeros(8, 5))
    arr = mo.make_rsvd_params([ok])
    assert arr[0].rows == 4 and arr[0].cols == 8 and arr[0].Omega == ok["Omega"].data_ptr()
    import math
    assert math.isnan(arr[0].gamma) and arr[0].O_out is None
    for bad in (dict(ok, M=torch.zeros(4, 8, dtype=torch.float64)), dict(ok, Omega=torch.zeros(7, 5)),
                dict(ok, G=torch.zeros(4, 8)), dict(ok, O_out=torch.zeros(4, 8, dtype=torch.bfloat16)),
                dict(ok, W=torch.zeros(32, dtype=torch.bfloat16)), dict(ok, M=torch.zeros(8, 4).t())):
        with pytest.raises(ValueError):
            mo.make_rsvd_params([bad])


def test_model_step_argument_checks(lib):
    L = lib
    buf = ctypes.create_string_buffer(4096)
    p = ctypes.cast(buf, ctypes.c_void_p).value
    arr = (mo.Param * 1)()
    arr[0].rows, arr[0].cols = 4, 4
    arr[0].W = arr[0].G = arr[0].G_prev = arr[0].A = arr[0].M = p
    hp = mo.HParams(0.9, 0.02, 0.0, 1.0, 0.9, 0.5)
    sched = mo.quintic_schedule(5)
    good = mo.AdamWHParams(1e-3, 0.9, 0.999, 1e-8, 0.1)
    vec = (mo.VecParam * 1)(mo.VecParam(8, p, p, p, p))
    args = lambda v, nv, a, t, ws=p, size=16: (arr, 1, v, nv, mo.BF16, mo.BF16, ctypes.byref(hp), a, t,
                                               ctypes.byref(sched), ws, size, None, None)
    assert L.muon_model_step(*args(vec, -1, ctypes.byref(good), 1)) == mo.ERR_INVALID_ARG
    assert L.muon_model_step(*args(vec, 1, None, 1)) == mo.ERR_INVALID_ARG                 # no AdamW hparams
    assert L.muon_model_step(*args(vec, 1, ctypes.byref(good), 0)) == mo.ERR_INVALID_ARG   # step t < 1
    bad = mo.AdamWHParams(1e-3, 1.0, 0.999, 1e-8, 0.1)                                        # beta1 = 1
    assert L.muon_model_step(*args(vec, 1, ctypes.byref(bad), 1)) == mo.ERR_INVALID_ARG
    nul = (mo.VecParam * 1)(mo.VecParam(8, p, None, p, p))
    assert L.muon_model_step(*args(nul, 1, ctypes.byref(good), 1)) == mo.ERR_INVALID_ARG
    # without vectors the AdamW arguments are not read; a too small workspace is then the error
    assert L.muon_model_step(*args(None, 0, None, 0)) == mo.ERR_WORKSPACE
