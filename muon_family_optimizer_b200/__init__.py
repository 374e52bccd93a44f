"""Python binding of the sm_100a Muon / MONA optimizer library (libmuon_b200.so).

Argument marshalling only: every step of the optimizer runs in the CUDA
kernels behind the C ABI of ``include/muon.h``.  PyTorch is used for device
memory and streams.  There is no fallback: if the shared library is missing
or cannot be loaded, every call raises.

Names follow the C ABI: :func:`muon_step_batched`, :func:`ns_polar`,
:func:`gram_polar`, :func:`muon_workspace_size`, :func:`ns_polar_workspace_size`,
:func:`gram_polar_workspace_size`, :func:`muon_lite_step_batched` (MONA-Lite),
:func:`adamw_step_batched` (vector parameters), :func:`muon_model_step` (matrices and
vector parameters in one step), :func:`limuon_step_batched` and
:func:`limuon_workspace_size` (LiMuon), :func:`ns_polar_noalloc`,
:func:`muon_status_string`.
"""
import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# the library next to this file; MUON_B200_LIB names another build of it (A/B comparisons)
LIB_PATH = os.environ.get("MUON_B200_LIB") or os.path.join(_HERE, "libmuon_b200.so")

BF16, FP16, FP32 = 0, 1, 2
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_NONFINITE, ERR_CUDA, ERR_TIMEOUT = range(7)
FLAG_NONFINITE, FLAG_TIMEOUT = 1, 2

# the fixed quintic coefficients (a, b, c) of the Muon iteration
QUINTIC = (3.4445, -4.7750, 2.0315)
# cubic Newton-Schulz for the polar factor (converges for 0 < sigma < sqrt(3))
CUBIC = (1.5, -0.5, 0.0)


class MuonError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {muon_status_string(status)} (status {status})")


class NsCoeff(ctypes.Structure):
    _fields_ = [("a", ctypes.c_float), ("b", ctypes.c_float), ("c", ctypes.c_float)]


class Schedule(ctypes.Structure):
    _fields_ = [("n_steps", ctypes.c_int), ("coeffs", ctypes.POINTER(NsCoeff)),
                ("eps", ctypes.c_float), ("restarts", ctypes.POINTER(ctypes.c_int)),
                ("n_restarts", ctypes.c_int), ("scale_f", ctypes.c_float), ("gram_aspect", ctypes.c_float)]


class HParams(ctypes.Structure):
    _fields_ = [("mu", ctypes.c_float), ("eta", ctypes.c_float), ("lambda_", ctypes.c_float),
                ("gamma", ctypes.c_float), ("beta_a", ctypes.c_float), ("alpha", ctypes.c_float)]


class Param(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int), ("cols", ctypes.c_int), ("W", ctypes.c_void_p),
                ("G", ctypes.c_void_p), ("G_prev", ctypes.c_void_p), ("A", ctypes.c_void_p),
                ("M", ctypes.c_void_p), ("gamma", ctypes.c_float), ("O_out", ctypes.c_void_p)]


class LiteParam(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int), ("cols", ctypes.c_int), ("W", ctypes.c_void_p),
                ("G", ctypes.c_void_p), ("B", ctypes.c_void_p), ("M", ctypes.c_void_p),
                ("gamma", ctypes.c_float), ("O_out", ctypes.c_void_p)]


class VecParam(ctypes.Structure):
    _fields_ = [("n", ctypes.c_longlong), ("W", ctypes.c_void_p), ("G", ctypes.c_void_p),
                ("m", ctypes.c_void_p), ("v", ctypes.c_void_p)]


class RsvdParam(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int), ("cols", ctypes.c_int), ("W", ctypes.c_void_p),
                ("G", ctypes.c_void_p), ("M", ctypes.c_void_p), ("Omega", ctypes.c_void_p),
                ("gamma", ctypes.c_float), ("O_out", ctypes.c_void_p)]


class RsvdHParams(ctypes.Structure):
    _fields_ = [("mu", ctypes.c_float), ("eta", ctypes.c_float), ("lambda_", ctypes.c_float),
                ("gamma", ctypes.c_float), ("rank", ctypes.c_int), ("oversample", ctypes.c_int)]


class AdamWHParams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float)]


(KERNEL_PREPASS, KERNEL_SYM, KERNEL_UPD, KERNEL_SIMT, KERNEL_OTHER, KERNEL_ADAMW, KERNEL_RSVD,
 KERNEL_RSVD_SMALL) = range(8)
KERNEL_NAMES = {KERNEL_PREPASS: "prepass", KERNEL_SYM: "tc_sym", KERNEL_UPD: "tc_upd", KERNEL_ADAMW: "adamw",
                KERNEL_SIMT: "simt", KERNEL_OTHER: "other", KERNEL_RSVD: "rsvd", KERNEL_RSVD_SMALL: "rsvd_small"}
TRACE_CAPACITY = 8192


class TraceRecord(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("work", ctypes.c_double), ("ms", ctypes.c_float)]


_lib = None


def lib():
    """Load libmuon_b200.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m muon_family_optimizer_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        st = ctypes.c_int
        vp = ctypes.c_void_p
        sz = ctypes.POINTER(ctypes.c_size_t)
        L.muon_status_string.restype = ctypes.c_char_p
        L.muon_status_string.argtypes = [st]
        L.muon_workspace_size.restype = st
        L.muon_workspace_size.argtypes = [ctypes.POINTER(Param), ctypes.c_int, ctypes.c_int,
                                          ctypes.POINTER(Schedule), sz]
        L.muon_step_batched.restype = st
        L.muon_step_batched.argtypes = [ctypes.POINTER(Param), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.POINTER(HParams), ctypes.POINTER(Schedule), vp,
                                        ctypes.c_size_t, vp, vp]
        L.muon_lite_workspace_size.restype = st
        L.muon_lite_workspace_size.argtypes = [ctypes.POINTER(LiteParam), ctypes.c_int, ctypes.c_int,
                                               ctypes.POINTER(Schedule), sz]
        L.muon_lite_step_batched.restype = st
        L.muon_lite_step_batched.argtypes = [ctypes.POINTER(LiteParam), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.POINTER(HParams), ctypes.POINTER(Schedule), vp,
                                             ctypes.c_size_t, vp, vp]
        L.limuon_workspace_size.restype = st
        L.limuon_workspace_size.argtypes = [ctypes.POINTER(RsvdParam), ctypes.c_int, ctypes.POINTER(RsvdHParams), sz]
        L.limuon_step_batched.restype = st
        L.limuon_step_batched.argtypes = [ctypes.POINTER(RsvdParam), ctypes.c_int, ctypes.c_int,
                                          ctypes.POINTER(RsvdHParams), vp, ctypes.c_size_t, vp, vp]
        L.muon_wait_selftest.restype = st
        L.muon_wait_selftest.argtypes = [ctypes.c_int, vp, vp]
        L.muon_model_step.restype = st
        L.muon_model_step.argtypes = [ctypes.POINTER(Param), ctypes.c_int, ctypes.POINTER(VecParam), ctypes.c_int,
                                      ctypes.c_int, ctypes.c_int, ctypes.POINTER(HParams),
                                      ctypes.POINTER(AdamWHParams), ctypes.c_int, ctypes.POINTER(Schedule), vp,
                                      ctypes.c_size_t, vp, vp]
        L.adamw_step_batched.restype = st
        L.adamw_step_batched.argtypes = [ctypes.POINTER(VecParam), ctypes.c_int, ctypes.c_int,
                                         ctypes.POINTER(AdamWHParams), ctypes.c_int, vp, vp]
        for name in ("ns_polar_workspace_size", "gram_polar_workspace_size"):
            f = getattr(L, name)
            f.restype = st
            f.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, sz]
        for name in ("ns_polar", "gram_polar"):
            f = getattr(L, name)
            f.restype = st
            f.argtypes = [vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_longlong,
                          ctypes.c_int, ctypes.POINTER(Schedule), vp, ctypes.c_size_t, vp, vp]
        L.ns_polar_noalloc.restype = st
        L.ns_polar_noalloc.argtypes = [vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_longlong,
                                       ctypes.c_int, ctypes.POINTER(Schedule), vp, vp]
        L.ns_polar_noalloc_capacity.restype = ctypes.c_size_t
        L.ns_polar_noalloc_capacity.argtypes = []
        L.muon_trace_enable.restype = st
        L.muon_trace_enable.argtypes = [ctypes.c_int]
        L.muon_trace_read.restype = ctypes.c_int
        L.muon_trace_read.argtypes = [ctypes.POINTER(TraceRecord), ctypes.c_int]
        _lib = L
    return _lib


def muon_status_string(status):
    return lib().muon_status_string(int(status)).decode()


def _check(status, where):
    if status != OK:
        raise MuonError(status, where)


def make_schedule(coeffs, eps=1e-7, restarts=(), scale_f=1.0, gram_aspect=0.0):
    """Build a C schedule; the returned object keeps its arrays alive.
    gram_aspect > 0: in an optimizer step, shape groups with long side >=
    gram_aspect * short side run the Gram route (restarts, scale_f)."""
    coeffs = [tuple(c) for c in coeffs]
    arr = (NsCoeff * len(coeffs))(*[NsCoeff(*c) for c in coeffs])
    rs = list(restarts)
    rarr = (ctypes.c_int * max(1, len(rs)))(*rs) if rs else None
    s = Schedule(len(coeffs), arr, eps, rarr, len(rs), scale_f, gram_aspect)
    s._keep = (arr, rarr)
    return s


def quintic_schedule(n_steps=5, eps=1e-7, scale_f=1.0):
    return make_schedule([QUINTIC] * n_steps, eps=eps, scale_f=scale_f)


# Restart of the Gram route inside the 5-step quintic optimizer step: before
# step 3.  Without a restart, 16-bit rounding leaves small negative eigenvalues
# in R that the quintic h(R) R h(R) multiplies by about 12 each step until they
# dominate; one restart recomputes R from Xb and keeps the result as close to
# the exact iteration as the direct route's (emulated and measured).
GRAM_STEP_RESTARTS = (3,)


def quintic_gram_schedule(n_steps=5, gram_aspect=2.0, eps=1e-7, restarts=GRAM_STEP_RESTARTS):
    """The quintic step schedule with the Gram route on shape groups whose long
    side is at least gram_aspect times the short side."""
    return make_schedule([QUINTIC] * n_steps, eps=eps, restarts=restarts, scale_f=1.0, gram_aspect=gram_aspect)


def _dtype_code(t):
    import torch
    return {torch.bfloat16: BF16, torch.float16: FP16, torch.float32: FP32}[t]


def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def make_params(params):
    """params: list of dicts with torch tensors W, G, G_prev, A, M (+ optional gamma, O_out)."""
    arr = (Param * len(params))()
    for i, p in enumerate(params):
        W = p["W"]
        rows, cols = W.shape
        for k in ("W", "G", "G_prev", "A", "M"):
            t = p[k]
            if tuple(t.shape) != (rows, cols) or not t.is_contiguous():
                raise ValueError(f"param {i}: {k} must be a contiguous {rows}x{cols} tensor")
        arr[i] = Param(rows, cols, W.data_ptr(), p["G"].data_ptr(), p["G_prev"].data_ptr(),
                       p["A"].data_ptr(), p["M"].data_ptr(), float(p.get("gamma", math.nan)),
                       p["O_out"].data_ptr() if p.get("O_out") is not None else None)
    return arr


def muon_workspace_size(params, ns_dtype, schedule=None):
    """Workspace bytes of muon_step_batched; schedule None sizes the direct route."""
    arr = params if isinstance(params, ctypes.Array) else make_params(params)
    out = ctypes.c_size_t(0)
    _check(lib().muon_workspace_size(arr, len(arr), int(ns_dtype), ctypes.byref(schedule) if schedule else None,
                                     ctypes.byref(out)), "muon_workspace_size")
    return out.value


def muon_step_batched(params, w_dtype, ns_dtype, hp, schedule, workspace, d_status=None, stream=None):
    """One MONA/Muon step on every parameter (see include/muon.h).

    params: list of dicts (see make_params) or a ctypes Param array.
    hp: dict with mu, eta, lambda, gamma, beta_a, alpha.  schedule: make_schedule(...).
    workspace: a CUDA uint8 tensor of at least muon_workspace_size(...) bytes.
    """
    arr = params if isinstance(params, ctypes.Array) else make_params(params)
    h = HParams(hp["mu"], hp["eta"], hp["lambda"], hp["gamma"], hp["beta_a"], hp["alpha"])
    _check(lib().muon_step_batched(arr, len(arr), int(w_dtype), int(ns_dtype), ctypes.byref(h),
                                   ctypes.byref(schedule), _ptr(workspace), workspace.numel(),
                                   _ptr(d_status), _stream_ptr(stream)), "muon_step_batched")


def muon_model_step(params, vecs, w_dtype, ns_dtype, hp, adamw_hp, step, schedule, workspace, d_status=None,
                    stream=None):
    """One step of a whole model (see include/muon.h): the matrices as
    muon_step_batched, the vector-valued parameters with AdamW as items of the
    same pre-pass launch.  vecs: list of dicts (see make_vec_params), a ctypes
    VecParam array, or None; adamw_hp: dict with lr, beta1, beta2, eps,
    weight_decay; step: t >= 1."""
    arr = params if isinstance(params, ctypes.Array) else make_params(params)
    varr = None
    if vecs is not None and len(vecs):
        varr = vecs if isinstance(vecs, ctypes.Array) else make_vec_params(vecs)
    h = HParams(hp["mu"], hp["eta"], hp["lambda"], hp["gamma"], hp["beta_a"], hp["alpha"])
    a = AdamWHParams(adamw_hp["lr"], adamw_hp["beta1"], adamw_hp["beta2"], adamw_hp["eps"],
                     adamw_hp["weight_decay"]) if adamw_hp else None
    _check(lib().muon_model_step(arr, len(arr), varr, len(varr) if varr is not None else 0, int(w_dtype),
                                 int(ns_dtype), ctypes.byref(h), ctypes.byref(a) if a else None, int(step),
                                 ctypes.byref(schedule), _ptr(workspace), workspace.numel(), _ptr(d_status),
                                 _stream_ptr(stream)), "muon_model_step")


def make_lite_params(params):
    """params: list of dicts with torch tensors W, G, B (bfloat16), M (+ optional gamma, O_out)."""
    import torch
    arr = (LiteParam * len(params))()
    for i, p in enumerate(params):
        W = p["W"]
        rows, cols = W.shape
        for k in ("W", "G", "B", "M"):
            t = p[k]
            if tuple(t.shape) != (rows, cols) or not t.is_contiguous():
                raise ValueError(f"param {i}: {k} must be a contiguous {rows}x{cols} tensor")
        if p["B"].dtype != torch.bfloat16 or p["M"].dtype != torch.float32:
            raise ValueError(f"param {i}: B must be bfloat16 and M float32")
        arr[i] = LiteParam(rows, cols, W.data_ptr(), p["G"].data_ptr(), p["B"].data_ptr(), p["M"].data_ptr(),
                           float(p.get("gamma", math.nan)),
                           p["O_out"].data_ptr() if p.get("O_out") is not None else None)
    return arr


def muon_lite_workspace_size(params, ns_dtype, schedule=None):
    arr = params if isinstance(params, ctypes.Array) else make_lite_params(params)
    out = ctypes.c_size_t(0)
    _check(lib().muon_lite_workspace_size(arr, len(arr), int(ns_dtype),
                                          ctypes.byref(schedule) if schedule else None, ctypes.byref(out)),
           "muon_lite_workspace_size")
    return out.value


def muon_lite_step_batched(params, w_dtype, ns_dtype, hp, schedule, workspace, d_status=None, stream=None):
    """One MONA-Lite step on every parameter (see include/muon.h): B (bfloat16)
    replaces G_prev and A."""
    arr = params if isinstance(params, ctypes.Array) else make_lite_params(params)
    h = HParams(hp["mu"], hp["eta"], hp["lambda"], hp["gamma"], hp["beta_a"], hp["alpha"])
    _check(lib().muon_lite_step_batched(arr, len(arr), int(w_dtype), int(ns_dtype), ctypes.byref(h),
                                        ctypes.byref(schedule), _ptr(workspace), workspace.numel(),
                                        _ptr(d_status), _stream_ptr(stream)), "muon_lite_step_batched")


def make_vec_params(params):
    """params: list of dicts with torch tensors W, G (same dtype), m, v (float32), any shape, contiguous."""
    import torch
    arr = (VecParam * len(params))()
    for i, p in enumerate(params):
        n = p["W"].numel()
        for k in ("W", "G", "m", "v"):
            if p[k].numel() != n or not p[k].is_contiguous():
                raise ValueError(f"vector param {i}: {k} must be contiguous with {n} elements")
        if p["m"].dtype != torch.float32 or p["v"].dtype != torch.float32 or p["G"].dtype != p["W"].dtype:
            raise ValueError(f"vector param {i}: m and v must be float32 and G of W's dtype")
        arr[i] = VecParam(n, p["W"].data_ptr(), p["G"].data_ptr(), p["m"].data_ptr(), p["v"].data_ptr())
    return arr


def adamw_step_batched(params, w_dtype, hp, step, d_status=None, stream=None):
    """One AdamW step (see include/muon.h) on vector parameters.
    hp: dict with lr, beta1, beta2, eps, weight_decay; step: t >= 1."""
    arr = params if isinstance(params, ctypes.Array) else make_vec_params(params)
    h = AdamWHParams(hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"])
    _check(lib().adamw_step_batched(arr, len(arr), int(w_dtype), ctypes.byref(h), int(step), _ptr(d_status),
                                    _stream_ptr(stream)), "adamw_step_batched")


def make_rsvd_params(params):
    """params: list of dicts with torch tensors W, G (same dtype), M (float32), Omega (float32,
    cols x k), optional O_out (float32) and gamma (float); rows x cols, contiguous."""
    import torch
    arr = (RsvdParam * len(params))()
    for i, p in enumerate(params):
        W = p["W"]
        if W.dim() != 2:
            raise ValueError(f"param {i}: W must be 2-D")
        rows, cols = W.shape
        for k in ("W", "G", "M", "Omega") + (("O_out",) if p.get("O_out") is not None else ()):
            if not p[k].is_contiguous():
                raise ValueError(f"param {i}: {k} must be contiguous")
        if p["G"].shape != W.shape or p["M"].shape != W.shape or p["G"].dtype != W.dtype:
            raise ValueError(f"param {i}: G must match W; M must be rows x cols")
        if p["M"].dtype != torch.float32 or p["Omega"].dtype != torch.float32 or p["Omega"].dim() != 2 \
                or p["Omega"].shape[0] != cols:
            raise ValueError(f"param {i}: M must be float32 and Omega float32 cols x k")
        O = p.get("O_out")
        if O is not None and (O.shape != W.shape or O.dtype != torch.float32):
            raise ValueError(f"param {i}: O_out must be float32 rows x cols")
        arr[i] = RsvdParam(rows, cols, W.data_ptr(), p["G"].data_ptr(), p["M"].data_ptr(), p["Omega"].data_ptr(),
                           float(p.get("gamma", float("nan"))), O.data_ptr() if O is not None else None)
    return arr


def _rsvd_hp(hp):
    return RsvdHParams(hp["mu"], hp["eta"], hp["lambda"], hp["gamma"], int(hp["rank"]), int(hp["oversample"]))


def limuon_workspace_size(params, hp):
    arr = params if isinstance(params, ctypes.Array) else make_rsvd_params(params)
    out = ctypes.c_size_t(0)
    h = _rsvd_hp(hp)
    _check(lib().limuon_workspace_size(arr, len(arr), ctypes.byref(h), ctypes.byref(out)), "limuon_workspace_size")
    return out.value


def limuon_step_batched(params, w_dtype, hp, workspace, d_status=None, stream=None):
    """One LiMuon step (see include/muon.h).  hp: dict with mu, eta, lambda, gamma, rank,
    oversample; every Omega has rank + oversample columns."""
    arr = params if isinstance(params, ctypes.Array) else make_rsvd_params(params)
    h = _rsvd_hp(hp)
    _check(lib().limuon_step_batched(arr, len(arr), int(w_dtype), ctypes.byref(h), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _ptr(d_status),
                                     _stream_ptr(stream)), "limuon_step_batched")


def muon_wait_selftest(wait_ms, d_status, stream=None):
    """Run the bounded-wait self-test (see include/muon.h): sets FLAG_TIMEOUT in d_status."""
    _check(lib().muon_wait_selftest(int(wait_ms), _ptr(d_status), _stream_ptr(stream)), "muon_wait_selftest")


def ns_polar_workspace_size(batch, rows, cols, dtype):
    out = ctypes.c_size_t(0)
    _check(lib().ns_polar_workspace_size(batch, rows, cols, int(dtype), ctypes.byref(out)),
           "ns_polar_workspace_size")
    return out.value


def gram_polar_workspace_size(batch, rows, cols, dtype):
    out = ctypes.c_size_t(0)
    _check(lib().gram_polar_workspace_size(batch, rows, cols, int(dtype), ctypes.byref(out)),
           "gram_polar_workspace_size")
    return out.value


def _polar(fn, X_in, X_out, schedule, workspace, d_status, stream):
    if X_in.dim() == 2:
        batch, (rows, cols) = 1, X_in.shape
    else:
        batch, rows, cols = X_in.shape
    if not X_in.is_contiguous() or not X_out.is_contiguous() or X_out.shape != X_in.shape \
            or X_out.dtype != X_in.dtype:
        raise ValueError("X_in / X_out must be contiguous tensors of the same shape and dtype")
    _check(fn(_ptr(X_in), _ptr(X_out), batch, rows, cols, rows * cols, _dtype_code(X_in.dtype),
              ctypes.byref(schedule), _ptr(workspace), workspace.numel(), _ptr(d_status),
              _stream_ptr(stream)), fn.__name__)


def ns_polar_noalloc(X_in, X_out, schedule, d_status=None, stream=None):
    """ns_polar on the library's fixed device scratch, for callers that cannot
    allocate a workspace (e.g. during CUDA graph capture).  The first call on a
    device should come before any capture; calls on one device must not overlap."""
    if X_in.dim() == 2:
        batch, (rows, cols) = 1, X_in.shape
    else:
        batch, rows, cols = X_in.shape
    if not X_in.is_contiguous() or not X_out.is_contiguous() or X_out.shape != X_in.shape \
            or X_out.dtype != X_in.dtype:
        raise ValueError("X_in / X_out must be contiguous tensors of the same shape and dtype")
    _check(lib().ns_polar_noalloc(_ptr(X_in), _ptr(X_out), batch, rows, cols, rows * cols,
                                  _dtype_code(X_in.dtype), ctypes.byref(schedule), _ptr(d_status),
                                  _stream_ptr(stream)), "ns_polar_noalloc")


def ns_polar_noalloc_capacity():
    return lib().ns_polar_noalloc_capacity()


def ns_polar(X_in, X_out, schedule, workspace, d_status=None, stream=None):
    """Direct Newton-Schulz orthogonalisation of a (batch of) matrices."""
    _polar(lib().ns_polar, X_in, X_out, schedule, workspace, d_status, stream)


def gram_polar(X_in, X_out, schedule, workspace, d_status=None, stream=None):
    """The same iteration through the Gram matrix (restarts, divisor scale_f)."""
    _polar(lib().gram_polar, X_in, X_out, schedule, workspace, d_status, stream)


def converged_schedule(eps=1e-7):
    """8 quintic + 6 cubic steps, restarts before steps 3, 5 and 7, divisor 1.05.

    Converges to the polar factor for condition numbers up to about 1e3; the
    restarts keep the Gram route stable in 16-bit arithmetic."""
    return make_schedule([QUINTIC] * 8 + [CUBIC] * 6, eps=eps, restarts=(3, 5, 7), scale_f=1.05)


def muon_trace_enable(enable=True):
    _check(lib().muon_trace_enable(1 if enable else 0), "muon_trace_enable")


def muon_trace_read():
    """List of (kind, work, ms) for the launches recorded since the last read."""
    buf = (TraceRecord * TRACE_CAPACITY)()
    n = lib().muon_trace_read(buf, TRACE_CAPACITY)
    if n < 0:
        raise MuonError(ERR_CUDA, "muon_trace_read")
    return [(buf[i].kind, buf[i].work, buf[i].ms) for i in range(n)]
