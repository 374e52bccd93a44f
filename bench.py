#!/usr/bin/env python
"""Benchmark of one MONA / Muon optimizer step on B200 (one JSON line).

A step is one call of muon_step_batched over every matrix of the workload:
the fused MONA pre-pass with the Frobenius norms, 5 quintic Newton-Schulz
steps on tensor cores (grouped by shape), and the weight update fused into
the last step.  Inputs are synthetic (seeded; shapes of the named model).
The default workload is the largest configuration that fits one GPU: the
Llama-3-8B layer set (224 matrices, 6.98 G elements).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

value = Newton-Schulz TFLOP/s over all ranks (algorithmic flops: symmetric
products count the half they need), timed with CUDA events on the step's
stream between barriers, max over ranks.  Under torchrun the matrices are
partitioned across the ranks (flop-balanced, whole matrices) and every step
ends with one all-gather of the updated weights (strong scaling: the model's
step is shared); --replicas makes each rank step its own copy instead.
--impl reference times the fp64 CPU oracle on a bounded sample instead.
"""
import argparse
import ctypes
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Muon step ms & Newton-Schulz TFLOP/s on 1 B200; % of bf16 tensor / HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama3_8b")
    ap.add_argument("--layers", type=int, default=0,
                    help="take only the first N layers of a layered workload (smaller cases for profiling)")
    ap.add_argument("--step-route", default="direct", choices=["direct", "gram"],
                    help="route of the headline step: the direct quintic iteration (default) or the Gram route on "
                         "shape groups with long side >= --gram-aspect x short side (one restart before step 3)")
    ap.add_argument("--gram-aspect", type=float, default=2.0)
    ap.add_argument("--no-route-compare", action="store_true",
                    help="skip timing the other route of the step (single GPU only)")
    ap.add_argument("--replicas", action="store_true",
                    help="under torchrun: every rank steps its own copy of the workload (weak scaling) "
                         "instead of its share of one model (strong scaling, the default)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ns-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--launch", default="graph", choices=["graph", "eager"],
                    help="replay each step as a captured CUDA graph (default) or launch it eagerly")
    ap.add_argument("--variant", default="mona", choices=["mona", "lite"],
                    help="mona: G_prev and A state (default); lite: MONA-Lite, one bfloat16 buffer B")
    ap.add_argument("--route", default="step", choices=["step", "gram", "direct", "adamw", "limuon", "model"],
                    help="step: the optimizer step (default); gram / direct: the orthogonalisation alone "
                         "(gram_polar / ns_polar, converged schedule) of the workload's matrices, one batch per shape; "
                         "adamw: the AdamW step of the model's vector-valued parameters; "
                         "limuon: the LiMuon step (randomized SVD, r = 16, p = 16) of the workload's matrices; "
                         "model: muon_model_step (matrices plus the vector-valued parameters' AdamW in one pre-pass "
                         "launch) against the two separate calls")
    return ap.parse_args()


def peaks(path=None):
    """Roofline denominators: the measured figures of MEASURED_PEAKS.json where it has them
    (positive numbers under the keys of FALLBACK_PEAKS), the fallback figures otherwise."""
    p = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    out = dict(FALLBACK_PEAKS)
    if not os.path.exists(p):
        return out, "fallback"
    try:
        with open(p) as fh:
            d = json.load(fh)
    except (OSError, ValueError):
        return out, "fallback (MEASURED_PEAKS.json unreadable)"
    found = []
    for k in FALLBACK_PEAKS:
        v = d.get(k) if isinstance(d, dict) else None
        if isinstance(v, (int, float)) and not isinstance(v, bool) and v > 0:
            out[k] = float(v)
            found.append(k)
    if not found:
        return out, "fallback (MEASURED_PEAKS.json has none of the peaks)"
    if len(found) < len(FALLBACK_PEAKS):
        return out, "measured (" + ", ".join(found) + "; fallback for the rest)"
    return out, "measured"


# Sources whose change invalidates a recorded DRAM-traffic figure, per kernel.
_COMMON = ("muon_family_optimizer_b200/csrc/muon_internal.cuh", "muon_family_optimizer_b200/csrc/gemm.h",
           "muon_family_optimizer_b200/csrc/muon_api.cu")
TRAFFIC_SOURCES = {
    "tc_sym": _COMMON + ("muon_family_optimizer_b200/csrc/gemm_tc.cu", "muon_family_optimizer_b200/csrc/epilogue.cuh"),
    "tc_upd": _COMMON + ("muon_family_optimizer_b200/csrc/gemm_tc.cu", "muon_family_optimizer_b200/csrc/epilogue.cuh"),
    "prepass": _COMMON + ("muon_family_optimizer_b200/csrc/prepass.cu",),
}


def sources_digest(kernel="tc_sym"):
    import hashlib
    h = hashlib.sha256()
    for rel in TRAFFIC_SOURCES.get(kernel, TRAFFIC_SOURCES["tc_sym"]):
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload, ns_steps, elements=None):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of
    ``kernel`` from the ncu summaries under profiles/: a line
    ``traffic-record: {json}`` written when the counters were taken.  A record
    taken on a leading slice of the workload's layers (its "elements" below the
    launch's) is scaled to the launch by elements: every matrix of a shape
    group is processed alike, so the traffic grows in proportion.  None when
    no record matches the workload or the kernel sources changed since."""
    d = os.path.join(ROOT, "profiles")
    if not os.path.isdir(d):
        return None, None
    digest = sources_digest(kernel)
    for name in sorted(os.listdir(d)):
        if not name.endswith(".md"):
            continue
        with open(os.path.join(d, name)) as fh:
            for line in fh:
                if not line.startswith("traffic-record:"):
                    continue
                try:
                    rec = json.loads(line.split(":", 1)[1])
                except ValueError:
                    continue
                if (rec.get("kernel") == kernel and rec.get("workload") == workload
                        and rec.get("ns_steps") == ns_steps and rec.get("sources") == digest):
                    b = float(rec["bytes_per_launch"])
                    rec_el = rec.get("elements")
                    if rec_el and elements and rec_el != elements:
                        return b * elements / rec_el, f"profiles/{name} (scaled by elements from {rec_el})"
                    return b, f"profiles/{name}"
    return None, None


def ns_flops(shapes, ns_steps):
    """Algorithmic flops of the iteration: per step s^2 l (X X^T, half) + s^3 (A A, half) + 2 s^2 l (B X)."""
    tot = 0.0
    for r, c in shapes:
        s, l = min(r, c), max(r, c)
        tot += ns_steps * (3.0 * s * s * l + float(s) ** 3)
    return tot


def ns_flops_dense(shapes, ns_steps):
    """Dense-equivalent flops: both symmetric products counted in full, 4 s^2 l + 2 s^3 per step."""
    tot = 0.0
    for r, c in shapes:
        s, l = min(r, c), max(r, c)
        tot += ns_steps * (4.0 * s * s * l + 2.0 * float(s) ** 3)
    return tot


def describe(name, w):
    from collections import Counter
    cnt = Counter((min(r, c), max(r, c)) for r, c in w["shapes"])
    groups = " + ".join(f"{n} x {s}x{l}" for (s, l), n in sorted(cnt.items()))
    nel = sum(r * c for r, c in w["shapes"])
    return groups, nel


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.index)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle (baseline and reference arm)

def oracle_sample_run(w, picks, seed_base=0):
    """One full MONA/Muon step in fp64 on the matrices `picks` ((j, rows, cols),
    j = the matrix's index in the workload); returns seconds."""
    import numpy as np
    import oracle
    from muon_family_optimizer_b200 import synthetic as syn
    arrays = []
    for j, r, c in picks:
        W = syn.initial_weight(w["name"], j, r, c).double().numpy()
        G = syn.gradient(w["name"], j, seed_base, r, c).double().numpy()
        Gp = syn.gradient(w["name"], j, seed_base + 8, r, c).double().numpy()
        arrays.append((W, G, Gp, np.zeros_like(W), np.zeros_like(W)))
    hp = w["hp"]
    t0 = time.perf_counter()
    for W, G, Gp, A, M in arrays:
        oracle.muon_step(W, G, Gp, A, M, mu=hp["mu"], eta=hp["eta"], lam=hp["lambda"], gamma=hp["gamma"],
                         beta_a=hp["beta_a"], alpha=hp["alpha"], coeffs=[tuple(syn.QUINTIC)] * 5)
    return time.perf_counter() - t0


def shape_groups(shapes):
    """Matrices of each (short side, long side) group: [(cost, [(j, rows, cols), ...])],
    cheapest group first (cost = one matrix's algorithmic NS flops)."""
    groups = {}
    for j, (r, c) in enumerate(shapes):
        groups.setdefault((min(r, c), max(r, c)), []).append((j, r, c))
    out = [(ns_flops([(m[0][1], m[0][2])], 5), m) for m in groups.values()]
    return sorted(out, key=lambda x: x[0])


# fp64 oracle work per matrix beyond which it is left out of the bench's CPU legs
# (a 4096 x 4096 matrix is 1.4 TFLOP: about half a minute on 16 host cores)
ORACLE_MATRIX_FLOPS = 2.5e11


def cpu_baseline(w, ns_steps, budget_s=25.0, floor_s=10.0):
    """The fp64 oracle's rate on a bounded sample of the workload: one matrix of
    each shape group, cheapest first, while the predicted time stays within
    budget_s, then further matrices of the cheapest group until floor_s."""
    import oracle
    groups = shape_groups(w["shapes"])
    picks, secs, fl = [], 0.0, 0.0
    for cost, members in groups:
        if picks and (cost > ORACLE_MATRIX_FLOPS or secs + cost * secs / fl > budget_s):
            break
        secs += oracle_sample_run(w, [members[0]])
        fl += ns_flops([members[0][1:]], ns_steps)
        picks.append(members[0])
    more = iter(groups[0][1][1:])
    for m in more:
        if secs >= floor_s:
            break
        secs += oracle_sample_run(w, [m])
        fl += ns_flops([m[1:]], ns_steps)
        picks.append(m)
    full = ns_flops(w["shapes"], ns_steps)
    from collections import Counter
    desc = ", ".join(f"{n} x {r}x{c}" for (r, c), n in Counter((r, c) for _, r, c in picks).items())
    return {"value": fl / secs / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{len(picks)} matrices of the workload ({desc}): full fp64 MONA step with {ns_steps} "
                      f"quintic steps each, {secs:.2f} s; rate = their algorithmic NS flops / time",
            "ms_per_step_extrapolated": secs * full / fl * 1e3}


def group_parity(w, ns_steps, dev):
    """Maximum relative errors per shape group: one matrix of each (s, l) group,
    one step on the GPU through muon_step_batched (with O stored) and the same
    step in the fp64 oracle from the same 16-bit inputs (the iteration started
    from the same rounded momentum).  Groups whose oracle step would take more
    than a few seconds are listed as skipped (the full-size GPU tests check
    them).  Returns {"s x l": {"O": e, "W": e, "M": e}}."""
    import numpy as np
    import torch
    import muon_family_optimizer_b200 as mo
    import oracle
    from muon_family_optimizer_b200 import synthetic as syn
    w_dt, ns_dt = w["w_dtype"], w["ns_dtype"]
    pick, out = [], {}
    for cost, members in shape_groups(w["shapes"]):
        j, r, c = members[0]
        if cost > ORACLE_MATRIX_FLOPS:
            out[f"{min(r, c)}x{max(r, c)}"] = {"skipped": f"{cost / 1e12:.2f} TFLOP per matrix in fp64; "
                                                           "checked by the full-size GPU tests"}
        else:
            pick.append((j, r, c))
    host, params = [], []
    for j, r, c in pick:
        st = dict(W=syn.initial_weight(w["name"], j, r, c).to(w_dt), G=syn.gradient(w["name"], j, 0, r, c).to(w_dt),
                  G_prev=syn.gradient(w["name"], j, 8, r, c).to(w_dt), A=torch.zeros(r, c), M=torch.zeros(r, c))
        host.append(st)
        p = {k: v.to(dev).contiguous() for k, v in st.items()}
        p["O_out"] = torch.empty(r, c, device=dev)
        params.append(p)
    if not params:
        return out
    ws = torch.empty(mo.muon_workspace_size(params, mo._dtype_code(ns_dt), None), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    mo.muon_step_batched(params, mo._dtype_code(w_dt), mo._dtype_code(ns_dt), w["hp"],
                         mo.quintic_schedule(ns_steps), ws, d_status=status)
    torch.cuda.synchronize(dev)
    rnd = {torch.bfloat16: oracle.ROUND_BF16, torch.float16: oracle.ROUND_FP16}.get(ns_dt, oracle.ROUND_NONE)
    hp = w["hp"]
    rel = lambda a, b: float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
    for (j, r, c), st, p in zip(pick, host, params):
        f = {k: v.double().numpy() for k, v in st.items()}
        ref = oracle.muon_step(f["W"], f["G"], f["G_prev"], f["A"], f["M"], mu=hp["mu"], eta=hp["eta"],
                               lam=hp["lambda"], gamma=hp["gamma"], beta_a=hp["beta_a"], alpha=hp["alpha"],
                               coeffs=[tuple(syn.QUINTIC)] * ns_steps, round_to=rnd)
        g = {k: p[k].double().cpu().numpy() for k in ("W", "M", "O_out")}
        out[f"{min(r, c)}x{max(r, c)}"] = {"O": rel(g["O_out"], ref["O"]), "W": rel(g["W"], ref["W"]),
                                          "M": rel(g["M"], ref["M"]), "status": int(status.item())}
    return out


def run_reference(args, w, ns_steps):
    """The reference arm: the fp64 oracle on the host cores.  Each timed step is
    one full MONA step of one matrix of the workload (the shape groups whose
    oracle step takes at most a few seconds, in turn), so K steps finish within
    minutes; value = algorithmic NS flops / time, ms_per_step = the timed
    sample step, the whole-workload time extrapolated by flops."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    groups = [members for cost, members in shape_groups(w["shapes"]) if cost <= ORACLE_MATRIX_FLOPS]
    if not groups:
        groups = [shape_groups(w["shapes"])[0][1]]
    # step i takes group i % len(groups), cycling through that group's matrices
    order = [groups[i % len(groups)][(i // len(groups)) % len(groups[i % len(groups)])]
             for i in range(args.warmup + args.steps)]
    for i in range(args.warmup):
        oracle_sample_run(w, [order[i]], seed_base=i)
    fl = secs = 0.0
    steps = 0
    for i in range(args.steps):
        m = order[args.warmup + i]
        secs += oracle_sample_run(w, [m], seed_base=i)
        fl += ns_flops([m[1:]], ns_steps)
        steps += 1
    value = fl / secs / 1e12
    full = ns_flops(w["shapes"], ns_steps)
    groups_desc, nel = describe(args.workload, w)
    from collections import Counter
    used = ", ".join(f"{r}x{c}" for (r, c) in Counter((m[1], m[2]) for m in order[args.warmup:]))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": args.warmup, "ms_per_step": secs / steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{w['name']}: {groups_desc}", "elements": nel, "ns_steps": ns_steps},
            "ms_per_step_extrapolated": secs / fl * full * 1e3,
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"{steps} timed steps, each one full fp64 MONA step of one matrix of the "
                                       f"workload ({used}); ms_per_step is that sample step, "
                                       "ms_per_step_extrapolated the whole workload by flops"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm

def run_adamw_route(args, w):
    """Time adamw_step_batched on the model family's vector-valued parameters
    (bf16 W and G, fp32 moments): a streaming pass, 22 bytes per element."""
    import torch
    import muon_family_optimizer_b200 as mo
    from muon_family_optimizer_b200 import synthetic as syn
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    shapes = syn.VECTOR_SHAPES[w["name"]]
    g = torch.Generator(device=dev).manual_seed(77)
    params = []
    for sh in shapes:
        params.append(dict(W=(torch.randn(sh, generator=g, device=dev) * 0.02).to(torch.bfloat16),
                           G=torch.randn(sh, generator=g, device=dev).to(torch.bfloat16),
                           m=torch.zeros(sh, device=dev), v=torch.zeros(sh, device=dev)))
    arr = mo.make_vec_params(params)
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.1)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    nel = sum(p["W"].numel() for p in params)
    for t in range(1, args.warmup + 1):
        mo.adamw_step_batched(arr, mo.BF16, hp, t, d_status=status)
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    with torch.cuda.graph(graph, stream=cap):
        mo.adamw_step_batched(arr, mo.BF16, hp, args.warmup + 1, d_status=status,
                              stream=torch.cuda.current_stream(dev))
    for _ in range(3):
        graph.replay()
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1) / args.steps
    gbs = nel * 22.0 / (ms / 1e3) / 1e9
    pk, src = peaks()
    line = {"metric": "AdamW step of the vector-valued parameters, GB/s", "value": gbs, "unit": "GB/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16 W/G, fp32 moments", "data": "synthetic",
            "config": {"workload": f"{w['name']} vector parameters: {len(shapes)} tensors, {nel} elements",
                       "bytes_per_element": 22, "l2": f"inputs larger than L2: {nel * 22 / 1e9:.2f} GB per step"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": None, "peak_source": f"{src} (copy)"},
            "gpu_launches": args.steps, "clocks": clk, "launch": "graph (one CUDA graph per step)"}
    print(json.dumps(line), flush=True)
    del graph


def run_model_route(args, w):
    """Time muon_model_step (the matrices' MONA step with the vector-valued
    parameters' AdamW as items of its pre-pass launch) against
    muon_step_batched followed by adamw_step_batched on the same state."""
    import torch
    import muon_family_optimizer_b200 as mo
    from muon_family_optimizer_b200 import synthetic as syn
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    if w["name"] not in syn.VECTOR_SHAPES:
        raise SystemExit(f"--route model: no vector-valued parameters for {w['name']}")
    shapes = w["shapes"]
    mats = []
    for j, (r, c) in enumerate(shapes):
        G = syn.gradient(w["name"], j, 0, r, c, device=dev)
        mats.append(dict(W=syn.initial_weight(w["name"], j, r, c, device=dev).to(torch.bfloat16),
                         G=G.to(torch.bfloat16), G_prev=(G * 0.5).to(torch.bfloat16),
                         A=torch.zeros(r, c, device=dev), M=torch.zeros(r, c, device=dev)))
    g = torch.Generator(device=dev).manual_seed(77)
    vecs = []
    for sh in syn.VECTOR_SHAPES[w["name"]]:
        vecs.append(dict(W=(torch.randn(sh, generator=g, device=dev) * 0.02).to(torch.bfloat16),
                         G=torch.randn(sh, generator=g, device=dev).to(torch.bfloat16),
                         m=torch.zeros(sh, device=dev), v=torch.zeros(sh, device=dev)))
    arr, varr = mo.make_params(mats), mo.make_vec_params(vecs)
    sched = mo.quintic_schedule(args.ns_steps)
    ws = torch.empty(mo.muon_workspace_size(arr, mo.BF16, sched), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ahp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.1)
    fused = lambda st: mo.muon_model_step(arr, varr, mo.BF16, mo.BF16, w["hp"], ahp, 5, sched, ws,
                                          d_status=status, stream=st)

    def separate(st):
        mo.muon_step_batched(arr, mo.BF16, mo.BF16, w["hp"], sched, ws, d_status=status, stream=st)
        mo.adamw_step_batched(varr, mo.BF16, ahp, 5, d_status=status, stream=st)

    stream = torch.cuda.current_stream(dev)
    out = {}
    for name, fn in (("fused", fused), ("separate", separate)):
        for _ in range(args.warmup):
            fn(stream)
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        with torch.cuda.graph(graph, stream=cap):
            fn(torch.cuda.current_stream(dev))
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        out[name] = e0.elapsed_time(e1) / args.steps
        del graph
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())}")
    nvec = sum(v["W"].numel() for v in vecs)
    fl = ns_flops(shapes, args.ns_steps)
    line = {"metric": "Muon + AdamW model step time, ms", "value": out["fused"], "unit": "ms", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": out["fused"], "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{w['name']}: {len(shapes)} matrices + {len(vecs)} vector-valued parameters "
                                   f"({nvec} elements)", "ns_steps": args.ns_steps},
            "separate_calls_ms": out["separate"], "NS_TFLOP/s": fl / (out["fused"] / 1e3) / 1e12,
            "launch": "graph (one CUDA graph per step)"}
    print(json.dumps(line), flush=True)


# LiMuon: rank r, oversampling p (k = r + p columns of the test matrix)
LIMUON_HP = dict(mu=0.95, eta=0.02, gamma=1.0, rank=16, oversample=16, **{"lambda": 0.0})
# fp32 FMA peak: 148 SMs x 128 lanes x 2 flops at the 1965 MHz maximum SM clock
def tf32_tflops(pk):
    """Dense tf32 tensor peak: the bf16 peak times the nominal tf32 / bf16 ratio (1.1 / 2.25)."""
    return pk["bf16_tflops"] * 1.1 / 2.25


LIMUON_KERNELS = ["lim_sketch", "lim_chol", "lim_rowmul_q", "lim_project", "lim_eig", "lim_rowmul_z", "lim_update"]


def limuon_kernel_work(shapes, k, w_bytes=2):
    """Algorithmic bytes and fp32/fp64 flops per launch of the seven LiMuon
    kernels for matrices `shapes` (one launch each): per element, the sketch
    reads G and M and writes M (w_bytes + 8), the projection reads M (4), the
    update reads and writes W (2 w_bytes); each of these three products is k
    FMAs per element and moves its k-column factor (4 k bytes per row / column).
    The row transforms read and write the rows x KT factor (8 KT bytes per row,
    2 k^2 flops); the Cholesky and eigen steps move two KT x KT fp64 matrices
    per matrix."""
    kt = 32 if k <= 32 else 64
    el = sum(r * c for r, c in shapes)
    rows = sum(r for r, _ in shapes)
    rk = rows * k
    ck = sum(c for _, c in shapes) * k
    small = 2 * 8 * kt * kt * len(shapes)
    by = [el * (w_bytes + 8) + 4 * rk, small, 8 * rows * kt + small // 2, el * 4 + 4 * (rk + ck), small,
          8 * rows * kt + small // 2, el * 2 * w_bytes + 4 * (rk + ck)]
    fl = [2.0 * el * k, 0.0, 2.0 * rows * k * k, 2.0 * el * k, 0.0, 2.0 * rows * k * k, 2.0 * el * k]
    return by, fl


def run_limuon_route(args, w):
    """Time limuon_step_batched on the workload's matrices (bf16 W and G, fp32
    M, one Gaussian test matrix per distinct column count), with the first
    step of one matrix per shape group checked against the fp64 oracle."""
    import numpy as np
    import torch
    import muon_family_optimizer_b200 as mo
    from muon_family_optimizer_b200 import synthetic as syn
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    hp = LIMUON_HP
    k = hp["rank"] + hp["oversample"]
    shapes = [tuple(sh) for sh in w["shapes"]]
    omegas, params = {}, []
    for j, (r, c) in enumerate(shapes):
        if c not in omegas:
            omegas[c] = torch.randn(c, k, generator=torch.Generator(device=dev).manual_seed(c), device=dev)
        params.append(dict(W=syn.initial_weight(w["name"], j, r, c).to(torch.bfloat16).to(dev),
                           G=syn.gradient(w["name"], j, 0, r, c, device=dev).to(torch.bfloat16),
                           M=torch.zeros(r, c, device=dev), Omega=omegas[c]))
    # parity: the first step of one matrix per shape group, O stored
    pick = {}
    for j, sh in enumerate(shapes):
        pick.setdefault(sh, j)
    probe = [dict(W=params[j]["W"].clone(), G=params[j]["G"], M=torch.zeros_like(params[j]["M"]),
                  Omega=params[j]["Omega"], O_out=torch.empty_like(params[j]["M"])) for j in pick.values()]
    ws = torch.empty(mo.limuon_workspace_size(params, hp), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    mo.limuon_step_batched(probe, mo.BF16, hp, ws, d_status=status)
    torch.cuda.synchronize(dev)
    parity, cpu = {}, None
    if not args.no_cpu_baseline:
        # CPU-baseline leg: the fp64 oracle's LiMuon step on one matrix per shape group,
        # timed, and its O compared with the GPU's
        from oracle import limuon as lim
        secs, el_sample = 0.0, 0
        for ((r, c), j), p in zip(pick.items(), probe):
            W0 = params[j]["W"].double().cpu().numpy()       # not yet stepped
            G = p["G"].double().cpu().numpy()
            Om = p["Omega"].double().cpu().numpy()
            t0 = time.perf_counter()
            ref = lim.limuon_step(W0, G, np.zeros_like(G), Om, mu=hp["mu"],
                                  eta=hp["eta"], lam=hp["lambda"], gamma=hp["gamma"], rank=hp["rank"])
            secs += time.perf_counter() - t0
            el_sample += r * c
            O = lim.rsvd_orthogonal(p["M"].double().cpu().numpy(), Om, hp["rank"])
            Og = p["O_out"].double().cpu().numpy()
            parity[f"{r}x{c}"] = {"O": float(np.linalg.norm(Og - O) / max(np.linalg.norm(O), 1e-300)),
                                  "W": float(np.linalg.norm(p["W"].double().cpu().numpy() - ref["W"])
                                             / np.linalg.norm(ref["W"])),
                                  "status": int(status.item())}
        el_all = sum(r * c for r, c in shapes)
        cpu = {"value": secs * el_all / el_sample * 1e3, "unit": "ms", "cores": len(os.sched_getaffinity(0)),
               "kind": "oracle", "sample": f"one matrix per shape group ({', '.join(f'{r}x{c}' for r, c in pick)}): "
                                           f"fp64 LiMuon step (numpy QR and SVD), {secs:.2f} s, scaled to all "
                                           f"{len(shapes)} matrices by element count"}
    arr = mo.make_rsvd_params(params)
    for _ in range(args.warmup):
        mo.limuon_step_batched(arr, mo.BF16, hp, ws, d_status=status)
    torch.cuda.synchronize(dev)
    # per-kernel device times: one traced eager pass
    mo.muon_trace_enable(True)
    mo.muon_trace_read()
    n_tr = 5
    for _ in range(n_tr):
        mo.limuon_step_batched(arr, mo.BF16, hp, ws, d_status=status)
    torch.cuda.synchronize(dev)
    recs = mo.muon_trace_read()
    mo.muon_trace_enable(False)
    per = len(recs) // n_tr
    kms = [0.0] * per
    for i, (_, _, ms_) in enumerate(recs):
        kms[i % per] += ms_ / n_tr
    stream = torch.cuda.current_stream(dev)
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    with torch.cuda.graph(graph, stream=cap):
        mo.limuon_step_batched(arr, mo.BF16, hp, ws, d_status=status, stream=torch.cuda.current_stream(dev))
    for _ in range(3):
        graph.replay()
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1) / args.steps
    by, fl = limuon_kernel_work(shapes, k)
    pk, src = peaks()
    kernels = {}
    # The sketch, projection and update products run on tensor cores in tf32, three MMAs per
    # product (split operands): their arithmetic floor is 3 x flops at the tf32 dense peak, taken
    # as the bf16 peak x 1.1 / 2.25 (the nominal tf32 / bf16 ratio).  The row transforms are fp64
    # sums on CUDA cores; the Cholesky and eigen steps are latency-bound k x k work.
    tf32_peak = tf32_tflops(pk)
    tc_kernels = (0, 3, 6)
    for i, name in enumerate(LIMUON_KERNELS[:per]):
        t = kms[i] / 1e3
        kernels[name] = {"us": kms[i] * 1e3, "GB/s": by[i] / t / 1e9, "TFLOP/s": fl[i] / t / 1e12,
                         "hbm_frac": by[i] / t / 1e9 / pk["hbm_gbs"]}
        if i in tc_kernels:
            kernels[name]["tf32_frac"] = 3.0 * fl[i] / t / 1e12 / tf32_peak
    top = max(range(per), key=lambda i: kms[i])
    t_top = kms[top] / 1e3
    # the binding roof of the dominant kernel: the larger of its memory and arithmetic times
    if top in tc_kernels and 3.0 * fl[top] / (tf32_peak * 1e12) > by[top] / (pk["hbm_gbs"] * 1e9):
        roof = {"bound": "tensor", "achieved": 3.0 * fl[top] / t_top / 1e12, "peak": tf32_peak, "unit": "TFLOP/s",
                "frac": 3.0 * fl[top] / t_top / 1e12 / tf32_peak, "traffic": None,
                "peak_source": f"{src} bf16 peak x 1.1 / 2.25 (tf32), three MMAs per product"}
    else:
        roof = {"bound": "hbm", "achieved": by[top] / t_top / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": by[top] / t_top / 1e9 / pk["hbm_gbs"], "traffic": None, "peak_source": f"{src} (copy)"}
    roof["kernel"] = LIMUON_KERNELS[top]
    el = sum(r * c for r, c in shapes)
    line = {"metric": "LiMuon optimizer step time, ms", "value": ms, "unit": "ms", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16 W/G, fp32 M and products, fp64 k x k factors",
            "data": "synthetic",
            "config": {"workload": f"{w['name']}: {len(shapes)} matrices, {el} elements, rank {hp['rank']}, "
                                   f"oversampling {hp['oversample']}",
                       "l2": f"inputs larger than L2: {el * 14 / 1e9:.2f} GB of W, G and M per step",
                       "kernels": kernels, "launches_per_step": per},
            "roofline": roof, "cpu_baseline": cpu,
            "parity": {"vs": "fp64 oracle from the GPU's own fp32 momentum, relative Frobenius", "groups": parity},
            "gpu_launches": per * args.steps, "clocks": clk, "launch": "graph (one CUDA graph per step)"}
    print(json.dumps(line), flush=True)
    del graph


def run_polar_route(args, w):
    """Time gram_polar (Gram route with restarts and the 1.05 divisor) or ns_polar
    with the same converged schedule on the workload's matrices (log-spaced
    spectra, condition numbers 1e1..1e3), one call per shape batch per step.
    Work is the library's own algorithmic flop count of the launches."""
    import torch
    import muon_family_optimizer_b200 as mo
    from collections import OrderedDict
    from muon_family_optimizer_b200 import synthetic as syn
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    dt = w["ns_dtype"]
    groups = OrderedDict()
    for j, (r, c) in enumerate(w["shapes"]):
        groups.setdefault((r, c), []).append(j)
    kappas = [1e1, 1e2, 1e3]
    batches = []
    for (r, c), idx in groups.items():
        X = torch.stack([syn.log_spectrum(r, c, kappas[i % 3], 4000 + j, device=dev) for i, j in enumerate(idx)])
        X = X.to(dt).contiguous()
        size = (mo.gram_polar_workspace_size if args.route == "gram" else mo.ns_polar_workspace_size)(
            len(idx), r, c, mo._dtype_code(dt))
        batches.append((X, torch.empty_like(X), torch.empty(size, dtype=torch.uint8, device=dev)))
    sched = mo.converged_schedule()
    fn = mo.gram_polar if args.route == "gram" else mo.ns_polar
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(st=None):
        for X, out, ws in batches:
            fn(X, out, sched, ws, d_status=status, stream=st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} after warm-up")
    mo.muon_trace_enable(True)
    mo.muon_trace_read()
    step()
    torch.cuda.synchronize(dev)
    mo.muon_trace_enable(False)
    recs = mo.muon_trace_read()
    work = sum(wk for k, wk, ms in recs if k in (mo.KERNEL_SYM, mo.KERNEL_UPD))
    stream = torch.cuda.current_stream(dev)
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    with torch.cuda.graph(g, stream=cap):
        step(torch.cuda.current_stream(dev))
    for _ in range(max(2, args.warmup)):
        g.replay()
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        g.replay()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1) / args.steps
    groups_desc = " + ".join(f"{len(v)} x {r}x{c}" for (r, c), v in groups.items())
    line = {"metric": METRIC, "value": work / (ms / 1e3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": {torch.bfloat16: "bf16", torch.float16: "fp16", torch.float32: "fp32"}[dt],
            "data": "synthetic (log-spaced spectra, condition numbers 1e1, 1e2, 1e3)",
            "config": {"workload": f"{w['name']}: {groups_desc}, {'gram_polar' if args.route == 'gram' else 'ns_polar'}"
                                   " with the converged schedule (8 quintic + 6 cubic, restarts 3/5/7, divisor 1.05)",
                       "route": args.route, "launches_per_step": len(recs), "work_flops_per_step": work},
            "gpu_launches": len(recs) * args.steps, "clocks": clk, "launch": "graph (one CUDA graph per step)"}
    print(json.dumps(line), flush=True)
    del g


def select_workload(args):
    from muon_family_optimizer_b200 import synthetic as syn
    w = dict(syn.WORKLOADS[args.workload])
    w["name"] = args.workload
    if args.layers:
        if not w.get("layer_size"):
            raise SystemExit(f"--layers: {args.workload} has no layer structure")
        n = args.layers * w["layer_size"]
        if n > len(w["shapes"]):
            raise SystemExit(f"--layers: {args.workload} has {len(w['shapes']) // w['layer_size']} layers")
        w["shapes"] = w["shapes"][:n]
    return w


def workload_label(args, w):
    name = args.workload + (f"[{args.layers} layers]" if args.layers else "")
    return name


def main():
    args = parse()
    w = select_workload(args)
    ns_steps = args.ns_steps
    if args.impl == "reference":
        return run_reference(args, w, ns_steps)
    if args.route == "adamw":
        return run_adamw_route(args, w)
    if args.route == "limuon":
        return run_limuon_route(args, w)
    if args.route == "model":
        return run_model_route(args, w)
    if args.route != "step":
        return run_polar_route(args, w)
    return run_step_route(args, w, ns_steps)


def run_step_route(args, w, ns_steps):
    import torch
    import torch.distributed as dist
    import muon_family_optimizer_b200 as mo
    from muon_family_optimizer_b200 import sharding
    from muon_family_optimizer_b200 import synthetic as syn

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    sharded = world > 1 and not args.replicas
    lite = args.variant == "lite"

    w_dt, ns_dt = w["w_dtype"], w["ns_dtype"]
    shapes = w["shapes"]
    assignment = sharding.partition(shapes, world) if sharded else None
    owned = assignment[rank] if sharded else list(range(len(shapes)))
    # ---- state: weights of every matrix (replicas); gradients and optimizer
    # state of the matrices this rank steps; two gradient sets in one buffer each
    nel_owned = sum(shapes[j][0] * shapes[j][1] for j in owned)
    nel = sum(r * c for r, c in shapes)
    esz = torch.empty((), dtype=w_dt).element_size()
    gbuf = [torch.empty(max(1, nel_owned), dtype=w_dt, device=dev) for _ in range(2)]
    full = [[None] * len(shapes), [None] * len(shapes)]   # per gradient set: every matrix's dict
    torch.manual_seed(1234 + rank)
    cache = {}
    off = 0
    mine = set(owned)
    for j, (r, c) in enumerate(shapes):
        W = syn.initial_weight(args.workload, j, r, c, device=dev).to(w_dt)
        if j not in mine:
            full[0][j] = full[1][j] = dict(W=W)
            continue
        key = (r, c)
        if key not in cache:
            cache[key] = [syn.gradient(args.workload, j, t, r, c, device=dev) for t in range(2)]
        M = torch.zeros(r, c, dtype=torch.float32, device=dev)
        if lite:
            B = (cache[key][1] * -0.01).to(torch.bfloat16).contiguous()
        else:
            Gp = cache[key][1].to(w_dt).contiguous()
            A = torch.zeros(r, c, dtype=torch.float32, device=dev)
        for t in range(2):
            g = gbuf[t][off:off + r * c].view(r, c)
            sign = torch.randint(0, 2, (1, c), device=dev, dtype=torch.int8).float() * 2 - 1
            g.copy_(cache[key][t] * sign)
            full[t][j] = dict(W=W, G=g, B=B, M=M) if lite else dict(W=W, G=g, G_prev=Gp, A=A, M=M)
        off += r * c
    del cache
    params = [[full[t][j] for j in owned] for t in range(2)]
    arrs = [(mo.make_lite_params if lite else mo.make_params)(p) for p in params] if owned else None
    scheds = {"direct": mo.quintic_schedule(ns_steps),
              "gram": mo.quintic_gram_schedule(ns_steps, gram_aspect=args.gram_aspect)}
    sched = scheds[args.step_route]
    other = "gram" if args.step_route == "direct" else "direct"
    compare = world == 1 and not args.no_route_compare
    size_fn = mo.muon_lite_workspace_size if lite else mo.muon_workspace_size
    ws_size = max([size_fn(arrs[0], mo._dtype_code(ns_dt), scheds[r]) for r in
                   ((args.step_route, other) if compare else (args.step_route,))]) if owned else 256
    ws = torch.empty(ws_size, dtype=torch.uint8, device=dev)
    step_fn = mo.muon_lite_step_batched if lite else mo.muon_step_batched
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    wcode, ncode = mo._dtype_code(w_dt), mo._dtype_code(ns_dt)
    if sharded and lite:
        raise SystemExit("the sharded step runs the MONA variant; use --replicas with --variant lite")
    xbuf = None
    if sharded:
        per = sharding.exchange_numel([full[0][j]["W"] for j in range(len(shapes))], assignment)
        xbuf = (torch.empty(per, dtype=w_dt, device=dev), torch.empty(world * per, dtype=w_dt, device=dev))

    def step(i, st=None, sc=None):
        st = st if st is not None else stream
        sc = sc if sc is not None else sched
        if sharded:
            sharding.sharded_step(full[i % 2], wcode, ncode, w["hp"], sc, ws, rank, world, d_status=status,
                                  stream=st, buffers=xbuf)
        elif owned:
            step_fn(arrs[i % 2], wcode, ncode, w["hp"], sc, ws, d_status=status, stream=st)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} after warm-up")

    # One step per gradient set captured as a CUDA graph (the library's launches
    # are plain stream work: capturable once its one-time set-up ran above).
    # The sharded step (with its collective) is launched eagerly.
    graphs = None
    if args.launch == "graph" and not sharded:
        graphs = []
        cap = torch.cuda.Stream(dev)
        for i in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                step(i, torch.cuda.current_stream(dev))
            graphs.append(g)
        for i in range(max(2, args.warmup)):
            graphs[i % 2].replay()
        torch.cuda.synchronize(dev)

    def run(i):
        if graphs is not None:
            graphs[i % 2].replay()
        else:
            step(i)

    # ---- timed region (device time, CUDA events on the step's stream)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(args.steps):
        run(i)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms_total = ev0.elapsed_time(ev1)
    if world > 1:
        t = torch.tensor([ms_total], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_total = float(t.item())
    ms_step = ms_total / args.steps
    copies = 1 if sharded else world               # model steps per timed step, all ranks

    # ---- per-kernel device times: steps launched eagerly with every launch of
    # the library bracketed by CUDA events on its stream (about 5 s of steps)
    ktrace = max(2, min(args.steps, 50, int(5000.0 / max(ms_step, 1e-3))))
    mo.muon_trace_enable(True)
    mo.muon_trace_read()
    for i in range(ktrace):
        if owned:
            step_fn(arrs[i % 2], wcode, ncode, w["hp"], sched, ws, d_status=status, stream=stream)
    torch.cuda.synchronize(dev)
    mo.muon_trace_enable(False)
    recs = mo.muon_trace_read()
    # the work the kernels of one step do (the Gram route's own algorithmic flops)
    fl_exec = sum(wk for kind, wk, _ in recs if kind in (mo.KERNEL_SYM, mo.KERNEL_UPD, mo.KERNEL_SIMT)) / ktrace
    per = {}
    for kind, work, ms in recs:
        d = per.setdefault(mo.KERNEL_NAMES[kind], {"launches": 0, "work": 0.0, "ms": 0.0})
        d["launches"] += 1
        d["work"] += work
        d["ms"] += ms
    # headline work: the direct iteration's algorithmic flops, or the Gram
    # route's own count (what its kernels execute) when it is the headline
    fl_step = ns_flops(shapes, ns_steps)
    if args.step_route == "gram":
        fl_step = fl_exec
        if sharded:     # every rank traced its own share
            t = torch.tensor([fl_exec], device=dev, dtype=torch.float64)
            dist.all_reduce(t)
            fl_step = float(t.item())
    value = copies * fl_step * args.steps / (ms_total / 1e3) / 1e12
    pk, pk_src = peaks()
    dom = max(per.items(), key=lambda kv: kv[1]["ms"])[0] if per else None
    roofline = None
    if dom:
        d = per[dom]
        if dom in ("prepass", "other"):
            ach, peak, unit, bound = d["work"] / (d["ms"] / 1e3) / 1e9, pk["hbm_gbs"], "GB/s", "hbm"
        else:
            sustained = ms_total > 1000.0
            peak = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
            ach, unit, bound = d["work"] / (d["ms"] / 1e3) / 1e12, "TFLOP/s", "tensor"
        nel_launch = nel_owned
        traffic, traffic_src = recorded_traffic(dom, args.workload, ns_steps, elements=nel_launch)
        roofline = {"bound": bound, "kernel": dom, "achieved": ach, "peak": peak, "unit": unit,
                    "frac": ach / peak, "traffic": traffic,
                    "traffic_source": traffic_src or "no ncu record for the current kernel sources",
                    "peak_source": f"{pk_src} ({'sustained' if bound == 'tensor' and ms_total > 1000 else 'burst' if bound == 'tensor' else 'copy'})"}
    kernels = {}
    for name, d in per.items():
        rate = d["work"] / (d["ms"] / 1e3)
        kernels[name] = {"launches": d["launches"], "ms_per_step": round(d["ms"] / ktrace, 4),
                         "share": round(d["ms"] / max(1e-9, sum(x["ms"] for x in per.values())), 4),
                         ("GB/s" if name in ("prepass", "other") else "TFLOP/s"):
                             round(rate / 1e9, 1) if name in ("prepass", "other") else round(rate / 1e12, 1)}
    launches_per_step = len(recs) / max(1, ktrace)

    # ---- the other route of the same step, timed the same way (one GPU)
    route_cmp = None
    if compare and owned and not sharded:
        sc2 = scheds[other]
        for i in range(2):
            step(i, sc=sc2)
        torch.cuda.synchronize(dev)
        mo.muon_trace_enable(True)
        mo.muon_trace_read()
        step(0, sc=sc2)
        torch.cuda.synchronize(dev)
        mo.muon_trace_enable(False)
        recs2 = mo.muon_trace_read()
        fl2 = sum(wk for kind, wk, _ in recs2 if kind in (mo.KERNEL_SYM, mo.KERNEL_UPD, mo.KERNEL_SIMT))
        g2 = []
        cap = torch.cuda.Stream(dev)
        for i in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                step(i, torch.cuda.current_stream(dev), sc=sc2)
            g2.append(g)
        for i in range(2):
            g2[i % 2].replay()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            g2[i % 2].replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms2 = e0.elapsed_time(e1) / args.steps
        if int(status.item()) != 0:
            raise RuntimeError(f"device status {int(status.item())} after the {other} route")
        gram_ms, direct_ms = (ms2, ms_step) if other == "gram" else (ms_step, ms2)
        gram_fl, direct_fl = (fl2, fl_exec) if other == "gram" else (fl_exec, fl2)
        route_cmp = {"other_route": other, "ms_per_step": ms2, "launches_per_step": len(recs2),
                     "TFLOP/s": fl2 / (ms2 / 1e3) / 1e12, "flops_per_step": fl2,
                     "gram_aspect": args.gram_aspect, "gram_restarts": list(mo.GRAM_STEP_RESTARTS),
                     "gram_vs_direct": {"flops": gram_fl / direct_fl, "ms": gram_ms / direct_ms},
                     "note": "same inputs and launch mode; Gram route on shape groups with long side >= "
                             f"{args.gram_aspect:g} x short side, direct iteration elsewhere"}
        del g2

    # ---- end to end through the public API: each step's gradients copied from
    # pinned host memory (one host set, into the two device buffers in turn, on
    # a copy stream overlapping the previous step), the step, then a
    # device->host read of the step's status word
    e2e = None
    if not args.no_e2e:
        host_g = torch.empty(gbuf[0].numel(), dtype=w_dt, pin_memory=True)
        host_g.copy_(gbuf[0])
        host_status = torch.zeros(1, dtype=torch.int32).pin_memory()
        s_copy = torch.cuda.Stream(dev)
        copied = [torch.cuda.Event() for _ in range(2)]
        used = [torch.cuda.Event() for _ in range(2)]
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        k = max(3, min(args.steps, 50, int(10000.0 / max(ms_step, 1e-3))))

        def issue_copy(i):
            with torch.cuda.stream(s_copy):
                s_copy.wait_event(used[i % 2])          # buffer no longer read by step i-2
                gbuf[i % 2].copy_(host_g, non_blocking=True)
                copied[i % 2].record(s_copy)

        for e in used:
            e.record(stream)
        t0 = time.perf_counter()
        issue_copy(0)
        for i in range(k):
            if i + 1 < k:
                issue_copy(i + 1)
            stream.wait_event(copied[i % 2])
            run(i)
            used[i % 2].record(stream)
            host_status.copy_(status, non_blocking=True)   # D2H read of the step's result
            stream.synchronize()
            if int(host_status.item()) != 0:
                raise RuntimeError(f"device status {int(host_status.item())}")
        e_s = time.perf_counter() - t0
        e_ms = e_s * 1e3
        h2d = float(nel_owned * esz)
        if world > 1:
            t = torch.tensor([e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t.item())
            t = torch.tensor([h2d], device=dev, dtype=torch.float64)
            dist.all_reduce(t)
            h2d = float(t.item())
        e2e = {"value": copies * fl_step * k / (e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": 4 * world, "ms_per_step": e_ms / k,
               "steps": k, "timing": "wall clock over the loop, H2D of step i+1 overlapped with step i"}
        del host_g

    launch_desc = args.launch + (" (one CUDA graph per step)" if graphs is not None else
                                 " (eager: the sharded step's collective)" if sharded else "")
    cpu = None
    parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        del gbuf, params, arrs, full, ws, graphs
        torch.cuda.empty_cache()
        cpu = cpu_baseline(w, ns_steps)
        if not lite:
            parity = group_parity(w, ns_steps, dev)

    if rank == 0:
        groups, _ = describe(args.workload, w)
        # W, G, G_prev (w dtype), A, M (fp32); MONA-Lite: W, G, B (bf16), M
        state_bytes = nel * (2 * esz + 2 + 4) if lite else nel * (3 * esz + 8)
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
                "scaling": "strong" if sharded else "weak",
                "vs_baseline": None, "dtype": {torch.bfloat16: "bf16", torch.float16: "fp16",
                                               torch.float32: "fp32"}[ns_dt],
                "data": "synthetic (seeded; shapes of the named model, random values)",
                "config": {"workload": f"{workload_label(args, w)}{' (MONA-Lite)' if lite else ''}: {groups} "
                                       "(wide view s x l)",
                           "variant": args.variant, "elements": nel,
                           "ns_steps": ns_steps, "w_dtype": str(w_dt).replace("torch.", ""),
                           "state_bytes": state_bytes,
                           "l2": f"inputs larger than L2: {state_bytes / 1e9:.2f} GB of state per step",
                           "parallelism": (f"sharded over {world} ranks: whole matrices, flop-balanced, one "
                                           "all-gather of the updated weights per step" if sharded else
                                           f"{world} replica(s), each rank steps its own copy")},
                "dense_equivalent": {"value": copies * ns_flops_dense(shapes, ns_steps) * args.steps
                                     / (ms_total / 1e3) / 1e12,
                                     "unit": "TFLOP/s", "note": "symmetric products counted in full (not the headline)"}
                                    if args.step_route == "direct" else None,
                "step_route": args.step_route + (f" (Gram route where long side >= {args.gram_aspect:g} x short "
                                                 "side)" if args.step_route == "gram" else ""),
                "route_compare": route_cmp,
                "roofline": roofline, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
                "parity": parity and {"vs": "fp64 oracle from the same 16-bit inputs, one matrix per shape group, "
                                            "relative Frobenius", "groups": parity},
                "gpu_launches": int(round(launches_per_step * args.steps)), "clocks": clk,
                "launch": launch_desc,
                "kernel_timing": f"per-kernel device time from {ktrace} eagerly launched steps of this rank's "
                                 "matrices, each launch bracketed by CUDA events on its stream"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
