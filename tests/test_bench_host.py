"""Host logic of bench.py (CPU).

The headline metric counts algorithmic Newton-Schulz flops: per quintic step
and matrix (s x l wide view) s^2 l for X X^T (half of the dense product), s^3
for A A (half) and 2 s^2 l for B X.  Checked against values worked out from
that definition: 5 steps of a 768 x 2048 matrix = 5 (3 * 768^2 * 2048 + 768^3).
The roofline's DRAM-traffic figure is read from an ncu record only while the
kernel sources still hash to the recorded digest.
"""
import json
import os
import shutil

import pytest

import bench
from muon_family_optimizer_b200 import synthetic as syn


@pytest.mark.parametrize("shape,expect", [((768, 2048), 20.38e9), ((2048, 768), 20.38e9),
                                          ((1024, 4096), 69.79e9), ((4096, 14336), 3.952e12),
                                          ((2048, 16384), 1.0737e12), ((1024, 1024), 21.47e9)])
def test_ns_flops_per_matrix(shape, expect):
    assert abs(bench.ns_flops([shape], 5) - expect) / expect < 1e-3


@pytest.mark.parametrize("workload,expect", [("gpt2_small", 1.1415e12), ("llama_430m", 7.086e12),
                                             ("llama3_8b", 471.8e12)])
def test_ns_flops_per_workload(workload, expect):
    assert abs(bench.ns_flops(syn.WORKLOADS[workload]["shapes"], 5) - expect) / expect < 1e-3


def test_dense_equivalent_counts_symmetric_products_in_full():
    s, l = 768, 3072
    assert bench.ns_flops_dense([(s, l)], 1) == 4.0 * s * s * l + 2.0 * s ** 3
    assert abs(bench.ns_flops_dense(syn.WORKLOADS["llama3_8b"]["shapes"], 5) - 665.9e12) / 665.9e12 < 1e-3


def test_recorded_traffic_requires_matching_sources(tmp_path, monkeypatch):
    root = tmp_path / "repo"
    for rel in set(sum((list(v) for v in bench.TRAFFIC_SOURCES.values()), [])):
        dst = root / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(bench.ROOT, rel), dst)
    monkeypatch.setattr(bench, "ROOT", str(root))
    (root / "profiles").mkdir()
    rec = {"kernel": "tc_sym", "workload": "gpt2_small", "ns_steps": 5, "bytes_per_launch": 123456,
           "sources": bench.sources_digest("tc_sym")}
    (root / "profiles" / "k.md").write_text("# summary\n\ntraffic-record: " + json.dumps(rec) + "\n")
    assert bench.recorded_traffic("tc_sym", "gpt2_small", 5) == (123456.0, "profiles/k.md")
    assert bench.recorded_traffic("tc_sym", "llama_430m", 5) == (None, None)      # other workload
    assert bench.recorded_traffic("tc_sym", "gpt2_small", 14) == (None, None)     # other schedule
    # a change to one of the kernel's sources retires the record
    with open(root / "muon_family_optimizer_b200" / "csrc" / "gemm_tc.cu", "a") as fh:
        fh.write("\n// changed\n")
    assert bench.recorded_traffic("tc_sym", "gpt2_small", 5) == (None, None)


def test_limuon_kernel_work_counts():
    # one 4 x 6 matrix, k = 3 (32-column factors), 16-bit W/G: per element the sketch moves
    # 2 + 4 + 4 bytes, the projection 4, the update 2 + 2; each of these three products is
    # 3 FMAs per element; the row transforms move 4 rows of 32 floats each way and do
    # 2 k^2 flops per row; the two k x k steps move two 32 x 32 fp64 matrices
    by, fl = bench.limuon_kernel_work([(4, 6)], 3)
    small = 2 * 8 * 32 * 32
    assert by == [24 * 10 + 4 * 12, small, 8 * 4 * 32 + small // 2, 24 * 4 + 4 * (12 + 18), small,
                  8 * 4 * 32 + small // 2, 24 * 4 + 4 * (12 + 18)]
    assert fl == [2.0 * 24 * 3, 0.0, 2.0 * 4 * 9, 2.0 * 24 * 3, 0.0, 2.0 * 4 * 9, 2.0 * 24 * 3]
    by32, _ = bench.limuon_kernel_work([(4, 6)], 3, w_bytes=4)
    assert by32[0] - by[0] == 24 * 2 and by32[6] - by[6] == 24 * 4
    assert len(bench.LIMUON_KERNELS) == len(by)


def test_tf32_peak_from_bf16_peak():
    # 1.1 PF tf32 against 2.25 PF bf16 dense, nominal; applied to the measured bf16 figure
    assert abs(bench.tf32_tflops({"bf16_tflops": 1670.9}) - 1670.9 * 1.1 / 2.25) < 1e-9
    assert abs(bench.tf32_tflops({"bf16_tflops": 2250.0}) - 1100.0) < 1e-9


def test_layers_slice_keeps_whole_layers():
    class A:
        workload, layers = "llama3_8b", 1
    w = bench.select_workload(A)
    assert w["shapes"] == syn.WORKLOADS["llama3_8b"]["shapes"][:7]
    A.layers = 32
    assert len(bench.select_workload(A)["shapes"]) == 224
    A.layers = 33
    with pytest.raises(SystemExit):
        bench.select_workload(A)
    A.workload, A.layers = "moe_gram", 1          # no layer structure
    with pytest.raises(SystemExit):
        bench.select_workload(A)


def test_shape_groups_cheapest_first():
    g = bench.shape_groups(syn.WORKLOADS["llama3_8b"]["shapes"])
    assert [len(m) for _, m in g] == [64, 64, 96]
    costs = [c for c, _ in g]
    assert costs == sorted(costs)
    # both orientations of a shape share a group
    assert {(r, c) for _, r, c in g[2][1]} == {(14336, 4096), (4096, 14336)}


def test_recorded_traffic_scales_a_layer_slice_by_elements(tmp_path, monkeypatch):
    root = tmp_path / "repo"
    for rel in set(sum((list(v) for v in bench.TRAFFIC_SOURCES.values()), [])):
        dst = root / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(bench.ROOT, rel), dst)
    monkeypatch.setattr(bench, "ROOT", str(root))
    (root / "profiles").mkdir()
    rec = {"kernel": "tc_upd", "workload": "llama3_8b", "ns_steps": 5, "bytes_per_launch": 1000.0,
           "elements": 218103808, "sources": bench.sources_digest("tc_upd")}
    (root / "profiles" / "k.md").write_text("traffic-record: " + json.dumps(rec) + "\n")
    b, src = bench.recorded_traffic("tc_upd", "llama3_8b", 5, elements=32 * 218103808)
    assert b == 32000.0 and "scaled" in src
    assert bench.recorded_traffic("tc_upd", "llama3_8b", 5, elements=218103808)[0] == 1000.0


def test_peaks_from_measured_file_and_fallbacks(tmp_path):
    # the generated file: every key measured
    p = tmp_path / "MEASURED_PEAKS.json"
    p.write_text(json.dumps({"hbm_gbs": 6530.6, "bf16_tflops": 1670.9, "bf16_tflops_sustained": 1410.8,
                             "clocks": {"sm": 1965}}))
    pk, src = bench.peaks(str(p))
    assert src == "measured"
    assert pk == {"hbm_gbs": 6530.6, "bf16_tflops": 1670.9, "bf16_tflops_sustained": 1410.8}
    # a key missing: that one from the fallback figures, and the source says so
    p.write_text(json.dumps({"hbm_gbs": 6530.6, "bf16_tflops": 1670.9}))
    pk, src = bench.peaks(str(p))
    assert pk["bf16_tflops_sustained"] == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]
    assert pk["hbm_gbs"] == 6530.6 and src.startswith("measured (")
    # nothing usable, unreadable, or absent: the fallback figures
    for text in (json.dumps({"hbm_gbs": "fast", "bf16_tflops": -1}), "{not json", json.dumps([1, 2])):
        p.write_text(text)
        pk, src = bench.peaks(str(p))
        assert pk == bench.FALLBACK_PEAKS and src.startswith("fallback")
    pk, src = bench.peaks(str(tmp_path / "absent.json"))
    assert pk == bench.FALLBACK_PEAKS and src == "fallback"
