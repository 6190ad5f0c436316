"""Host logic of bench.py (no GPU): the peak denominators, the per-expert
byte counts, and the ncu-traffic lookup that reports `roofline.traffic` only
for the kernel sources it was captured from."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import workloads as W  # noqa: E402


def fake_root(tmp_path, peaks=None):
    csrc = tmp_path / "moe_expert_layer_08_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("gemm.cu", "moe_common.cuh", "moe_internal.h"):
        (csrc / f).write_text(f"// {f}\n")
    (tmp_path / "profiles").mkdir()
    if peaks is not None:
        (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(peaks))
    return tmp_path


def test_peaks_measured_and_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(fake_root(tmp_path / "a", {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0,
                                                                       "bf16_tflops_sustained": 1300.0})))
    assert bench.peaks() == dict(hbm=6000.0, bf16=1600.0, bf16_sustained=1300.0, source="measured")
    monkeypatch.setattr(bench, "ROOT", str(fake_root(tmp_path / "b")))
    assert bench.peaks()["source"] == "fallback"


def test_expert_bytes():
    w = W.WORKLOADS[1]
    b1, b2 = bench.expert_bytes(w, "mx")
    assert (b1, b2) == (2 * 3072 * 7168 * 17 // 32, 7168 * 3072 * 17 // 32) == (23396352, 11698176)
    n1, n2 = bench.expert_bytes(w, "nvfp4")
    assert (n1, n2) == (2 * 3072 * 7168 * 9 // 16, 7168 * 3072 * 9 // 16)


def test_traffic_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    root = fake_root(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    decode, prefill = W.WORKLOADS[1], W.WORKLOADS[3]
    for regime, g1, g2 in (("decode", 100.0, 50.0), ("prefill", 110.0, 60.0)):
        (root / "profiles" / f"gemm_{regime}_traffic.json").write_text(json.dumps(
            {"kernel_source_sha256": bench.kernel_source_hash(),
             "gemm1_bytes_per_touched_expert": g1, "gemm2_bytes_per_touched_expert": g2}))
    assert bench.measured_traffic(decode, 10, True) == 1000.0
    assert bench.measured_traffic(decode, 10, False) == 500.0
    assert bench.measured_traffic(prefill, 10, True) == 1100.0      # T*k > 8E: the prefill capture
    assert bench.measured_traffic(decode, 10, True, "nvfp4") is None
    # any edit to the GEMM sources retires the capture
    (root / "moe_expert_layer_08_b200" / "csrc" / "gemm.cu").write_text("// changed\n")
    assert bench.measured_traffic(decode, 10, True) is None


def test_cublas_fp8_context(tmp_path, monkeypatch):
    root = fake_root(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.cublas_fp8() is None
    (root / "profiles" / "cublas_fp8_matmul_8192.json").write_text(json.dumps(
        {"per_tensor": {"burst_tflops": 3000.0, "sustained_tflops": 2500.0},
         "mx_blockwise_1x32": {"burst_tflops": 2700.0, "sustained_tflops": 2200.0}}))
    assert bench.cublas_fp8() == {"per_tensor": dict(burst=3000.0, sustained=2500.0),
                                  "mx_blockwise_1x32": dict(burst=2700.0, sustained=2200.0)}


def test_committed_cublas_fp8_figure_is_below_the_derived_denominator():
    # the measured FP8 figure is context: the reported roofline keeps the
    # stricter 2 x bf16 sustained denominator while it is the larger one
    c8, pk = bench.cublas_fp8(), bench.peaks()
    assert c8 is not None and set(c8) == {"mx_blockwise_1x32", "per_tensor"}
    for c in c8.values():
        assert 0 < c["sustained"] <= c["burst"]
        if pk["source"] == "measured":
            assert c["sustained"] <= 2.0 * pk["bf16_sustained"]


def test_both_arms_print_the_same_config_keys():
    # the driver compares the two arms' `config` objects: the GPU arm's and
    # the oracle arm's come from the same function with the same arguments
    import types
    args = types.SimpleNamespace(layout="packets")
    for w in W.WORKLOADS.values():
        b12 = bench.expert_bytes(w, "mx")
        a = bench.workload_config(w, args, 1, 44, b12)
        b = bench.workload_config(w, args, 1, 44, b12)
        assert a == b
        assert set(a) == {"workload", "T", "E", "k", "H", "I", "seed", "routing", "parallelism",
                          "weight_layout", "l2"}
        assert a["workload"] == w.name and a["parallelism"] == "replicas x1"


def test_shared_roofline_takes_the_binding_bound():
    """The shared expert's roofline: HBM (its bf16 weights read once) while
    that takes longer than the FLOPs at the tensor peak, else the tensor pipe;
    the fraction is achieved / peak in the bound's unit, the other beside it."""
    pk = dict(hbm=6000.0, bf16=1600.0, bf16_sustained=1200.0, source="measured")
    wbytes = 3 * 7168 * 2048 * 2
    for T, us in [(8, 40.0), (8192, 600.0)]:
        flops = 2.0 * T * 3 * 7168 * 2048
        r = bench.shared_roofline(flops, wbytes, us * 1e-3, pk)
        t_hbm, t_tc = wbytes / 6000e9, flops / 1200e12
        assert r["bound"] == ("hbm" if t_hbm > t_tc else "tensor")
        assert r["other"]["bound"] == ("tensor" if t_hbm > t_tc else "hbm")
        tf = flops / (us * 1e-6) / 1e12
        gbps = wbytes / (us * 1e-6) / 1e9
        if r["bound"] == "hbm":
            assert r["unit"] == "GB/s" and r["frac"] == pytest.approx(gbps / 6000.0)
            assert r["other"]["frac"] == pytest.approx(tf / 1200.0)
        else:
            assert r["unit"] == "TFLOP/s" and r["frac"] == pytest.approx(tf / 1200.0)
            assert r["other"]["frac"] == pytest.approx(gbps / 6000.0)
    assert bench.shared_roofline(2.0 * 8 * 3 * 7168 * 2048, wbytes, 0.04, pk)["bound"] == "hbm"
    assert bench.shared_roofline(2.0 * 8192 * 3 * 7168 * 2048, wbytes, 0.6, pk)["bound"] == "tensor"


def test_layer_roofline_takes_the_binding_bound():
    """The layer's roofline is the dominant GEMM's binding one: HBM when its
    algorithmic bytes at the measured bandwidth take longer than its FLOPs at
    the sustained tensor peak (decode; NVFP4 at prefill, whose FP4 MMA runs at
    twice the FP8 rate), else the tensor pipe (FP8 x FP4 prefill), with the
    other fraction beside it."""
    import types

    import numpy as np
    import torch
    pk = bench.peaks()
    for wi, fmt, want in [(1, "mx", "hbm"), (3, "mx", "tensor"), (3, "nvfp4", "hbm"), (4, "mx", "tensor")]:
        w = W.WORKLOADS[wi]
        idx = (torch.arange(w.T * w.k) % w.E).view(w.T, w.k)
        r = dict(g={"idx": idx}, ms=2.0, stage_ms=np.array([[0.01, 1.2, 0.6, 0.05]]), staged_ms=2.0, clocks={})
        f = bench.layer_figures(types.SimpleNamespace(format=fmt, steps=1), w, r, 1)
        ro = f["roofline"]
        b1, _ = bench.expert_bytes(w, fmt)
        kbytes = min(w.T * w.k, w.E) * b1  # the experts the routing touches
        kflops = 2.0 * w.T * w.k * 2 * w.I * w.H
        peak_tc = (2.0 if fmt == "mx" else 4.0) * pk["bf16_sustained"]
        assert ro["bound"] == want, (w.name, fmt)
        assert want == ("hbm" if kbytes / (pk["hbm"] * 1e9) >= kflops / (peak_tc * 1e12) else "tensor")
        if want == "hbm":
            assert ro["frac"] == pytest.approx(kbytes / 1.2e-3 / 1e9 / pk["hbm"])
            assert ro["tensor"]["frac"] == pytest.approx(kflops / 1.2e-3 / 1e12 / peak_tc)
        else:
            assert ro["frac"] == pytest.approx(kflops / 1.2e-3 / 1e12 / peak_tc)
            assert ro["hbm"]["frac"] == pytest.approx(kbytes / 1.2e-3 / 1e9 / pk["hbm"])
