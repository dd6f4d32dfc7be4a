"""Host-side pieces of the benchmark (no GPU): the per-workload figures its
roofline is computed from, the choice of bound, the labels, and the int8
denominator."""
import types

import pytest

import bench
import workloads as WL

PEAKS = {"hbm_gbs": 6453.7, "bf16_tflops": 1686.7}

# name -> (algorithmic MB, GFLOP, bound)
EXPECTED = {
    "tiny_w8a16_perchannel_f16": (0.0458, 0.0010486, "hbm"),
    "w8a16_pertensor_bf16_2048x4096x4096": (67.12, 68.72, "tensor"),
    "w4a16_g128_bf16_4096x4096x4096": (76.02, 137.44, "tensor"),
    "decode_w4a16_g64_bf16_1x16x8192x28672": (133.36, 7.52, "hbm"),
    "w8a8_pertoken_4x2048x8192x1024": (109.09, 137.44, "tensor"),
    "fp8_perchannel_bf16_4096x4096x4096": (83.89, 137.44, "tensor"),
    "w4a16_g128_bf16_256x4096x4096": (13.11, 8.59, "tensor"),
    "nonquant_bf16_4096x4096x4096": (100.66, 137.44, "tensor"),
}


def _prob(name):
    case = WL.workload(name)
    return types.SimpleNamespace(case=case, int8=not hasattr(case, "wdt"), flops=2.0 * case.m * case.n * case.k,
                                 bytes=bench.algorithmic_bytes(case))


def test_every_named_workload_has_its_figures():
    assert sorted(EXPECTED) == sorted(WL.WORKLOAD_NAMES)


@pytest.mark.parametrize("name", sorted(EXPECTED))
def test_algorithmic_bytes_flops_and_bound(name):
    mb, gflop, bound = EXPECTED[name]
    p = _prob(name)
    assert p.bytes / 1e6 == pytest.approx(mb, rel=2e-3)
    assert p.flops / 1e9 == pytest.approx(gflop, rel=2e-3)
    got_bound, peak, unit, _ = bench.workload_roofline(p, PEAKS, {"peak_tops": 3061.6, "peak_from": "x", "shape": "s"})
    assert got_bound == bound
    assert unit == ("GB/s" if bound == "hbm" else "TFLOP/s")


def test_int8_denominator_is_the_measured_peak_else_twice_bf16():
    p = _prob("w8a8_pertoken_4x2048x8192x1024")
    _, peak, _, src = bench.workload_roofline(p, PEAKS, {"peak_tops": 3061.6, "peak_from": "x", "shape": "8192^3"})
    assert peak == 3061.6 and "measured in this run" in src
    _, peak, _, src = bench.workload_roofline(p, PEAKS, None)
    assert peak == 2 * PEAKS["bf16_tflops"] and "nominal" in src


def test_labels():
    d = {n: bench.describe_weight(WL.workload(n)) for n in WL.WORKLOAD_NAMES}
    assert d["w4a16_g128_bf16_4096x4096x4096"] == "int4 packed, per-group g=128 scale + offset"
    assert d["fp8_perchannel_bf16_4096x4096x4096"] == "fp8-e4m3 packed, per-channel scale"
    assert d["nonquant_bf16_4096x4096x4096"].startswith("bf16 (non-quantised)")
    assert d["w8a8_pertoken_4x2048x8192x1024"].startswith("int8 x int8")
    assert bench.arithmetic_dtype(WL.workload("w8a8_pertoken_4x2048x8192x1024")) == "i8"
    assert bench.arithmetic_dtype(WL.workload("tiny_w8a16_perchannel_f16")) == "f16"
