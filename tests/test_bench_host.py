"""bench.py's roofline arithmetic (host logic, no GPU).

Checks the per-launch algorithmic work of each kernel class, the peaks (measured file or
the stated fallback) and the achieved / peak fractions that go into the JSON line.
"""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_kernel_units():
    m, n, r, K, T = 11008, 4096, 1000, 4, 262144
    assert bench.kernel_units("calib", m, n, r, K, T) == (T * (m + n), "B", "hbm")
    assert bench.kernel_units("rhs", m, n, r, K, T) == (2.0 * m * n * r, "FLOP", "tensor")
    # symmetric Gram: half of 2 rows r^2, averaged over the two sides
    assert bench.kernel_units("gram", m, n, r, K, T)[0] == pytest.approx((m + n) * r * r / 2)
    assert bench.kernel_units("solve", m, n, r, K, T)[0] == pytest.approx((m + n) * r * r)
    # the method's Cholesky: r^3 / 3 (the inverse the library also forms is not counted)
    assert bench.kernel_units("chol", m, n, r, K, T) == (float(r) ** 3 / 3, "FLOP", "alu")
    assert bench.kernel_units("ginv", m, n, r, K, T) == (float(r) ** 3 / 3, "FLOP", "tensor")
    assert bench.kernel_units("svid", m, n, r, K, T)[0] == pytest.approx(2.0 * K * (m + n) * r)
    assert bench.kernel_units("objective", m, n, r, K, T) is None


def test_square_layer_calibration_bytes_are_one_stream():
    # on a square layer both streams have C = n: T x n x 2 bytes per launch
    assert bench.kernel_units("calib", 4096, 4096, 2032, 4, 1024)[0] == 1024 * 4096 * 2


def test_roofline_entry_fractions():
    peaks = dict(hbm_gbs=6000.0, bf16_tflops=1600.0, bf16_tflops_sustained=1400.0,
                 fp32_tflops=70.0, source="test")
    m = n = 4096
    r, K, T = 2032, 4, 262144
    e = bench.roofline_entry("rhs", 10, 1.0, m, n, r, K, T, peaks)   # 10 launches in 1 ms
    flops = 2.0 * m * n * r
    assert e["achieved"] == pytest.approx(flops / 1e-4 / 1e12, rel=1e-3)
    assert e["peak"] == 1400.0 and e["unit"] == "TFLOP/s" and e["bound"] == "tensor"
    assert e["frac"] == pytest.approx(e["achieved"] / 1400.0, rel=1e-3)
    c = bench.roofline_entry("calib", 2, 0.5, m, n, r, K, T, peaks)
    assert c["unit"] == "GB/s" and c["achieved"] == pytest.approx(T * 2 * n / 2.5e-4 / 1e9,
                                                                   rel=1e-3)
    # the capture: 1.446 GB for one 65536 x 11008 BF16 stream (1.002 x its T x C x 2 bytes)
    assert c["traffic"] == pytest.approx(1.446e9 * T * n / (65536 * 11008))
    assert c["traffic"] == pytest.approx(T * n * 2, rel=0.01)
    assert bench.roofline_entry("rhs", 0, 1.0, m, n, r, K, T, peaks) is None


def test_traffic_only_for_captured_kernels():
    # the calibration capture scales with the stream size; the inverse update's holds for
    # the rank it was taken at only
    assert bench.ncu_traffic("calib", 4096, 4096, 2032, 262144) > 0
    assert bench.ncu_traffic("newton", 11008, 4096, 1000, 262144) == 55.0e6
    assert bench.ncu_traffic("newton", 4096, 4096, 2032, 262144) is None
    assert bench.ncu_traffic("chol", 4096, 4096, 2032, 262144) is None
    assert bench.ncu_traffic("svid", 4096, 4096, 2032, 262144) is None


def test_alu_peak_is_marked_derived():
    peaks = dict(hbm_gbs=6000.0, bf16_tflops=1600.0, bf16_tflops_sustained=1400.0,
                 fp32_tflops=70.0, source="test")
    e = bench.roofline_entry("chol", 2, 1.0, 4096, 4096, 2032, 4, 1024, peaks)
    assert e["bound"] == "alu" and e["peak"] == 70.0 and "derived" in e["peak_kind"]


def test_peaks_measured_or_fallback(tmp_path, monkeypatch):
    p = bench.read_peaks()
    assert p["source"] in ("measured", "fallback")
    assert p["fp32_tflops"] == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f = bench.read_peaks()
    assert f["source"] == "fallback" and f["hbm_gbs"] == 6650.0 and f["bf16_tflops"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(dict(hbm_gbs=1.0, bf16_tflops=2.0)))
    g = bench.read_peaks()
    assert g["source"] == "measured" and g["bf16_tflops_sustained"] == 2.0


def test_update_units_count_its_own_products():
    # two r x r x r products (2 r^3 each) per step of the Newton-Schulz update
    amount, unit, bound = bench.kernel_units("newton", 11008, 4096, 1000, 4, 262144, ns_steps=4)
    assert (unit, bound) == ("FLOP", "tensor") and amount == 4.0 * 1000 ** 3 * 4
    assert bench.kernel_units("newton", 11008, 4096, 1000, 4, 262144, ns_steps=0)[0] == 4.0e9
