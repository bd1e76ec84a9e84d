"""Host logic of the benchmark line, on CPU: which peak each roofline is taken against,
the arithmetic of the fractions, and that the reference arm and the GPU arm describe the
same workload (`config` carries no arm-specific key)."""
from __future__ import annotations

import pytest

import bench
from mixture_experts_layer_26_b200 import inputs as minp

PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 2000.0, "bf16_tflops_sustained": 1500.0}
PROBE = {"burst_tflops": 3100.0, "sustained_tflops": 2600.0, "how": "test"}


def test_tensor_peak_sources():
    # a measured FP8 figure of the pool wins, then this run's probe, then 2 x bf16
    assert bench.tensor_peak(True, dict(PEAKS, fp8_tflops=3500.0), "measured", PROBE)[0] == 3500.0
    assert bench.tensor_peak(True, PEAKS, "measured", PROBE)[0] == 3100.0
    peak, how = bench.tensor_peak(True, PEAKS, "measured", None)
    assert peak == 4000.0 and "2 x" in how
    assert bench.tensor_peak(False, PEAKS, "measured", PROBE)[0] == 2000.0  # bf16: its own peak


def _measure(kern_ms, ms_step=1.0, touched=8, max_rows=1024):
    return dict(kern_ms=kern_ms, ms_step=ms_step, touched=touched, max_rows=max_rows)


def test_prefill_roofline_is_tensor_bound_against_the_burst_probe():
    s = minp.shape("prefill_fp8")
    m = _measure({"router": 0.02, "gemm1_pair": 0.9, "gemm2_pair": 0.45, "combine": 0.03}, 1.4)
    variant, roof, hbm, ten = bench.roofline_of(s, m, PEAKS, "measured", PROBE, "prefill_fp8")
    assert variant == "normal_pair"
    assert roof["bound"] == "tensor" and roof["kernel"] == "gemm1_pair" and roof["peak"] == 3100.0
    flops = 4.0 * s.R * s.H * s.I
    assert roof["achieved"] == pytest.approx(flops / 0.9e-3 / 1e12, rel=1e-3)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 3100.0, rel=1e-3)
    assert ten["flops"] == 6.0 * s.R * s.H * s.I
    assert ten["frac"] == pytest.approx(6.0 * s.R * s.H * s.I / 1.4e-3 / 1e12 / 3100.0, rel=1e-3)


def test_decode_roofline_is_hbm_bound_on_touched_expert_weights():
    s = minp.shape("mixtral_fp8_decode", 64)
    m = _measure({"router_permute": 0.02, "gemm1_swapab": 0.15, "gemm2_swapab": 0.08}, 0.24, touched=8)
    variant, roof, hbm, _ = bench.roofline_of(s, m, PEAKS, "fallback", PROBE, "mixtral_fp8_decode")
    assert variant == "swap_ab"
    w1 = 8 * 2 * s.H * s.I
    assert roof["bound"] == "hbm" and roof["algorithmic_bytes"] == w1 and roof["peak"] == 6000.0
    assert roof["achieved"] == pytest.approx(w1 / 0.15e-3 / 1e9, rel=1e-3)
    assert "fallback" in roof["peak_kind"]
    assert hbm["weight_bytes"] == 8 * 3 * s.H * s.I and hbm["touched_experts"] == 8


def test_config_is_the_same_for_both_arms():
    for name in ("prefill_fp8", "dsv3_grouped_fp8_decode", "tiny_bf16"):
        cfg = bench.workload_config(minp.shape(name))
        assert "variant" not in cfg and cfg["workload"].startswith(name)


def test_profiled_traffic_matches_whole_workload_tags(tmp_path, monkeypatch):
    """The ncu summaries carry their DRAM traffic under a source hash; the lookup takes the
    kernel's summary for exactly the workload and batch size asked for, and none whose hash
    is not the current source's (synthetic summaries, so no real kernel source is involved)."""
    import bench
    prof = tmp_path / "profiles"
    prof.mkdir()
    for name, traffic, h in (("gemm1_swapab_mixtral_fp8_decode_T1.md", 111, "aa"),
                             ("gemm1_swapab_mixtral_fp8_decode_T64.md", 6464, "aa"),
                             ("gemm1_swapab_mixtral_fp8_decode_T16.md", 1616, "stale")):
        (prof / name).write_text(f"traffic_bytes_per_launch: {traffic}\nsource_hash: {h}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "gemm_source_hash", lambda kernel="": "aa")
    assert bench.profiled_traffic("gemm1_swapab", "mixtral_fp8_decode_T1") == 111
    assert bench.profiled_traffic("gemm1_swapab", "mixtral_fp8_decode_T64") == 6464
    assert bench.profiled_traffic("gemm1_swapab", "mixtral_fp8_decode_T6") is None
    assert bench.profiled_traffic("gemm1_swapab", "mixtral_fp8_decode_T16") is None  # stale hash
    assert bench.profiled_traffic("gemm2_swapab", "mixtral_fp8_decode_T1") is None
