"""bench.py's roofline arithmetic on made-up numbers (no GPU): the bound is
the slower of bytes at the HBM peak and flops at the tensor peak, the tensor
peak switches to the sustained figure from 10 ms steps on, NVFP4 uses four
times the bf16 peaks, and every fraction is achieved / peak."""
import pytest

import bench

PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}


def alg(gb, tflop, block_gb=None, block_tflop=None, touched=100):
    return {"gateup_bytes": gb * 1e9, "gateup_flops": tflop * 1e12,
            "block_bytes": (block_gb or gb) * 1e9, "expert_flops": (block_tflop or tflop) * 1e12,
            "touched_experts": touched}


def test_bytes_bound_kernel():
    # 12 GB and 0.04 TFLOP: 2 ms of HBM against 25 us of tensor work
    roof, block = bench.roofline(alg(12.0, 0.04), 2.5, 3.0, PEAKS, "measured", False)
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s" and roof["peak"] == 6000.0
    assert roof["achieved"] == pytest.approx(12.0e9 / 2.5e-3 / 1e9)
    assert roof["frac"] == pytest.approx(4800.0 / 6000.0)
    assert block["hbm_frac"] == pytest.approx(12e9 / 3e-3 / 1e9 / 6000.0)
    assert block["tensor_peak_kind"] == "burst" and roof["kernel"] == "gateup_grouped_gemm"


def test_flop_bound_kernel_and_the_sustained_peak():
    # 2 GB and 30 TFLOP: a 40 ms step runs against the sustained peak
    roof, block = bench.roofline(alg(2.0, 30.0), 25.0, 40.0, PEAKS, "measured", False)
    assert roof["bound"] == "tensor" and roof["peak_kind"] == "sustained"
    assert roof["peak"] == 1400.0
    assert roof["frac"] == pytest.approx(30.0 / 25e-3 / 1400.0)
    assert block["tensor_frac"] == pytest.approx(30.0 / 40e-3 / 1400.0)
    assert block["tensor_frac_of_burst"] == pytest.approx(30.0 / 40e-3 / 1600.0)
    # the same kernel in a short step is measured against the burst peak
    roof, block = bench.roofline(alg(2.0, 30.0), 5.0, 8.0, PEAKS, "measured", False)
    assert roof["peak"] == 1600.0 and roof["peak_kind"] == "burst"


def test_nvfp4_peaks_are_four_times_bf16():
    roof, block = bench.roofline(alg(1.0, 30.0), 5.0, 12.0, PEAKS, "measured", True)
    assert roof["bound"] == "tensor" and roof["peak"] == 4 * 1400.0
    assert block["tensor_frac_of_burst"] == pytest.approx(30.0 / 12e-3 / (4 * 1600.0))
    assert roof["kernel"] == "gateup_grouped_gemm_nvfp4" and "peak_note" in roof


def test_no_kernel_time_gives_no_fraction_and_fallback_is_named():
    roof, block = bench.roofline(alg(12.0, 0.04), None, 3.0, PEAKS, "fallback", False)
    assert roof["achieved"] is None and roof["frac"] is None
    assert roof["peak_source"] == "fallback"
    assert block["hbm_frac"] > 0


def test_gateup_traffic_scales_by_its_unit_and_needs_matching_sources(monkeypatch):
    import synth

    rec = dict(bench.GATEUP_TRAFFIC["long"], bytes=100, sha256="not-the-sources")
    monkeypatch.setitem(bench.GATEUP_TRAFFIC, "long", rec)
    wl = synth.workload("long")
    alg = {"touched_experts": 3}
    assert bench.gateup_traffic(wl, alg) is None  # sources changed since the capture
    rec["sha256"] = bench.sources_sha256(rec["sources"])
    assert bench.gateup_traffic(wl, alg) == 100 * wl.T * wl.K  # per assignment
    dec = dict(bench.GATEUP_TRAFFIC["decode"], bytes=7)
    dec["sha256"] = bench.sources_sha256(dec["sources"])
    monkeypatch.setitem(bench.GATEUP_TRAFFIC, "decode", dec)
    assert bench.gateup_traffic(synth.workload("decode"), alg) == 21  # per touched expert
    assert bench.gateup_traffic(synth.workload("prefill"), alg) is None  # no record
