"""Host-side arithmetic of the benchmark: the dominant kernel's algorithmic
bytes and flops per launch for each expert precision (the roofline's
numerator), the bound it is reported against, and the rule that committed
ncu traffic is used only while the kernel sources still hash to the capture's.
No GPU: these are the formulas, checked against sums written out here.
"""
import json

import pytest

import bench
from synth import workloads as W

PEAKS = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
H, F = 2688, 1856


def entry(cfg, touched, up_ms, down_ms, workload):
    return bench.roofline_entry(W.WORKLOADS[cfg], {"up_gemm": up_ms, "down_gemm": down_ms}, touched, PEAKS,
                                "measured", workload)


def test_decode_bf16_bytes_and_hbm_bound():
    r = entry(1, 121, 0.2, 0.1, "decode")
    rows = 64 * 6
    assert r["kernel"] == "up_gemm" and r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["algorithmic_bytes_per_launch"] == 121 * F * H * 2 + rows * H * 2 + rows * F * 2
    assert r["algorithmic_flops_per_launch"] == 2.0 * rows * F * H
    assert r["achieved"] == pytest.approx(r["algorithmic_bytes_per_launch"] / 0.2e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / PEAKS["hbm_gbs"])


def test_down_projection_is_picked_when_slower():
    r = entry(1, 121, 0.1, 0.2, "decode")
    rows = 64 * 6
    assert r["kernel"] == "down_gemm"
    assert r["algorithmic_bytes_per_launch"] == 121 * F * H * 2 + rows * F * 2 + rows * H * 2


def test_shared_expert_adds_one_expert_of_weights_and_T_rows():
    base = entry(1, 121, 0.2, 0.1, "decode")
    sh = entry(7, 121, 0.2, 0.1, "decode_shared")
    assert sh["algorithmic_bytes_per_launch"] - base["algorithmic_bytes_per_launch"] == F * H * 2 + 64 * (H + F) * 2
    assert sh["algorithmic_flops_per_launch"] == 2.0 * 64 * 7 * F * H


def test_nvfp4_bytes_count_half_byte_codes_and_padded_block_scales():
    r = entry(5, 121, 0.3, 0.2, "decode_nvfp4")
    rows = 64 * 6
    ksp_h, ksp_f = 176, 128          # 2688/16 = 168 -> 176;  1856/16 = 116 -> 128
    assert r["algorithmic_bytes_per_launch"] == (121 * F * (H // 2 + ksp_h) + rows * (H // 2 + ksp_h)
                                                 + rows * (F // 2 + ksp_f))


def test_nvfp4_prefill_takes_the_fp4_tensor_peak():
    """A contraction is reported against its own dtype's peak: for NVFP4 the measured bf16 burst
    peak times the nominal fp4/bf16 ratio of 4."""
    r = entry(6, 128, 0.2, 0.19, "prefill_nvfp4")
    assert r["bound"] == "tensor" and r["peak"] == pytest.approx(4 * PEAKS["bf16_tflops"])
    assert r["frac"] == pytest.approx(r["achieved"] / (4 * PEAKS["bf16_tflops"]))
    assert "x 4" in r["peak_source"]


def test_fp8_b128_bytes_count_padded_codes_and_block_scales():
    up = entry(9, 121, 0.2, 0.1, "decode_fp8_b128")
    rows = 64 * 6
    assert up["bound"] == "hbm"
    assert up["algorithmic_bytes_per_launch"] == 121 * F * (2688 + 21 * 4) + rows * H + rows * F
    down = entry(10, 128, 0.2, 0.3, "prefill_fp8_b128")
    rows = 4096 * 6
    assert down["bound"] == "tensor" and down["peak"] == 2 * PEAKS["bf16_tflops"]
    assert down["algorithmic_bytes_per_launch"] == 128 * H * (1920 + 15 * 4) + rows * F + rows * H * 2


def test_prefill_is_reported_against_the_burst_tensor_peak():
    """The GEMM is timed launch by launch inside steps of well under a second: the burst peak
    applies; the fraction of the sustained peak is reported beside it."""
    r = entry(2, 128, 0.3, 0.31, "prefill")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["kernel"] == "down_gemm"
    assert r["achieved"] == pytest.approx(2.0 * 4096 * 6 * F * H / 0.31e-3 / 1e12)
    assert r["peak"] == PEAKS["bf16_tflops"]
    assert r["tensor_frac_of_sustained"] == pytest.approx(r["achieved"] / PEAKS["bf16_tflops_sustained"])
    fp8 = entry(4, 128, 0.3, 0.31, "chain")
    assert fp8["peak"] == 2 * PEAKS["bf16_tflops"]      # no probe: fp8 dense = 2x bf16 (nominal ratio)
    probed = dict(PEAKS, fp8_tflops=3000.0, fp8_source="probe")
    fp8 = bench.roofline_entry(W.WORKLOADS[4], {"up_gemm": 0.3, "down_gemm": 0.31}, 128, probed, "measured", "chain")
    assert fp8["peak"] == 3000.0 and fp8["peak_source"] == "probe"


def test_traffic_is_used_only_while_the_sources_match(tmp_path, monkeypatch):
    csrc = tmp_path / "routed_expert_moe_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cu").write_text("kernel v1")
    (tmp_path / "profiles").mkdir()
    import hashlib
    sha = hashlib.sha256(b"kernel v1").hexdigest()
    (csrc / "b.cu").write_text("another kernel")
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"up_gemm@decode": {"dram_bytes_per_launch": 1234, "source_sha256": sha,
                            "sources": ["routed_expert_moe_b200/csrc/a.cu"]}}))
    monkeypatch.setattr(bench, "ROOT", tmp_path)
    assert bench.traffic_from_profile("up_gemm", "decode") == 1234
    assert bench.traffic_from_profile("down_gemm", "decode") is None
    (csrc / "b.cu").write_text("a file the captured kernel does not use")
    assert bench.traffic_from_profile("up_gemm", "decode") == 1234
    (csrc / "a.cu").write_text("kernel v2")
    assert bench.traffic_from_profile("up_gemm", "decode") is None


def test_one_launch_ffn_counts_both_projections():
    """With both projections in one launch, the dominant kernel is that launch: the weight bytes
    of both banks of the touched experts, the activations in and out of both, twice the flops."""
    st = bench.stage_view({"up_gemm": 0.4, "down_gemm": 0.001, "combine": 0.01}, True)
    assert set(st) == {"expert_ffn", "combine"} and st["expert_ffn"] == pytest.approx(0.401)
    r = bench.roofline_entry(W.WORKLOADS[1], st, 121, PEAKS, "measured", "decode")
    rows = 64 * 6
    assert r["bound"] == "hbm" and r["kernel"].startswith("expert_ffn")
    assert r["algorithmic_bytes_per_launch"] == 2 * 121 * F * H * 2 + rows * (H + F) * 2 + rows * (F + H) * 2
    assert r["algorithmic_flops_per_launch"] == 2 * 2.0 * rows * F * H
    assert bench.stage_view({"up_gemm": 1.0, "down_gemm": 2.0}, False) == {"up_gemm": 1.0, "down_gemm": 2.0}


def _line(sm, reasons_active):
    flags = ["Active" if r else "Not Active" for r in reasons_active]
    return ", ".join([str(sm), "1965", "700.0", "0x0"] + flags)


def test_clock_summary_keeps_the_timed_window():
    """Only samples taken between the timed region's start and end count: idle samples before
    the loop (a low clock) must not pull the median down, nor their reasons leak in."""
    s = bench.ClockSampler(None)
    s.lines = [(0.0, _line(345, [0, 0, 0, 0])), (1.0, _line(1965, [0, 0, 0, 1])),
               (2.0, _line(1950, [0, 0, 0, 0])), (3.0, _line(900, [1, 0, 0, 0]))]
    s.window(0.5, 2.5)
    c = s.summary()
    assert c["samples"] == 2 and c["sm_mhz"] == pytest.approx(1957.5) and c["reasons"] == ["sw_power_cap"]
    s.window(2.9, 2.95)      # shorter than the sampling period: the sample nearest its middle
    c = s.summary()
    assert c["samples"] == 1 and c["sm_mhz"] == 900 and c["reasons"] == ["hw_slowdown"]


def test_clock_sampler_reads_nvml_every_few_milliseconds():
    import time

    class FakeNvml:
        NVML_CLOCK_SM = 1
        nvmlClocksEventReasonHwSlowdown = 0x8
        nvmlClocksEventReasonHwThermalSlowdown = 0x40
        nvmlClocksEventReasonSwThermalSlowdown = 0x20
        nvmlClocksEventReasonSwPowerCap = 0x4

        def nvmlInit(self): pass
        def nvmlShutdown(self): pass
        def nvmlDeviceGetHandleByUUID(self, u): return u
        def nvmlDeviceGetHandleByIndex(self, i): return i
        def nvmlDeviceGetClockInfo(self, h, c): return 1965
        def nvmlDeviceGetMaxClockInfo(self, h, c): return 1965
        def nvmlDeviceGetPowerUsage(self, h): return 950000
        def nvmlDeviceGetCurrentClocksEventReasons(self, h): return 0x4

    s = bench.ClockSampler("GPU-0", nvml=FakeNvml())
    s.start()
    t0 = time.perf_counter()
    time.sleep(0.05)
    s.window(t0, time.perf_counter())
    c = s.stop()
    assert c["sampler"].startswith("nvml") and c["samples"] >= 5
    assert c["sm_mhz"] == 1965 and c["reasons"] == ["sw_power_cap"]


def test_one_launch_nvfp4_ffn_counts_both_banks_codes_and_scales():
    """The one-launch NVFP4 FFN moves both banks (half a byte per value plus padded block scales),
    x's codes in, H's codes out and back in, and bf16 Y out; its flops go against the fp4 peak."""
    st = {"expert_ffn": 0.2, "combine": 0.01}
    r = bench.roofline_entry(W.WORKLOADS[5], st, 121, PEAKS, "measured", "decode_nvfp4")
    rows = 64 * 6
    ksp_h, ksp_f = 176, 128
    assert r["bound"] == "hbm" and r["kernel"].startswith("expert_ffn")
    assert r["algorithmic_bytes_per_launch"] == (121 * F * (H // 2 + ksp_h) + 121 * H * (F // 2 + ksp_f)
                                                 + rows * (H // 2 + ksp_h) + 2 * rows * (F // 2 + ksp_f)
                                                 + rows * H * 2)
    p = bench.roofline_entry(W.WORKLOADS[6], st, 128, PEAKS, "measured", "prefill_nvfp4")
    assert p["bound"] == "tensor" and p["peak"] == pytest.approx(4 * PEAKS["bf16_tflops"])


def test_one_launch_fp8_b128_ffn_counts_padded_codes_and_block_scales():
    st = {"expert_ffn": 0.2}
    r = bench.roofline_entry(W.WORKLOADS[9], st, 121, PEAKS, "measured", "decode_fp8_b128")
    rows = 64 * 6
    assert r["bound"] == "hbm"
    assert r["algorithmic_bytes_per_launch"] == (121 * F * (2688 + 21 * 4) + 121 * H * (1920 + 15 * 4)
                                                 + rows * H + 2 * rows * F + rows * H * 2)
    p = bench.roofline_entry(W.WORKLOADS[10], st, 128, PEAKS, "measured", "prefill_fp8_b128")
    assert p["bound"] == "tensor" and p["peak"] == 2 * PEAKS["bf16_tflops"]


def test_one_launch_ffn_with_a_shared_expert_counts_its_chunks():
    """With a shared expert of Fs = F the one-launch FFN also streams that expert's weights (one
    more 'touched' expert) and T more rows through both projections."""
    st = {"expert_ffn": 0.4}
    base = bench.roofline_entry(W.WORKLOADS[1], st, 121, PEAKS, "measured", "decode")
    sh = bench.roofline_entry(W.WORKLOADS[7], st, 121, PEAKS, "measured", "decode_shared")
    assert sh["algorithmic_bytes_per_launch"] - base["algorithmic_bytes_per_launch"] == 2 * F * H * 2 + 64 * (H + F) * 2 * 2
    assert sh["algorithmic_flops_per_launch"] == 4.0 * 64 * 7 * F * H


def test_hbm_roofline_names_the_routers_l2_prefetch():
    """At decode the router's spare clusters prefetch a bf16 up bank's first 48 MiB into L2
    before the FFN launch (the whole bank when it is smaller); NVFP4 and FP8_B128 banks are not
    prefetched, nor is anything for a batch whose router clusters fill the device."""
    st = {"expert_ffn": 0.35}
    r = bench.roofline_entry(W.WORKLOADS[1], st, 121, PEAKS, "measured", "decode")
    assert r["l2_warm_bytes_before_launch"] == 48 << 20
    f = bench.roofline_entry(W.WORKLOADS[5], st, 121, PEAKS, "measured", "decode_nvfp4")
    assert f["l2_warm_bytes_before_launch"] == 0                 # NVFP4 bank: not prefetched
    b = bench.roofline_entry(W.WORKLOADS[9], st, 121, PEAKS, "measured", "decode_fp8_b128")
    assert b["l2_warm_bytes_before_launch"] == 0
    s = bench.roofline_entry(W.WORKLOADS[3], st, 128, PEAKS, "measured", "skewed")
    assert s["l2_warm_bytes_before_launch"] == 0                 # 72 clusters of 8 tokens: none spare
    t = bench.roofline_entry(W.WORKLOADS[0], st, 8, PEAKS, "measured", "tiny")
    assert t["l2_warm_bytes_before_launch"] == 8 * 128 * 256 * 2  # the whole bf16 bank
    e = bench.roofline_entry(W.Workload("t60", 60, 2688, 128, 6, 1856, seed=1), st, 121, PEAKS, "measured", "decode")
    assert e["l2_warm_bytes_before_launch"] == 0                 # 15 clusters of 4 tokens fill the device
