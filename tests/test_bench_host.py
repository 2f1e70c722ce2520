"""Host logic of bench.py on CPU: the work account of the replay, the clock
record, the traffic record's staleness rule and the peak source."""
import io
import json
import os

import pytest

import bench
import synthetic

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_replay_work_account_closed_forms():
    """One 8-step replay: 24 blocks x {qkv, out, up, down} at d = 1536, M = 432."""
    acc = bench.step_account()
    params = 1536 * 4608 + 1536 * 1536 + 1536 * 6144 + 6144 * 1536   # weights per block
    ops = 8 * 24 * 2 * 432 * params
    for k in ("q8", "q4", "w8a8_gemm"):
        assert acc[k][0] == ops
    assert abs(ops / 1e12 - 4.6965) < 1e-3
    # bytes: packed weights + scales + fp16 X read + fp16 Y written (+ fp32 steering vector once)
    xy = sum(2 * 432 * k + 2 * 432 * n for _, k, n in bench.LINEARS)
    steer = 4 * 1536
    q8 = 24 * (params + sum(4 * n for _, k, n in bench.LINEARS) + xy) + steer
    q4 = 24 * (params // 2 + sum(2 * n * (k // 32) for _, k, n in bench.LINEARS) + xy) + steer
    assert acc["q8"][1] == 8 * q8
    assert acc["q4"][1] == 8 * q4
    w8 = 24 * (params + sum(432 * k + 4 * 432 + 4 * n + 2 * 432 * n for _, k, n in bench.LINEARS)) + steer
    assert acc["w8a8_gemm"][1] == 8 * w8
    assert acc["act_quant"][1] == 8 * 24 * sum(3 * 432 * k + 4 * 432 for _, k, _ in bench.LINEARS)
    # q4 footprint per parameter: 0.5 B codes + 2 B per group of 32
    n, k = 6144, 1536
    assert (bench.bytes_wo("q4", 0, n, k, False)) / (n * k) == 0.5625


def _sampler(lines, bus="00000000:1B:00.0"):
    s = bench.ClockSampler(bus)
    s.proc = object()                 # pretend the sampler ran
    s.out = io.StringIO("\n".join(lines) + "\n")
    return s


def test_clock_summary_median_under_load_and_reasons():
    row = "00000000:1B:00.0, {sm}, 1965, 700.5, 0x0, {hw}, Not Active, Not Active, {pc}"
    lines = [row.format(sm=210, hw="Not Active", pc="Not Active")]            # idle sample, ignored
    lines += [row.format(sm=s, hw="Not Active", pc="Active") for s in (1965, 1950, 1965)]
    lines += ["00000000:2C:00.0, 900, 1965, 100, 0x0, Active, Active, Active, Active"]  # another GPU
    lines += ["garbage line"]
    out = _sampler(lines).summary()
    assert out["sm_mhz"] == 1965 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]
    assert out["samples"] == 4


def test_clock_summary_flags_slowdown_and_unsampled():
    row = "00000000:1B:00.0, 1200, 1965, 900, 0x8, Active, Not Active, Not Active, Not Active"
    assert _sampler([row]).summary()["reasons"] == ["hw_slowdown"]
    assert _sampler([]).summary()["reasons"] == ["unsampled"]
    assert bench.ClockSampler(None).summary()["reasons"] == ["unsampled"]


def test_traffic_record_scaled_and_stale(monkeypatch):
    rec = json.load(open(os.path.join(ROOT, "profiles", "roofline_traffic.json")))
    assert set(rec["kernels"]) == {"qgemm_kernel<Q8>", "qgemm_kernel<Q4>", "qgemm_kernel<W8A8>"}
    k = rec["kernels"]["qgemm_kernel<Q4>"]
    monkeypatch.setattr(bench, "kernel_source_sha256", lambda: rec["source_sha256"])
    t, src = bench.measured_traffic("qgemm_kernel<Q4>", 2 * k["algorithmic_bytes"])
    assert t == pytest.approx(2 * k["dram_bytes"]) and "scaled" in src
    monkeypatch.setattr(bench, "kernel_source_sha256", lambda: "0" * 64)
    t, src = bench.measured_traffic("qgemm_kernel<Q4>", 1.0)
    assert t is None and src.startswith("stale")


def test_peaks_measured_or_fallback(monkeypatch, tmp_path):
    peaks, src = bench.load_peaks()
    assert set(peaks) == set(bench.FALLBACK_PEAKS) and all(v > 0 for v in peaks.values())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))   # no MEASURED_PEAKS.json there
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks == bench.FALLBACK_PEAKS


def test_per_config_cases_cover_every_configured_shape():
    """Every per-shape case of the benchmark configurations is timed: the tiny
    q8 case, q8 d=1024 at M in {1,16,432}, W8A8 d=1536 at M in {432,4096}
    with its activation quantisation, q4 d=1536 at M in {1,8,432}, plus the
    fp16 rung and the two packs."""
    cases = {(c, n, k, m) for _, c, _, n, k, m in bench.CONFIG_CASES}
    for _, k, n in synthetic.D1024:
        for m in (1, 16, 432):
            assert ("q8", n, k, m) in cases
    for _, k, n in synthetic.D1536:
        for m in (432, 4096):
            assert ("w8a8", n, k, m) in cases
        for m in (1, 8, 432):
            assert ("q4", n, k, m) in cases
        assert ("pack_q8", n, k, 0) in cases and ("pack_q4", n, k, 0) in cases
    for m in (432, 4096):
        for k in (1536, 6144):
            assert ("act_quant", 0, k, m) in cases
    assert ("q8", 256, 256, 64) in cases
    assert len(bench.CONFIG_CASES) == len(cases)          # no case timed twice


def test_case_targets_are_the_stated_bars():
    assert bench.case_target("q8", 1) == ("hbm_frac", 0.70)
    assert bench.case_target("q8", 16) == ("hbm_frac", 0.70)
    assert bench.case_target("q4", 8) == ("hbm_frac", 0.70)
    assert bench.case_target("w8a8", 4096) == ("tensor_frac", 0.60)
    assert bench.case_target("q8", 432) is None and bench.case_target("w8a8", 432) is None


def test_roof_entry_picks_the_binding_roof():
    R = bench.roofs({"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0})
    assert R == {"f16": 1600.0, "i8": 3200.0, "hbm": 6000.0}
    # weight-bound: 4 MB and 8 MFLOP in 1 us -> 4 TB/s, HBM-bound
    d = bench.roof_entry(8e6, 4e6, 1e-6, R["f16"], R["hbm"])
    assert d["bound"] == "hbm" and d["frac"] == pytest.approx(4000 / 6000)
    # compute-bound: 8 GFLOP, 10 MB in 10 us -> 800 TFLOP/s
    d = bench.roof_entry(8e9, 10e6, 10e-6, R["f16"], R["hbm"])
    assert d["bound"] == "tensor" and d["frac"] == pytest.approx(800 / 1600)
    d = bench.roof_entry(0.0, 3e6, 1e-6, R["f16"], R["hbm"])   # a quantiser: bytes only
    assert d["bound"] == "hbm" and "tops" not in d


def test_fp16_rung_account():
    acc = bench.step_account()
    params = 1536 * 4608 + 1536 * 1536 + 1536 * 6144 + 6144 * 1536
    assert acc["f16"][0] == acc["q8"][0]
    xy = sum(2 * 432 * k + 2 * 432 * n for _, k, n in bench.LINEARS)
    assert acc["f16"][1] == 8 * (24 * (2 * params + xy) + 4 * 1536)


def test_fused_w8a8_account():
    """The fused W8A8 leg counts the fp16 activations once, not the codes'
    round trip through the workspace."""
    acc = bench.step_account()
    assert acc["w8a8"][0] == acc["q8"][0]
    params = 1536 * 4608 + 1536 * 1536 + 1536 * 6144 + 6144 * 1536
    per_block = params + sum(2 * 432 * k + 4 * n + 2 * 432 * n for _, k, n in bench.LINEARS)
    assert acc["w8a8"][1] == 8 * (24 * per_block + 4 * 1536)
    assert bench.Replay.ORDER == ("q8", "act_quant", "w8a8_gemm", "q4")
    assert "w8a8_fused" in bench.Replay.EXTRA
