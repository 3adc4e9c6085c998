"""Host logic of the benchmark that needs no GPU: algorithmic bytes, the recorded
capture's scale, peak lookup and the clock-sample summary."""
import json

import bench


def test_decode_bytes_of_the_profiled_launch_equal_the_recorded_algorithmic_bytes():
    # 128 units (16 x 8) at 32758 tokens: 1023 records of 3200 B and 22 residual rows each,
    # plus 4 query rows (bf16) and 4 output rows (fp32) per unit
    assert bench.decode_bytes(32758, 128, 4, 3200) == 128 * (1023 * 3200 + 22 * 512 + 4 * 256 + 4 * 512)
    assert bench.decode_bytes(0, 3, 7, 3200) == 3 * (7 * 256 + 7 * 512)
    # the captured launch: the third append + decode step of --profile-decode --steps 3
    # --warmup 2, from 32768 - 15 cached tokens to 32756, plus each unit's new K and V row
    ctx = 32768 - 3 * (3 + 2) + 3
    assert bench.decode_bytes(ctx, 128, 4, 3200) + 128 * 2 * 2 * 128 * 2 == bench.DECODE_CAPTURE["algorithmic_bytes"]


def test_captured_traffic_scales_with_the_launch_or_is_withheld(monkeypatch):
    alg = bench.DECODE_CAPTURE["algorithmic_bytes"]
    t = bench.captured_traffic(2 * alg)
    if t is not None:   # the decode sources still hash to the captured ones
        assert t == 2 * bench.DECODE_CAPTURE["traffic_bytes"]
    monkeypatch.setitem(bench.DECODE_CAPTURE, "sources_sha256_16", "0" * 16)
    assert bench.captured_traffic(alg) is None


def test_measured_peaks_prefer_the_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6000.5}))
    assert bench.measured_peaks() == (6000.5, "measured")


def test_clock_summary_names_every_reason_seen_and_the_median_clock():
    c = bench.ClockSampler(0)
    assert c.summary() is None
    c.max_mhz = 1965
    c.samples = [(1965, 0x0), (1900, 0x4), (1800, 0x4 | 0x40), (1965, 0x0)]
    s = c.summary()
    assert s["sm_mhz"] == 1932.5 and s["sm_max_mhz"] == 1965 and s["samples"] == 4
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_whole_job_value_counts_every_rank():
    ms = 2.0
    assert bench.whole_job_tokens_per_s(1, 10, ms) * 4 == bench.whole_job_tokens_per_s(4, 10, ms)

