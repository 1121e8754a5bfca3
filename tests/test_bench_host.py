"""Host-side logic of bench.py that its JSON line depends on (no GPU needed).

* roofline.traffic is the committed ncu DRAM byte count only while the kernel source
  is the one it was captured on, and null otherwise;
* every traffic entry's source summary exists under profiles/;
* the ALU roofline of the MSE-searched Q4_K fit counts 92 FP32 operations per element
  against SMs x 128 FP32 lanes x the SM clock;
* the compact per-format summary (the line's last key) carries every workload, the
  one-call step where there is one, and the pack-only fractions.
"""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
bench = pytest.importorskip("bench")


def test_traffic_is_reported_only_for_the_captured_source(monkeypatch, tmp_path):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps({
        "k_x@wl": {"csrc_sha": "aaaa", "dram_bytes_per_launch": 123.0},
        "k_y@wl": {"csrc_sha": "bbbb", "dram_bytes_per_launch": 456.0}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "csrc_digest", lambda: "aaaa")
    assert bench.traffic_for("k_x", "wl") == 123.0
    assert bench.traffic_for("k_y", "wl") is None          # captured on another source
    assert bench.traffic_for("k_x", "other") is None       # no capture of that workload
    monkeypatch.setattr(bench, "csrc_digest", lambda: "cccc")
    assert bench.traffic_for("k_x", "wl") is None          # the kernel changed since


def test_committed_traffic_entries_name_existing_summaries():
    t = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    assert t
    shas = {e["csrc_sha"] for e in t.values()}
    assert len(shas) == 1                                  # one capture of one source
    for key, e in t.items():
        assert "@" in key and e["dram_bytes_per_launch"] > 0
        assert os.path.exists(os.path.join(ROOT, e["source"])), e["source"]


def test_mse_alu_roofline_counts():
    assert bench.MSE_OPS_PER_ELEM == 92
    assert bench.FP32_LANES_PER_SM == 128

    class Props:
        multi_processor_count = 148

    orig = bench.torch.cuda.get_device_properties
    bench.torch.cuda.get_device_properties = lambda dev: Props()
    try:
        tops, how = bench.fp32_peak_tops(None, 1965)
        assert tops == pytest.approx(148 * 128 * 1965e6 / 1e12)
        assert "148 SMs" in how
        tops2, how2 = bench.fp32_peak_tops(None, None)     # no NVML clock: the recipe's 1965
        assert tops2 == pytest.approx(tops) and "1965 MHz" in how2
    finally:
        bench.torch.cuda.get_device_properties = orig


def test_format_summary_carries_every_workload_and_the_pack_only_fractions():
    peak = 6532.9
    result = {"value": 6160.0, "n_gpus": 1, "ms_per_step": 0.1357,
              "roofline": {"bound": "hbm", "frac": 0.984, "launch_us": 130.1},
              "pack_only": {"us": 80.0, "GB/s": 5000.0, "frac_of_hbm_peak": 0.7654321},
              "per_format": {
                  "nvfp4_tied": {"format": "nvfp4", "fused_us": 98.3, "fused_frac_of_hbm_peak": 1.013,
                                 "step_us": 145.4, "step_GB/s": 6436.0, "one_call_step_us": 141.4,
                                 "one_call_step_GB/s": 6619.6,
                                 "pack_only": {"frac_of_hbm_peak": 0.8123456}},
                  "q4k_mse": {"format": "q4k_mse", "fused_us": 414.0, "fused_frac_of_hbm_peak": 0.198,
                              "fused_GB/s": 1295.0, "alu_bound": {"frac": 0.7021}}}}
    out = bench.format_summary("w4a4", result, peak)
    assert out["cols"] == ["fused_us", "fused_frac", "step_us", "step_frac"]
    assert set(out) >= {"w4a4", "nvfp4_tied", "q4k_mse", "pack_only_frac", "q4k_mse_alu_frac"}
    # the one-call step is the step reported for a workload that has one
    r = bench._r                                   # three significant digits
    assert out["nvfp4_tied"] == [98.3, 1.01, 141.0, r(6619.6 / peak)]
    assert out["w4a4"] == [r(130.1), r(0.984), 136.0, r(6160.0 / peak)]
    assert out["pack_only_frac"] == {"w4a4": 0.765, "nvfp4_tied": 0.812}
    assert out["q4k_mse_alu_frac"] == 0.702
