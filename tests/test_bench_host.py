"""Host-side parts of bench.py that need no GPU: the roofline denominators'
loader (MEASURED_PEAKS.json complete, partial, malformed or absent) and the
peak-source wording beside each fraction."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def peaks_from(tmp_path, monkeypatch, content):
    if content is not None:
        (tmp_path / "MEASURED_PEAKS.json").write_text(content)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return bench.load_peaks()


def test_absent_file_uses_the_fallback(tmp_path, monkeypatch):
    p = peaks_from(tmp_path, monkeypatch, None)
    assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0 and p["bf16_tflops"] == 1590.0
    assert bench.peak_source(p, "hbm_gbs", "copy").startswith("of fallback")


def test_complete_file_is_measured(tmp_path, monkeypatch):
    d = {"hbm_gbs": 6540.5, "bf16_tflops": 1684, "bf16_tflops_sustained": 1391, "sm_max_mhz": 1965, "extra": "x"}
    p = peaks_from(tmp_path, monkeypatch, json.dumps(d))
    assert p["source"] == "measured"
    assert (p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"]) == (6540.5, 1684.0, 1391.0)
    assert bench.peak_source(p, "bf16_tflops", "gemm").startswith("of measured")


def test_partial_or_invalid_fields_fall_back_one_by_one(tmp_path, monkeypatch):
    d = {"hbm_gbs": "fast", "bf16_tflops": 1684, "sm_max_mhz": -1, "bf16_tflops_sustained": True}
    p = peaks_from(tmp_path, monkeypatch, json.dumps(d))
    assert p["bf16_tflops"] == 1684.0 and p["hbm_gbs"] == 6650.0 and p["sm_max_mhz"] == 1965.0
    assert p["bf16_tflops_sustained"] == 1400.0           # a boolean is not a number here
    assert p["source"].startswith("measured: bf16_tflops")
    # without a sustained figure the burst one stands in for it
    p = peaks_from(tmp_path, monkeypatch, json.dumps({"bf16_tflops": 1684}))
    assert p["bf16_tflops_sustained"] == 1684.0


def test_malformed_file_uses_the_fallback(tmp_path, monkeypatch):
    assert peaks_from(tmp_path, monkeypatch, "{not json")["source"] == "fallback"
    assert peaks_from(tmp_path, monkeypatch, "[1, 2]")["source"] == "fallback"
