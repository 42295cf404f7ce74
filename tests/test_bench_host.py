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


def test_l2_statement_follows_the_working_set():
    from activation_perturbation_es_b200 import inputs as I
    assert bench.l2_statement(I.SCALED, I.SCALED.K).startswith("inputs larger than L2")
    assert bench.l2_statement(I.HEAD_PAGES, 64).startswith("inputs larger than L2")
    assert bench.l2_statement(I.HEAD_SMALL, 16).startswith("inputs smaller than L2")
    # the scaled step streams about 11 GB: the costs and rewards of both hidden layers dominate
    assert 10e9 < bench.step_bytes(I.SCALED, I.SCALED.K) < 13e9


def test_reference_arm_names_the_same_workload_config():
    """The reference arm's line carries the library arm's config object, so the
    two lines compare as the same configuration."""
    import subprocess
    from activation_perturbation_es_b200 import inputs as I
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "head_small_fp32", "--steps", "1", "--warmup", "1"], cwd=ROOT, capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads([ln for ln in out.stdout.splitlines() if ln.startswith("{")][-1])
    assert line["impl"] == "reference"
    assert line["config"] == bench.workload_config(I.HEAD_SMALL, 16, 1, "sequences", False)
