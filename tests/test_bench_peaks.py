"""bench.py's roofline denominators: the measured peaks file when present, the fallback figures
otherwise, entry by entry, with the basis reported."""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))

import bench  # noqa: E402


def _load(monkeypatch, tmp_path, content):
    p = tmp_path / "peaks.json"
    if content is not None:
        p.write_text(content)
    monkeypatch.setattr(bench, "PEAKS_FILE", str(p))
    return bench.load_peaks()


def test_measured_file_is_used(monkeypatch, tmp_path):
    peaks, kind = _load(monkeypatch, tmp_path, json.dumps({"hbm_gbs": 6542.1, "bf16_tflops": 1671.6,
                                                            "bf16_tflops_sustained": 1407.4, "sm_mhz": 1350}))
    assert kind == "measured"
    assert peaks == {"hbm_gbs": 6542.1, "bf16_tflops": 1671.6, "bf16_tflops_sustained": 1407.4}


def test_missing_or_malformed_entries_fall_back_alone(monkeypatch, tmp_path):
    peaks, kind = _load(monkeypatch, tmp_path, json.dumps({"hbm_gbs": 6542.1, "bf16_tflops": "n/a"}))
    assert peaks["hbm_gbs"] == 6542.1 and peaks["bf16_tflops"] == 1590.0 and "fallback" in kind


def test_absent_or_unreadable_file_gives_the_fallback(monkeypatch, tmp_path):
    for content in (None, "not json", "[1, 2]"):
        peaks, kind = _load(monkeypatch, tmp_path, content)
        assert peaks["hbm_gbs"] == 6650.0 and peaks["bf16_tflops"] == 1590.0 and "fallback" in kind
