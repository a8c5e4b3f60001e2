"""Host-side arithmetic of bench.py's JSON line (CPU): the peaks it divides by
and which of the burst / sustained 8-bit denominators a run is put against."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_peaks_reads_the_measured_file(tmp_path):
    f = tmp_path / "MEASURED_PEAKS.json"
    f.write_text(json.dumps({"hbm_gbs": 6556.5, "bf16_tflops": 1638.7, "bf16_tflops_sustained": 1372.3}))
    pk = bench.peaks(str(f))
    assert pk == {"hbm_gbs": 6556.5, "bf16": 1638.7, "bf16_sustained": 1372.3, "source": "measured"}


@pytest.mark.parametrize("content", [None, "not json", json.dumps({"hbm_gbs": 1.0})])
def test_peaks_fall_back_when_the_file_is_missing_or_incomplete(tmp_path, content):
    f = tmp_path / "MEASURED_PEAKS.json"
    if content is not None:
        f.write_text(content)
    pk = bench.peaks(str(f))
    assert pk["source"] == "fallback" and pk["hbm_gbs"] == 6650.0 and pk["bf16"] == 1590.0


def test_a_short_timed_region_is_put_against_the_burst_peak():
    pk = {"hbm_gbs": 6556.5, "bf16": 1638.7, "bf16_sustained": 1372.3}
    peak, kind, burst, sustained = bench.gemm_peak(pk, 0.207)  # 20 steps of ~10 ms
    assert kind == "burst" and peak == burst == pytest.approx(3277.4) and sustained == pytest.approx(2744.6)
    # 2.1027e13 ops per step over 21 launches of 0.36357 ms: 2754 TOPS, 0.84 of the burst peak
    assert 2.1027e13 / (21 * 0.36357e-3) / 1e12 / peak == pytest.approx(0.84, abs=0.005)


def test_a_seconds_long_timed_region_is_put_against_the_sustained_peak():
    pk = {"hbm_gbs": 6556.5, "bf16": 1638.7, "bf16_sustained": 1372.3}
    peak, kind, _, sustained = bench.gemm_peak(pk, bench.SUSTAINED_REGION_S)
    assert kind == "sustained" and peak == sustained == pytest.approx(2744.6)
