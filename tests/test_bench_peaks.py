"""The roofline denominators bench.py reads from the measured-peaks file (CPU only): the flat form,
values given as objects, and files it cannot use, which fall back to the recipe's figures instead
of stopping the benchmark."""

import json

import bench


def _write(tmp_path, obj):
    p = tmp_path / "peaks.json"
    p.write_text(obj if isinstance(obj, str) else json.dumps(obj))
    return str(p)


def test_flat_values(tmp_path):
    p = _write(tmp_path, {"hbm_gbs": 7012.5, "bf16_tflops": 1612.0, "bf16_tflops_sustained": 1398.0, "clocks": {}})
    assert bench._peaks(p) == (7012.5, 1612.0, 1398.0, "measured")


def test_values_as_objects(tmp_path):
    p = _write(tmp_path, {"hbm_gbs": {"value": 7000}, "bf16_tflops": {"value": 1600.5},
                          "bf16_tflops_sustained": 1400})
    assert bench._peaks(p) == (7000.0, 1600.5, 1400.0, "measured")


def test_unusable_files_fall_back(tmp_path):
    for bad in ("{not json", {"hbm_gbs": 7000}, {"hbm_gbs": "n/a", "bf16_tflops": 1, "bf16_tflops_sustained": 1},
                {"hbm_gbs": 0, "bf16_tflops": 1600, "bf16_tflops_sustained": 1400}, [1, 2, 3]):
        assert bench._peaks(_write(tmp_path, bad)) == (*bench.FALLBACK_PEAKS, "fallback")


def test_missing_file_falls_back(tmp_path):
    assert bench._peaks(str(tmp_path / "absent.json")) == (*bench.FALLBACK_PEAKS, "fallback")
