"""bench.py's DRAM-traffic figure: the ratio of measured to algorithmic bytes from
the committed ncu record, applied to the timed launch while the kernel source is
the one that was captured, and no figure (None) once the source has changed."""

import json
import os
import sys

sys.path.insert(0, os.path.join(os.path.dirname(__file__), ".."))
import bench  # noqa: E402


def _write(root, src_text, prefix):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    os.makedirs(os.path.join(root, "k"), exist_ok=True)
    with open(os.path.join(root, "k", "kernel.cu"), "w") as f:
        f.write(src_text)
    rec = {"gemm_layer": {"dram_bytes_per_launch_small": 1012, "algorithmic_bytes_small": 1000,
                          "source": "k/kernel.cu", "source_sha256_prefix": prefix, "capture": "x"}}
    with open(os.path.join(root, "profiles", "traffic.json"), "w") as f:
        json.dump(rec, f)


def test_traffic_scales_while_the_source_is_unchanged(tmp_path, monkeypatch):
    import hashlib
    text = "// kernel\n"
    _write(str(tmp_path), text, hashlib.sha256(text.encode()).hexdigest()[:16])
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert abs(bench.measured_traffic("gemm_layer", 5000.0) - 5060.0) < 1e-9
    assert bench.measured_traffic("attention", 5000.0) is None  # no record for that class


def test_no_traffic_once_the_source_changed(tmp_path, monkeypatch):
    _write(str(tmp_path), "// kernel, edited\n", "0123456789abcdef")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("gemm_layer", 5000.0) is None

