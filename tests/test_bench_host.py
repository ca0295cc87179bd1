"""Host-side logic of bench.py that needs no GPU: the roofline traffic lookup
from the committed ncu capture data and the peak table."""
import hashlib
import json
import os

import bench


def _hash():
    csrc = os.path.join(bench.ROOT, "block_sparse_attention_30_b200", "csrc")
    return hashlib.sha256(b"".join(open(os.path.join(csrc, f), "rb").read()
                                   for f in bench.FINE_SOURCES)).hexdigest()[:16]


def test_traffic_is_reported_only_for_the_profiled_sources(tmp_path):
    data = tmp_path / "traffic.json"
    data.write_text(json.dumps({"sources_sha256": _hash(), "bytes_per_launch": {"wan14b_480p": 123456}}))
    assert bench.profiled_traffic("wan14b_480p", str(data)) == 123456
    assert bench.profiled_traffic("wan1.3b_480p", str(data)) is None      # not captured
    data.write_text(json.dumps({"sources_sha256": "0" * 16, "bytes_per_launch": {"wan14b_480p": 123456}}))
    assert bench.profiled_traffic("wan14b_480p", str(data)) is None       # sources changed since
    assert bench.profiled_traffic("wan14b_480p", str(tmp_path / "missing.json")) is None
    assert bench.fine_sources_hash() == _hash()


def test_peaks_fall_back_when_the_measured_table_is_absent(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks["hbm_gbs"] > 0 and peaks["bf16_tflops"] > 0
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 1.0, "bf16_tflops": 2.0}')
    peaks, src = bench.load_peaks()
    assert src == "measured" and peaks["hbm_gbs"] == 1.0
