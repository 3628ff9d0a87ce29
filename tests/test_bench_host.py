"""Host-side logic of bench.py (CPU): the DRAM traffic figure of the roofline is reported only
while the kernel sources match the hash the ncu capture was taken with."""
import copy
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_follows_the_source_hash():
    import hashlib
    t = bench.TRAFFIC["prefill_attention"]
    h = hashlib.sha256()
    for f in t["sources"]:
        with open(os.path.join(ROOT, "rope_context_extension_bifocal_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    want = t["bytes_per_launch"] if h.hexdigest() == t["sha256"] else None
    assert bench.measured_traffic("prefill_attention") == want


def test_traffic_null_once_the_kernel_changes(monkeypatch):
    changed = copy.deepcopy(bench.TRAFFIC)
    changed["prefill_attention"]["sha256"] = "0" * 64
    monkeypatch.setattr(bench, "TRAFFIC", changed)
    assert bench.measured_traffic("prefill_attention") is None
    assert bench.measured_traffic("no_such_kernel") is None


def test_peaks_fall_back_when_the_measured_file_is_absent(monkeypatch):
    monkeypatch.setattr(bench, "ROOT", "/nonexistent")
    peaks, kind = bench.load_peaks()
    assert kind == "fallback" and peaks["bf16_tflops"] > 0 and peaks["hbm_gbs"] > 0
