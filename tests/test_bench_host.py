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


def test_traffic_record_is_keyed_to_every_kernel_source():
    # the record follows every source the prefill attention kernel compiles from
    t = bench.TRAFFIC["prefill_attention"]
    assert set(t["sources"]) >= {"common.cuh", "prefill_tc.cuh", "prefill_tc2.cuh", "rope_loads.cuh"}


def test_roof_entry_reports_what_it_timed():
    r = bench.roof("tensor", 826.1, 1652.2, "TFLOP/s", "chunked prefill", "whole call", "measured")
    assert r["frac"] == 0.5 and r["bound"] == "tensor" and r["traffic"] is None
    assert r["peak_kind"] == "measured bf16 dense burst" and r["scope"] == "whole call"
    h = bench.roof("hbm", 3274.1, 6548.2, "GB/s", "paged decode", "whole step", "fallback", extra=1)
    assert h["frac"] == 0.5 and h["peak_kind"] == "fallback HBM copy" and h["extra"] == 1


def test_nvtx_range_is_a_no_op_without_nvtx():
    import types
    import torch
    with bench.nvtx_range(torch, "phase"):  # real NVTX (a host-side marker) where torch has it
        pass

    class NoNvtx:
        cuda = types.SimpleNamespace()  # no .nvtx attribute

    with bench.nvtx_range(NoNvtx, "phase") as r:
        assert r.on is False
