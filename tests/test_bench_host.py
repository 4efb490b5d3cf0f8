"""Host logic of bench.py's roofline fields on CPU: the DRAM traffic of a
kernel is reported only while the kernel's source is the one the ncu capture
was taken at (its SHA-256 prefix), scaled by the units a launch processes,
and null with a reason otherwise; the every-kernel table names existing
sources."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_reported_only_for_the_captured_source(monkeypatch):
    src = "mxfp4_expert_layers_b200/csrc/decode.cu"
    cur = bench.src_sha16(src)
    monkeypatch.setitem(bench.NCU_TRAFFIC, "decode_kernel",
                        {"bytes": 1000.0, "per": "layer", "src": src, "sha16": cur})
    t, note = bench.ncu_traffic("decode_kernel", 64)
    assert t == 64000.0 and cur in note
    monkeypatch.setitem(bench.NCU_TRAFFIC, "decode_kernel",
                        {"bytes": 1000.0, "per": "layer", "src": src, "sha16": "0" * 16})
    t, note = bench.ncu_traffic("decode_kernel", 64)
    assert t is None and "stale" in note
    monkeypatch.setitem(bench.NCU_TRAFFIC, "decode_kernel",
                        {"bytes": None, "per": "layer", "src": src, "sha16": None})
    t, note = bench.ncu_traffic("decode_kernel", 64)
    assert t is None and "no ncu capture" in note


def test_traffic_table_names_existing_sources():
    for name, entry in bench.NCU_TRAFFIC.items():
        assert os.path.exists(os.path.join(ROOT, entry["src"])), name
        assert entry["bytes"] is None or entry["bytes"] > 0, name
        assert entry["sha16"] is None or len(entry["sha16"]) == 16, name
