"""Host-side pieces of bench.py that need no GPU: the DRAM traffic figure
is taken from the committed ncu summary only while the raster sources hash
to the value recorded beside it."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_line_applies_only_to_matching_sources(tmp_path, monkeypatch):
    h = bench.raster_source_hash()
    assert len(h) == 16
    prof = tmp_path / "p.md"
    prof.write_text("text\n"
                    f"    traffic raster_bwd_hits_kernel bytes_per_launch=123.5 launches=4 source={h}\n"
                    "    traffic raster_fwd_kernel bytes_per_launch=77 launches=4 source=0000000000000000\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", "p.md")
    monkeypatch.setattr(bench, "raster_source_hash", lambda: h)
    assert bench.profiled_traffic("raster_bwd") == 123.5
    assert bench.profiled_traffic("raster_fwd") is None  # taken from other sources
    assert bench.profiled_traffic("preprocess") is None
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", "missing.md")
    assert bench.profiled_traffic("raster_bwd") is None


def test_committed_summary_lines_parse():
    # every traffic line of the committed summary has the three fields
    p = os.path.join(ROOT, bench.TRAFFIC_PROFILE)
    lines = [l.split() for l in open(p) if l.split()[:1] == ["traffic"]]
    assert lines
    for f in lines:
        kv = dict(t.split("=", 1) for t in f[2:])
        assert float(kv["bytes_per_launch"]) > 0 and int(kv["launches"]) > 0 and len(kv["source"]) == 16
