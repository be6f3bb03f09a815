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


def test_executed_ops_line_applies_only_to_matching_sources(tmp_path, monkeypatch):
    h = "0123456789abcdef"
    prof = tmp_path / "p.md"
    prof.write_text(f"    fp32ops raster_bwd_hits_kernel ops_per_launch=4.5e9 launches=4 source={h}\n"
                    "    fp32ops raster_fwd_kernel ops_per_launch=3e9 launches=4 source=ffffffffffffffff\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", "p.md")
    monkeypatch.setattr(bench, "raster_source_hash", lambda: h)
    assert bench.profiled_exec_ops("raster_bwd") == 4.5e9
    assert bench.profiled_exec_ops("raster_fwd") is None


def test_step_roofline_sums_the_binding_bound_of_each_stage():
    from differentiable_tile_rasterizer_b200 import synthetic as S
    sc = S.random_scene(1000, 160, 96, sh_degree=3, seed=1)
    counts = [{"V": 900, "I": 5000, "E": 10 ** 9, "E_bwd": 2 * 10 ** 9, "B": 10 ** 8, "A": 1000, "culled": False}]
    w = bench.stage_work(sc, counts)
    P, TT = 160 * 96, 10 * 6
    assert w["preprocess"]["bytes"] == 1000 * (236 + 64)
    assert w["bin_sort"]["bytes"] == 16 * 1000 + 12 * 5000 + 8 * TT
    assert w["raster_fwd"]["ops"] == bench.OPS_EVAL * 10 ** 9 + bench.OPS_BLEND_FWD * 10 ** 8
    assert w["raster_bwd"]["bytes"] == 53 * 5000 + 20 * P + 48 * 900
    assert w["preprocess_bwd"]["bytes"] == 1000 * 236 + 900 * (236 + 48 + 16)
    assert "cull" not in w
    culled = bench.stage_work(sc, [dict(counts[0], A=400, culled=True)])
    assert culled["cull"]["bytes"] == 1000 * 25 + 4 * 400 and culled["preprocess"]["bytes"] == 400 * (236 + 64)
    stage_ms = {k: 2.0 for k in w}  # two steps of 1 ms per stage
    r = bench.step_roofline(w, stage_ms, ms_per_step=10.0, steps=2, bw_gbs=1000.0, peak_alu_t=10.0)
    want = 0.0
    for k, v in w.items():
        t = max(v["bytes"] / 1e12 * 1e3, v["ops"] / 1e13 * 1e3)
        want += t
        assert abs(r["stages"][k]["frac"] - t / 1.0) < 1e-12
    assert abs(r["frac"] - want / 10.0) < 1e-12
    assert r["stages"]["raster_bwd"]["bound"] == "alu" and r["stages"]["preprocess"]["bound"] == "hbm"


def test_step_roofline_of_the_multiview_step():
    # the per-Gaussian stages of a multi-view step read the parameters once
    from differentiable_tile_rasterizer_b200 import synthetic as S
    sc = S.random_scene(1000, 160, 96, sh_degree=3, seed=1)
    c = {"V": 900, "I": 5000, "E": 10 ** 9, "E_bwd": 2 * 10 ** 9, "B": 10 ** 8, "A": 1000, "culled": False}
    counts = [c, dict(c, V=700)]
    w = bench.stage_work(sc, counts, multiview=True)
    par = 236
    assert "preprocess" not in w and "preprocess_bwd" not in w
    assert w["preprocess_multiview"]["bytes"] == 1000 * (par + 64 * 2)
    assert w["preprocess_bwd_multiview"]["bytes"] == 2 * 1000 * par + (4 * 1000 + 64 * 900) + (4 * 1000 + 64 * 700)
    single = bench.stage_work(sc, counts)
    for k in ("bin_sort", "raster_fwd", "raster_bwd"):
        assert w[k] == single[k]
