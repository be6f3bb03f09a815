"""Pins for the oracle's cull, scan, key emission, sort and tile ranges.

References: numpy sorts and cumulative sums, Python's stable sorted(), a
float64 distance, and a linear scan for ranges; the sort also on random
record sets drawn by hypothesis (repeated depths, invisible records,
one-tile images).
"""

import types

import numpy as np
import pytest

from differentiable_tile_rasterizer_b200 import synthetic as S
from tests._helpers import make_scene, simple_camera


def _emit_reference(rec, cam):
    keys, vals = [], []
    for i in range(rec["tiles"].shape[0]):
        if rec["tiles"][i] <= 0:
            continue
        d = int(np.float32(rec["xyzo"][i, 2]).view(np.uint32))
        x0, y0, x1, y1 = rec["rect"][i].astype(int)
        for ty in range(y0, y1):
            for tx in range(x0, x1):
                keys.append(((ty * cam.tiles_x + tx) << 32) | d)
                vals.append(i)
    order = sorted(range(len(keys)), key=lambda k: keys[k])  # stable
    return np.array([keys[k] for k in order], np.uint64), np.array([vals[k] for k in order], np.uint32)


@pytest.mark.parametrize("cfg", ["tiny", "ragged"])
def test_bin_sort_against_library_sort(orc, cfg):
    if cfg == "tiny":
        sc = S.make_config(0)
    else:
        sc = S.random_scene(300, 77, 45, sh_degree=1, seed=5)
    cam = sc.cameras[0]
    rec = orc.preprocess(sc, cam)
    b = orc.bin_sort(rec, cam)
    assert np.array_equal(b["offsets"], (np.cumsum(rec["tiles"]) - rec["tiles"]).astype(np.int32))
    keys, vals = _emit_reference(rec, cam)
    assert b["n_instances"] == keys.size
    assert np.array_equal(b["keys"], keys)
    assert np.array_equal(b["vals"], vals)
    TT = cam.tiles_x * cam.tiles_y
    tile_of = (keys >> np.uint64(32)).astype(np.int64)
    for t in range(TT):
        idx = np.nonzero(tile_of == t)[0]
        want = (idx[0], idx[-1] + 1) if idx.size else (0, 0)
        assert tuple(b["ranges"][t]) == want


def test_ties_keep_emission_order(orc):
    # Equal depths in one tile: order falls back to the Gaussian index.
    cam = simple_camera(32, 32, 40.0)
    N = 6
    means = np.zeros((3, N), np.float32)
    means[2] = 2.0
    sc = make_scene(means, np.full((3, N), -3.0), np.tile([[1], [0], [0], [0]], (1, N)),
                    np.zeros(N), np.ones((3, N)), 0, [cam])
    rec = orc.preprocess(sc, cam)
    b = orc.bin_sort(rec, cam)
    for t in range(4):
        s, e = b["ranges"][t]
        assert list(b["vals"][s:e]) == list(range(N))


def test_capacity_and_empty(orc):
    sc = S.make_config(0)
    cam = sc.cameras[0]
    rec = orc.preprocess(sc, cam)
    total = int(rec["tiles"].sum())
    b = orc.bin_sort(rec, cam, capacity=total - 1)
    assert b["rc"] == 2 and b["n_instances"] == total
    empty = {k: (np.zeros_like(v) if isinstance(v, np.ndarray) else v) for k, v in rec.items()}
    b = orc.bin_sort(empty, cam)
    assert b["n_instances"] == 0 and not b["ranges"].any()


def test_cull_against_numpy(orc):
    rng = np.random.default_rng(3)
    N = 20000
    means = rng.uniform(-100, 100, (3, N)).astype(np.float32)
    imp = rng.exponential(1.0, N).astype(np.float32)
    imp[:50] = imp[50]  # ties at various values
    cam = simple_camera()
    cam.campos = np.array([3.0, -2.0, 1.0], np.float32)
    for lod, q in [(80.0, 0.3), (0.0, 0.3), (80.0, 0.0), (0.0, 0.0), (1e-3, 0.9), (150.0, 0.999)]:
        sc = make_scene(means, np.zeros((3, N)), np.tile([[1], [0], [0], [0]], (1, N)), np.zeros(N),
                        np.zeros((3, N)), 0, [cam], importance=imp, lod_dist=lod, importance_q=q)
        out = orc.cull(sc, cam)
        keep = np.ones(N, bool)
        if lod > 0:
            d = np.linalg.norm(means.astype(np.float64) - cam.campos.astype(np.float64)[:, None], axis=0)
            keep_lod = d <= lod
            # the fp32 decision may differ from fp64 only right at the threshold
            d32 = (means - cam.campos[:, None]).astype(np.float32)
            s32 = ((d32[0] * d32[0]) + (d32[1] * d32[1])) + (d32[2] * d32[2])
            keep_lod32 = s32 <= np.float32(lod) * np.float32(lod)
            diff = keep_lod != keep_lod32
            assert np.all(np.abs(d[diff] - lod) < 1e-5 * lod)
            keep &= keep_lod32
        if q > 0:
            tau = np.sort(imp)[int(np.floor(np.float64(np.float32(q)) * N))]
            assert out["tau"] == tau
            keep &= imp >= tau
        assert np.array_equal(out["mask"].astype(bool), keep)
        assert np.array_equal(out["active_idx"], np.nonzero(keep)[0].astype(np.int32))
        assert out["n_active"] == keep.sum()


def _records_strategy():
    from hypothesis import strategies as st

    @st.composite
    def records(draw):
        W = draw(st.integers(1, 90))
        H = draw(st.integers(1, 70))
        TW, TH = (W + 15) // 16, (H + 15) // 16
        n = draw(st.integers(0, 30))
        depths = draw(st.lists(st.sampled_from([0.25, 0.5, 1.0, 1.0000001, 3.0, 7.5]), min_size=n, max_size=n))
        xyzo = np.zeros((n, 4), np.float32)
        rect = np.zeros((n, 4), np.uint16)
        tiles = np.zeros(n, np.int32)
        for i in range(n):
            xyzo[i, 2] = depths[i]
            if draw(st.booleans()):  # visible: a non-empty rect inside the grid
                x0 = draw(st.integers(0, TW - 1))
                x1 = draw(st.integers(x0 + 1, TW))
                y0 = draw(st.integers(0, TH - 1))
                y1 = draw(st.integers(y0 + 1, TH))
                rect[i] = (x0, y0, x1, y1)
                tiles[i] = (x1 - x0) * (y1 - y0)
        cam = types.SimpleNamespace(width=W, height=H, tiles_x=TW, tiles_y=TH)
        return {"xyzo": xyzo, "rect": rect, "tiles": tiles}, cam

    return records()


def test_bin_sort_properties_on_random_records(orc):
    # random rects, repeated depths, invisible records and one-tile images:
    # the sort equals Python's stable sort of the emitted keys, the ranges
    # are the runs of each tile, and the offsets the exclusive scan
    from hypothesis import given, settings

    @settings(max_examples=80, deadline=None)
    @given(_records_strategy())
    def check(rc):
        rec, cam = rc
        b = orc.bin_sort(rec, cam)
        assert b["rc"] == 0
        assert np.array_equal(b["offsets"], (np.cumsum(rec["tiles"]) - rec["tiles"]).astype(np.int32))
        keys, vals = _emit_reference(rec, cam)
        assert b["n_instances"] == keys.size
        assert np.array_equal(b["keys"], keys)
        assert np.array_equal(b["vals"], vals)
        tile_of = (keys >> np.uint64(32)).astype(np.int64)
        for t in range(cam.tiles_x * cam.tiles_y):
            idx = np.nonzero(tile_of == t)[0]
            assert tuple(b["ranges"][t]) == ((idx[0], idx[-1] + 1) if idx.size else (0, 0))

    check()


def test_cull_quantile_on_random_weights(orc):
    # sizes, quantiles and tie-heavy non-negative weights drawn by
    # hypothesis: tau is numpy's value of rank floor(q N), the mask keeps
    # w >= tau, and the active list is the kept indices in order
    from hypothesis import given, settings
    from hypothesis import strategies as st

    cam = simple_camera()
    cam.campos = np.array([0.5, -1.0, 2.0], np.float32)

    @settings(max_examples=40, deadline=None)
    @given(st.integers(1, 3000), st.floats(0.001, 0.999), st.integers(1, 50), st.integers(0, 2 ** 16))
    def check(N, q, n_values, seed):
        rng = np.random.default_rng(seed)
        imp = rng.choice(rng.exponential(1.0, n_values).astype(np.float32), N)  # many ties
        means = rng.uniform(-5, 5, (3, N)).astype(np.float32)
        sc = make_scene(means, np.zeros((3, N)), np.tile([[1], [0], [0], [0]], (1, N)), np.zeros(N),
                        np.zeros((3, N)), 0, [cam], importance=imp, lod_dist=0.0, importance_q=q)
        out = orc.cull(sc, cam)
        tau = np.sort(imp)[int(np.floor(np.float64(np.float32(q)) * N))]
        assert out["tau"] == tau
        keep = imp >= tau
        assert np.array_equal(out["mask"].astype(bool), keep)
        assert np.array_equal(out["active_idx"], np.nonzero(keep)[0].astype(np.int32))
        assert out["n_active"] == keep.sum()

    check()
