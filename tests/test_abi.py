"""The C-ABI library builds for sm_100a, loads without a GPU and exports every
entry point that include/gs.h declares (no compute calls here)."""

import ctypes
import os
import re
import subprocess

import pytest

from differentiable_tile_rasterizer_b200 import _build, gs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "gs.h")).read()
    return sorted(set(re.findall(r"GS_API\s+[\w\s\*]+?\b(gs_\w+)\s*\(", text)))


def test_header_declares_the_five_stages():
    names = _declared()
    for n in ["gs_cull", "gs_preprocess", "gs_bin_sort", "gs_rasterize_fwd", "gs_rasterize_bwd",
              "gs_status_string"]:
        assert n in names
    assert set(names) == set(gs.EXPORTED)


def test_library_exports_every_declared_symbol():
    path = _build.build()
    lib = ctypes.CDLL(path)
    for n in _declared():
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT\s+(gs_\w+)", out))
    assert set(_declared()) <= exported
    # nothing else with the public prefix leaks out
    assert exported == set(_declared())


def test_status_strings_and_version():
    L = gs.load()
    assert gs.version() == 1
    assert L.gs_status_string(0) == b"ok"
    assert L.gs_status_string(4).startswith(b"bounded")


def test_workspace_queries_need_no_gpu():
    cam = gs.GsCamera()
    cam.width, cam.height = 1920, 1080
    assert gs.gs_cull_workspace(1_000_000, cam) > 0
    small = gs.gs_bin_sort_workspace(1000, cam, 10_000)
    big = gs.gs_bin_sort_workspace(1000, cam, 10_000_000)
    assert big > small > 12 * 10_000
    cam.width = 0
    with pytest.raises(gs.GsError):
        gs.gs_cull_workspace(10, cam)


def test_tile_order_argument_checks_need_no_gpu():
    L = gs.load()
    assert L.gs_tile_order(None, -1, None, None) == gs.GS_ERR_INVALID_ARGUMENT
    assert L.gs_tile_order(None, 10, None, None) == gs.GS_ERR_INVALID_ARGUMENT
    assert L.gs_tile_order(None, 1 << 31, None, None) == gs.GS_ERR_INVALID_ARGUMENT


def test_multiview_backward_argument_checks_need_no_gpu():
    L = gs.load()
    cams = (gs.GsCamera * 17)()
    recs = (gs.GsProjected * 17)()
    g2d = (ctypes.c_void_p * 17)()
    args = lambda deg, nv: (None, None, None, None, None, deg, 0, ctypes.cast(cams, ctypes.c_void_p), nv,
                            ctypes.cast(recs, ctypes.c_void_p), ctypes.cast(g2d, ctypes.c_void_p),
                            None, None, None, None, None, None)
    assert L.gs_preprocess_bwd_multiview(*args(3, 0)) == gs.GS_ERR_INVALID_ARGUMENT   # no view
    assert L.gs_preprocess_bwd_multiview(*args(3, 17)) == gs.GS_ERR_INVALID_ARGUMENT  # past GS_MAX_VIEWS
    assert L.gs_preprocess_bwd_multiview(*args(-1, 2)) == gs.GS_ERR_INVALID_ARGUMENT
    assert L.gs_preprocess_bwd_multiview(*args(4, 2)) == gs.GS_ERR_UNSUPPORTED       # SH degree > 3
    with pytest.raises(ValueError):  # one record set and one 2-D gradient per camera, checked first
        gs.gs_preprocess_bwd_multiview(None, None, None, None, None, 3, 0, [gs.GsCamera()], [], [],
                                       None, None, None, None, None)


@pytest.mark.parametrize("lang,std", [("c", "c99"), ("c++", "c++17")])
def test_header_is_plain_c_and_cxx(lang, std):
    # the boundary is a C ABI: the header compiles as strict C99 and as C++
    cc = "gcc" if lang == "c" else "g++"
    r = subprocess.run([cc, "-fsyntax-only", f"-std={std}", "-Wall", "-Wextra", "-pedantic", "-Werror", "-x", lang,
                        os.path.join(ROOT, "include", "gs.h")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
