"""CPU oracle for differentiable tile rasterization of 3D Gaussian splats.

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and the
benchmark's CPU-baseline leg, never by the product path. It wraps
`libgs_oracle.so` (built from gs_oracle.cpp with g++; no code is shared with
the CUDA library) through ctypes and numpy.

Every function here cites, in gs_oracle.cpp, the passage it follows. Parity is
pinned by tests/test_oracle_*.py against closed forms, invariants, library
routines (std/numpy sorts, scipy spherical harmonics, libm exp) and float64
finite differences.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gs_oracle.cpp")
_SO = os.path.join(_HERE, "libgs_oracle.so")
_LOCK = threading.Lock()
_LIB = None

CXXFLAGS = ["-O2", "-std=c++17", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
            "-fPIC", "-shared", "-Wall", "-Wno-unused-function"]


def build(force: bool = False) -> str:
    """Compile the oracle library in place (g++, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", *CXXFLAGS, "-o", tmp, _SRC])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _LIB
    with _LOCK:
        if _LIB is None:
            build()
            _LIB = ctypes.CDLL(_SO)
            _declare(_LIB)
    return _LIB


P = ctypes.c_void_p
I64 = ctypes.c_int64
I32 = ctypes.c_int
F32 = ctypes.c_float


def _declare(L):
    L.or_version.restype = ctypes.c_int
    L.or_constants.argtypes = [P]
    L.or_exp2_array.argtypes = [P, P, I64]
    L.or_sh_basis_f64.argtypes = [P, I64, P]
    L.or_sh_basis_f32.argtypes = [P, I64, P]
    L.or_sh_basis_grad_f64.argtypes = [P, I64, P]
    L.or_cull.argtypes = [P, P, I64, P, F32, F32, P, P, P, P]
    L.or_cull.restype = ctypes.c_int
    L.or_preprocess.argtypes = [P, P, P, P, P, I32, I64, P, I64, P, I32, I32, P, P, P, P, P, P]
    L.or_preprocess.restype = ctypes.c_int
    L.or_bin_sort.argtypes = [P, P, P, I64, I32, I32, P, P, P, I64, P, P]
    L.or_bin_sort.restype = ctypes.c_int
    L.or_raster_fwd.argtypes = [P, P, P, P, P, I32, I32, P, P, P, P, P, P, I64]
    L.or_raster_fwd.restype = ctypes.c_int
    L.or_raster_fwd_bruteforce.argtypes = [P, P, P, P, P, I64, I32, I32, P, P, P, P, P]
    L.or_importance.argtypes = [P, P, P, P, P, I32, I32, P, P]
    for f in ("or_log2_spec", "or_log1p_spec", "or_expm1_spec"):
        getattr(L, f).argtypes = [ctypes.c_float]
        getattr(L, f).restype = ctypes.c_float
    L.or_quant_encode.argtypes = [P, I64, I64, I32, P, P]
    L.or_quant_decode.argtypes = [P, P, I64, I64, I32, P]
    D = ctypes.c_double
    L.or_adam_sh_quant.argtypes = [P, I64, I64, P, P, P, P, P, P, D, D, D, D, D, I64]
    L.or_importance.restype = ctypes.c_int
    L.or_loss_frozen_f64.argtypes = [P, P, P, P, P, I32, I64, P, I64, P, I32, I32,
                                     P, P, P, P, P, P, P, P, P]
    L.or_loss_frozen_f64.restype = ctypes.c_double
    L.or_backward_f64.argtypes = [P, P, P, P, P, I32, I64, P, I64, P, I32, I32,
                                  P, P, P, P, P, P, P, P, P, P] + [P] * 10 + [P, I64, I32]
    L.or_num_threads.restype = ctypes.c_int
    L.or_preprocess_bwd_f64.argtypes = [P, P, P, P, P, I32, I64, P, I64, P, I32, I32,
                                        P, P, P] + [P] * 10
    L.or_project_f64.argtypes = [P, P, P, P, P, I32, I64, P, I32, I32, P, P, P]


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


# ------------------------------------------------------------------ helpers
def constants() -> dict:
    out = np.zeros(32, np.float32)
    lib().or_constants(_p(out))
    return {"exp2_taylor": out[0:8].copy(), "log2e": out[8], "kh": out[9], "kf": out[10],
            "alpha_min": out[11], "alpha_max": out[12], "t_min": out[13],
            "dilation": out[14], "sh": out[16:32].copy()}


def exp2(x) -> np.ndarray:
    x = _c(x, np.float32)
    y = np.empty_like(x)
    lib().or_exp2_array(_p(x), _p(y), x.size)
    return y


def sh_basis(dirs, dtype=np.float64) -> np.ndarray:
    d = _c(dirs, dtype).reshape(-1, 3)
    Y = np.empty((d.shape[0], 16), dtype)
    fn = lib().or_sh_basis_f64 if dtype == np.float64 else lib().or_sh_basis_f32
    fn(_p(d), d.shape[0], _p(Y))
    return Y


def sh_basis_grad(dirs) -> np.ndarray:
    d = _c(dirs, np.float64).reshape(-1, 3)
    G = np.empty((d.shape[0], 16, 3), np.float64)
    lib().or_sh_basis_grad_f64(_p(d), d.shape[0], _p(G))
    return G


def cam_array(cam) -> np.ndarray:
    """Camera as the 20-float vector the library takes: R(9) t(3) campos(3) fx fy cx cy near."""
    v = np.zeros(20, np.float32)
    v[0:9] = np.asarray(cam.R, np.float32).reshape(9)
    v[9:12] = cam.t
    v[12:15] = cam.campos
    v[15:20] = [cam.fx, cam.fy, cam.cx, cam.cy, cam.near_z]
    return v


# -------------------------------------------------------------------- stages
def cull(scene, cam):
    N = scene.N
    means = _c(scene.means, np.float32)
    imp = None if scene.importance is None else _c(scene.importance, np.float32)
    mask = np.zeros(N, np.uint8)
    act = np.zeros(max(N, 1), np.int32)
    na = np.zeros(1, np.int64)
    tau = np.zeros(1, np.float32)
    rc = lib().or_cull(_p(means), _p(imp), N, _p(_c(cam.campos, np.float32)),
                       float(scene.lod_dist), float(scene.importance_q), _p(mask), _p(act),
                       _p(na), _p(tau))
    if rc != 0:
        raise ValueError(f"or_cull rc={rc}")
    return {"mask": mask, "active_idx": act[:int(na[0])].copy(), "n_active": int(na[0]),
            "tau": float(tau[0])}


def preprocess(scene, cam, active_idx=None, n_active=None):
    N = scene.N
    n_active = N if n_active is None else int(n_active)
    act = None if active_idx is None else _c(active_idx, np.int32)
    xyzo = np.empty((N, 4), np.float32)
    conic = np.empty((N, 4), np.float32)
    rgb = np.empty((N, 4), np.float32)
    radius = np.empty(N, np.int32)
    rect = np.empty((N, 4), np.uint16)
    tiles = np.empty(N, np.int32)
    rc = lib().or_preprocess(_p(_c(scene.means, np.float32)), _p(_c(scene.log_scales, np.float32)),
                             _p(_c(scene.quats, np.float32)), _p(_c(scene.opacity_logits, np.float32)),
                             _p(_c(scene.sh, np.float32)), scene.sh_degree, N, _p(act), n_active,
                             _p(cam_array(cam)), cam.width, cam.height, _p(xyzo), _p(conic),
                             _p(rgb), _p(radius), _p(rect), _p(tiles))
    if rc != 0:
        raise ValueError(f"or_preprocess rc={rc}")
    return {"xyzo": xyzo, "conic": conic, "rgb": rgb, "radius": radius, "rect": rect,
            "tiles": tiles, "n_active": n_active, "active_idx": act}


def bin_sort(rec, cam, capacity=None):
    n = rec["tiles"].shape[0]
    total = int(rec["tiles"].astype(np.int64).sum())
    cap = total if capacity is None else int(capacity)
    TT = cam.tiles_x * cam.tiles_y
    offsets = np.empty(n, np.int32)
    keys = np.empty(max(cap, 1), np.uint64)
    vals = np.empty(max(cap, 1), np.uint32)
    ranges = np.empty(2 * TT, np.uint32)
    ni = np.zeros(1, np.int64)
    rc = lib().or_bin_sort(_p(rec["xyzo"]), _p(rec["rect"]), _p(rec["tiles"]), n, cam.width,
                           cam.height, _p(offsets), _p(keys), _p(vals), cap, _p(ranges), _p(ni))
    out = {"offsets": offsets, "n_instances": int(ni[0]), "rc": rc}
    if rc == 0:
        out.update(keys=keys[:total], vals=vals[:total], ranges=ranges.reshape(TT, 2))
    return out


def raster_fwd(rec, bins, cam, bg, tile_subset=None):
    W, H = cam.width, cam.height
    image = np.zeros((3, H, W), np.float32)
    T = np.zeros((H, W), np.float32)
    nc = np.zeros((H, W), np.int32)
    last = np.zeros((H, W), np.int32)
    sub = None if tile_subset is None else _c(tile_subset, np.int32)
    vals = bins["vals"] if bins["vals"].size else np.zeros(1, np.uint32)
    lib().or_raster_fwd(_p(rec["xyzo"]), _p(rec["conic"]), _p(rec["rgb"]), _p(vals),
                        _p(_c(bins["ranges"], np.uint32)), W, H, _p(_c(bg, np.float32)),
                        _p(image), _p(T), _p(nc), _p(last), _p(sub),
                        0 if sub is None else sub.size)
    return {"image": image, "final_T": T, "n_contrib": nc, "last": last}


def importance(rec, bins, cam, n_gaussians, out=None):
    """Cross-view visibility weights (BlitzGS write-up, section 2.2): adds this
    view's sum over pixels of alpha*T per Gaussian (fp32 spec values of the
    forward walk, summed in float64) to `out` (float64 [n_gaussians], zeros if
    not given) and returns it. Record i belongs to Gaussian rec["active_idx"][i]
    when the records come from a culled view, else to Gaussian i."""
    if out is None:
        out = np.zeros(n_gaussians, np.float64)
    assert out.dtype == np.float64 and out.shape == (n_gaussians,)
    act = rec.get("active_idx")
    act = None if act is None else _c(act, np.int32)
    vals = bins["vals"] if bins["vals"].size else np.zeros(1, np.uint32)
    lib().or_importance(_p(rec["xyzo"]), _p(rec["conic"]), _p(rec["rgb"]), _p(vals),
                        _p(_c(bins["ranges"], np.uint32)), cam.width, cam.height, _p(act), _p(out))
    return out


def grad2d_norm(grad2d, tiles, active_idx, n_gaussians, norm_sum=None, view_count=None):
    """Densification statistic of one view: for every visible record i
    (tiles[i] > 0), adds |(dpx, dpy)| = hypot of grad2d[i][0:2] to
    norm_sum[g] and 1 to view_count[g], g = active_idx[i] (or i). float64."""
    if norm_sum is None:
        norm_sum = np.zeros(n_gaussians, np.float64)
    if view_count is None:
        view_count = np.zeros(n_gaussians, np.int64)
    g2 = np.asarray(grad2d, np.float64).reshape(-1, 12)
    vis = np.flatnonzero(np.asarray(tiles) > 0)
    gid = vis if active_idx is None else np.asarray(active_idx)[vis]
    norm_sum[gid] += np.sqrt(g2[vis, 0] ** 2 + g2[vis, 1] ** 2)
    view_count[gid] += 1
    return norm_sum, view_count


# ---- quantised SH Adam (Spirula Studio page: 16-bit SH value codes, 8-bit
# log codes of the Adam moments, per-256-unit block bounds)
def log2_spec(y):
    return lib().or_log2_spec(float(y))


def log1p_spec(z):
    return lib().or_log1p_spec(float(z))


def expm1_spec(y):
    return lib().or_expm1_spec(float(y))


def quant_encode(x, bits):
    """Block codes of float32 planes x [U, N]: (codes uint32 [U, Npad], bounds
    float32 [U, nblk, 2]); blocks of 256 consecutive units of a plane."""
    x = _c(x, np.float32)
    U, N = x.shape
    nblk = (N + 255) // 256
    codes = np.zeros((U, nblk * 256), np.uint32)
    bounds = np.zeros((U, nblk, 2), np.float32)
    lib().or_quant_encode(_p(x), U, N, int(bits), _p(codes), _p(bounds))
    return codes, bounds


def quant_decode(codes, bounds, N, bits):
    U = codes.shape[0]
    x = np.zeros((U, N), np.float32)
    lib().or_quant_decode(_p(_c(codes, np.uint32)), _p(_c(bounds, np.float32)), U, N, int(bits), _p(x))
    return x


def adam_sh_quant(grad, state, lr, beta1, beta2, eps, scale, step):
    """One Adam step in place on state = {"pc","pb","mc","mb","vc","vb"}
    (value codes 16-bit, moment log codes 8-bit, as quant_encode lays them
    out); grad float32 [U, N]."""
    g = _c(grad, np.float32)
    U, N = g.shape
    for k in ("pc", "mc", "vc"):
        assert state[k].dtype == np.uint32 and state[k].flags.c_contiguous
    for k in ("pb", "mb", "vb"):
        assert state[k].dtype == np.float32 and state[k].flags.c_contiguous
    lib().or_adam_sh_quant(_p(g), U, N, _p(state["pc"]), _p(state["pb"]), _p(state["mc"]), _p(state["mb"]),
                           _p(state["vc"]), _p(state["vb"]), float(lr), float(beta1), float(beta2), float(eps),
                           float(scale), int(step))
    return state


def raster_fwd_bruteforce(rec, cam, bg):
    W, H = cam.width, cam.height
    image = np.zeros((3, H, W), np.float32)
    T = np.zeros((H, W), np.float32)
    nc = np.zeros((H, W), np.int32)
    last = np.zeros((H, W), np.int32)
    n = rec["tiles"].shape[0]
    lib().or_raster_fwd_bruteforce(_p(rec["xyzo"]), _p(rec["conic"]), _p(rec["rgb"]),
                                   _p(rec["rect"]), _p(rec["tiles"]), n, W, H,
                                   _p(_c(bg, np.float32)), _p(image), _p(T), _p(nc), _p(last))
    return {"image": image, "final_T": T, "n_contrib": nc, "last": last}


def _param_ptrs(scene, dt):
    arrs = [_c(scene.means, dt), _c(scene.log_scales, dt), _c(scene.quats, dt),
            _c(scene.opacity_logits, dt), _c(scene.sh, dt)]
    return arrs


def loss_frozen(params64, scene, cam, rec, bins, dL_dimage, want_image=False):
    """fp64 loss sum(dL_dimage * image) with the fp32 run's decisions fixed.

    params64 = (means, log_scales, quats, logits, sh) as float64 SoA arrays."""
    means, ls, q, lg, sh = [_c(a, np.float64) for a in params64]
    act = rec.get("active_idx")
    img = np.zeros((3, cam.height, cam.width), np.float64) if want_image else None
    vals = bins["vals"] if bins["vals"].size else np.zeros(1, np.uint32)
    loss = lib().or_loss_frozen_f64(
        _p(means), _p(ls), _p(q), _p(lg), _p(sh), scene.sh_degree, scene.N,
        _p(None if act is None else _c(act, np.int32)), rec["n_active"], _p(cam_array(cam)),
        cam.width, cam.height, _p(rec["xyzo"]), _p(rec["conic"]), _p(rec["rgb"]),
        _p(rec["tiles"]), _p(vals), _p(_c(bins["ranges"], np.uint32)),
        _p(_c(scene.bg, np.float32)), _p(_c(dL_dimage, np.float32)), _p(img))
    return (loss, img) if want_image else loss


def num_threads() -> int:
    return int(lib().or_num_threads())


def backward(scene, cam, rec, bins, dL_dimage, params3d=True, tile_subset=None, records2d="fp32"):
    """Reference gradients (fp64, fp32 decisions) with magnitude bounds.

    records2d: "fp32" differentiates the compositing at the fp32 records (the
    raster stage's inputs); "fp64" at an fp64 re-projection of the parameters,
    the point the frozen-decision loss (finite differences) evaluates."""
    N, K = scene.N, scene.K
    na = rec["n_active"]
    act = rec.get("active_idx")
    g2 = np.zeros((max(na, 1), 9), np.float64)
    s2 = np.zeros((max(na, 1), 9), np.float64)
    out = {"g2d": g2[:na], "s2d": s2[:na]}
    d = m = [None] * 5
    if params3d:
        d = [np.zeros((3, N)), np.zeros((3, N)), np.zeros((4, N)), np.zeros(N), np.zeros((3 * K, N))]
        m = [np.zeros((3, N)), np.zeros((3, N)), np.zeros((4, N)), np.zeros(N), np.zeros((3 * K, N))]
    vals = bins["vals"] if bins["vals"].size else np.zeros(1, np.uint32)
    p = _param_ptrs(scene, np.float32)
    lib().or_backward_f64(
        *[_p(a) for a in p], scene.sh_degree, N, _p(None if act is None else _c(act, np.int32)), na,
        _p(cam_array(cam)), cam.width, cam.height, _p(rec["xyzo"]), _p(rec["conic"]),
        _p(rec["rgb"]), _p(rec["tiles"]), _p(vals), _p(_c(bins["ranges"], np.uint32)),
        _p(_c(scene.bg, np.float32)), _p(_c(dL_dimage, np.float32)), _p(g2), _p(s2),
        *[_p(a) for a in d], *[_p(a) for a in m],
        _p(None if tile_subset is None else _c(tile_subset, np.int32)),
        0 if tile_subset is None else len(tile_subset), 1 if records2d == "fp32" else 0)
    if params3d:
        names = ["means", "log_scales", "quats", "opacity_logits", "sh"]
        out.update({"d_" + k: v for k, v in zip(names, d)})
        out.update({"m_" + k: v for k, v in zip(names, m)})
    return out


def preprocess_bwd(scene, cam, rec, g2):
    """Parameter gradients from given 2-D gradients [n_active x 9] (fp64)."""
    N, K = scene.N, scene.K
    act = rec.get("active_idx")
    g2 = _c(g2, np.float64)
    d = [np.zeros((3, N)), np.zeros((3, N)), np.zeros((4, N)), np.zeros(N), np.zeros((3 * K, N))]
    m = [np.zeros((3, N)), np.zeros((3, N)), np.zeros((4, N)), np.zeros(N), np.zeros((3 * K, N))]
    p = _param_ptrs(scene, np.float32)
    lib().or_preprocess_bwd_f64(
        *[_p(a) for a in p], scene.sh_degree, N, _p(None if act is None else _c(act, np.int32)),
        rec["n_active"], _p(cam_array(cam)), cam.width, cam.height, _p(rec["rgb"]),
        _p(rec["tiles"]), _p(g2), *[_p(a) for a in d], *[_p(a) for a in m])
    names = ["means", "log_scales", "quats", "opacity_logits", "sh"]
    out = {"d_" + k: v for k, v in zip(names, d)}
    out.update({"m_" + k: v for k, v in zip(names, m)})
    return out


def project_f64(params64, sh_degree, N, cam):
    means, ls, q, lg, sh = [_c(a, np.float64) for a in params64]
    out = np.zeros((N, 10), np.float64)
    vis = np.zeros(N, np.int32)
    rad = np.zeros(N, np.int32)
    lib().or_project_f64(_p(means), _p(ls), _p(q), _p(lg), _p(sh), sh_degree, N,
                         _p(cam_array(cam)), cam.width, cam.height, _p(out), _p(vis), _p(rad))
    return out, vis, rad


def render(scene, pose=0, tile_subset=None):
    """Whole forward path for one pose: cull, preprocess, bin/sort, raster."""
    cam = scene.cameras[pose]
    cl = cull(scene, cam)
    use_cull = scene.lod_dist > 0 or scene.importance_q > 0
    rec = preprocess(scene, cam, cl["active_idx"] if use_cull else None,
                     cl["n_active"] if use_cull else None)
    bins = bin_sort(rec, cam)
    fwd = raster_fwd(rec, bins, cam, scene.bg, tile_subset)
    return {"cull": cl, "rec": rec, "bins": bins, "fwd": fwd, "cam": cam}
