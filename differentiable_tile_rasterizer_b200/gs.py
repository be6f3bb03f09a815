"""ctypes binding of libgs.so (include/gs.h), argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
CUDA tensors (or None where the C argument may be NULL) and raises GsError on
a non-zero status. No computation happens in Python; there is no fallback:
if the library is missing, loading raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import _build

GS_OK = 0
GS_ERR_INVALID_ARGUMENT = 1
GS_ERR_CAPACITY = 2
GS_ERR_CUDA = 3
GS_ERR_DEVICE_TIMEOUT = 4
GS_ERR_UNSUPPORTED = 5

EXPORTED = ["gs_version", "gs_status_string", "gs_cull", "gs_preprocess", "gs_preprocess_multiview",
            "gs_bin_sort", "gs_bin_sort_async", "gs_tile_order", "gs_accumulate_grad2d_norm", "gs_quant_encode",
            "gs_quant_decode", "gs_adam_sh_quant", "gs_route_ctas", "gs_route_count", "gs_route_pack",
            "gs_merge_received", "gs_unmerge_grad2d", "gs_return_grad2d",
            "gs_rasterize_fwd", "gs_rasterize_fwd_importance", "gs_rasterize_bwd", "gs_rasterize_bwd_2d", "gs_preprocess_bwd",
            "gs_preprocess_bwd_accumulate", "gs_preprocess_bwd_multiview",
            "gs_debug_set_stalled_sort_tile", "gs_debug_kernel_launches", "gs_debug_is_checked_build",
            "gs_debug_checked_status", "gs_cull_noalloc"]
GS_CULL_NOALLOC_MAX_N = 16777216
GS_MAX_VIEWS = 16
GS_WIRE_RECORD_BYTES = 64
GS_MAX_RANKS = 32


class GsError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: status {status} ({msg})")
        self.status = status


class GsAdamConfig(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double), ("beta2", ctypes.c_double),
                ("eps", ctypes.c_double), ("code_scale", ctypes.c_double), ("step", ctypes.c_int64)]


class GsCamera(ctypes.Structure):
    _fields_ = [("R", ctypes.c_float * 9), ("t", ctypes.c_float * 3),
                ("campos", ctypes.c_float * 3), ("fx", ctypes.c_float), ("fy", ctypes.c_float),
                ("cx", ctypes.c_float), ("cy", ctypes.c_float), ("near_z", ctypes.c_float),
                ("width", ctypes.c_int32), ("height", ctypes.c_int32)]


class GsProjected(ctypes.Structure):
    _fields_ = [("xyzo", ctypes.c_void_p), ("conic", ctypes.c_void_p), ("rgb", ctypes.c_void_p),
                ("radius", ctypes.c_void_p), ("rect", ctypes.c_void_p),
                ("tiles_touched", ctypes.c_void_p)]


_LIB = None
P = ctypes.c_void_p
I64 = ctypes.c_int64
PI64 = ctypes.POINTER(ctypes.c_int64)
PSZ = ctypes.POINTER(ctypes.c_size_t)
PCAM = ctypes.POINTER(GsCamera)
PPROJ = ctypes.POINTER(GsProjected)


def lib_path() -> str:
    """libgs.so, or its checked build (device-side bounds checks) when the
    environment sets GS_CHECKED=1."""
    return _build.LIB_CHECKED if os.environ.get("GS_CHECKED") == "1" else _build.LIB


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libgs.so (building it first if it is absent and nvcc is available)."""
    global _LIB
    if _LIB is None:
        path = lib_path()
        if not os.path.exists(path):
            if not build_if_missing:
                raise OSError(f"library not built: {path}")
            _build.build(checked=path == _build.LIB_CHECKED)
        L = ctypes.CDLL(path)
        L.gs_version.restype = ctypes.c_int
        L.gs_status_string.restype = ctypes.c_char_p
        L.gs_status_string.argtypes = [ctypes.c_int]
        L.gs_cull.argtypes = [P, P, I64, PCAM, ctypes.c_float, ctypes.c_float, P, P, P, P, PSZ, P]
        L.gs_preprocess.argtypes = [P, P, P, P, P, ctypes.c_int, I64, P, P, PCAM, PPROJ, P]
        L.gs_preprocess_multiview.argtypes = [P, P, P, P, P, ctypes.c_int, I64, P, ctypes.c_int, P, P]
        L.gs_accumulate_grad2d_norm.argtypes = [P, P, P, P, I64, P, P, P]
        L.gs_quant_encode.argtypes = [P, I64, I64, ctypes.c_int, P, P, P]
        L.gs_quant_decode.argtypes = [P, P, I64, I64, ctypes.c_int, P, P]
        L.gs_adam_sh_quant.argtypes = [P, I64, I64, P, P, P, P, P, P, ctypes.POINTER(GsAdamConfig), P]
        L.gs_route_ctas.argtypes = [I64]
        L.gs_route_ctas.restype = ctypes.c_int64
        L.gs_route_count.argtypes = [PPROJ, I64, ctypes.c_int, ctypes.c_int, P, P, P, P, P, P]
        L.gs_route_pack.argtypes = [PPROJ, P, I64, ctypes.c_int, ctypes.c_int, P, P, P, P, P]
        L.gs_merge_received.argtypes = [P, P, ctypes.c_int, I64, ctypes.c_int, ctypes.c_int, PPROJ, P, P]
        L.gs_unmerge_grad2d.argtypes = [P, P, I64, P, P]
        L.gs_return_grad2d.argtypes = [P, P, I64, P, P]
        L.gs_bin_sort.argtypes = [PPROJ, I64, PCAM, P, P, P, I64, P, PI64, P, PSZ, P]
        L.gs_bin_sort_async.argtypes = [PPROJ, I64, PCAM, P, P, P, I64, P, P, P, PSZ, P]
        L.gs_tile_order.argtypes = [P, I64, P, P]
        L.gs_rasterize_fwd.argtypes = [PPROJ, P, P, P, PCAM, P, P, P, P, P, P, P]
        L.gs_rasterize_fwd_importance.argtypes = [PPROJ, P, P, P, PCAM, P, P, P, P, P, P, P, P, P]
        L.gs_rasterize_bwd.argtypes = [P, P, P, P, P, ctypes.c_int, I64, P, P, P, PCAM, PPROJ, P, P, P, P, P,
                                       P, P, P, P, P, P, P, P, P, P]
        L.gs_preprocess_bwd.argtypes = [P, P, P, P, P, ctypes.c_int, I64, P, P, P, PCAM, PPROJ, P,
                                        P, P, P, P, P, P]
        L.gs_rasterize_bwd_2d.argtypes = [PPROJ, I64, P, P, P, P, PCAM, P, P, P, P, P, P]
        L.gs_preprocess_bwd_accumulate.argtypes = [P, P, P, P, P, ctypes.c_int, I64, P, P, PCAM, PPROJ, P,
                                                   P, P, P, P, P, P]
        L.gs_preprocess_bwd_multiview.argtypes = [P, P, P, P, P, ctypes.c_int, I64, P, ctypes.c_int, P, P,
                                                  P, P, P, P, P, P]
        L.gs_cull_noalloc.argtypes = [P, P, I64, PCAM, ctypes.c_float, ctypes.c_float, P, P, P, P]
        L.gs_cull_noalloc.restype = ctypes.c_int
        L.gs_debug_kernel_launches.restype = ctypes.c_int64
        L.gs_debug_kernel_launches.argtypes = []
        L.gs_debug_set_stalled_sort_tile.argtypes = [I64]
        L.gs_debug_set_stalled_sort_tile.restype = None
        L.gs_debug_is_checked_build.restype = ctypes.c_int
        L.gs_debug_is_checked_build.argtypes = []
        L.gs_debug_checked_status.restype = ctypes.c_uint32
        L.gs_debug_checked_status.argtypes = []
        for name in ["gs_cull", "gs_preprocess", "gs_preprocess_multiview", "gs_bin_sort", "gs_accumulate_grad2d_norm",
                     "gs_quant_encode", "gs_quant_decode", "gs_adam_sh_quant", "gs_route_count", "gs_route_pack",
                     "gs_merge_received", "gs_unmerge_grad2d", "gs_return_grad2d", "gs_bin_sort_async", "gs_rasterize_fwd",
                     "gs_rasterize_fwd_importance",
                     "gs_rasterize_bwd", "gs_rasterize_bwd_2d", "gs_preprocess_bwd", "gs_preprocess_bwd_accumulate",
                     "gs_preprocess_bwd_multiview"]:
            getattr(L, name).restype = ctypes.c_int
        _LIB = L
    return _LIB


def _check(fn: str, status: int):
    if status != GS_OK:
        raise GsError(fn, status, load().gs_status_string(status).decode())


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def camera(cam) -> GsCamera:
    """gs_camera from any object with R, t, campos, fx, fy, cx, cy, width, height, near_z."""
    c = GsCamera()
    R = [float(v) for v in torch.as_tensor(cam.R, dtype=torch.float32).reshape(9).tolist()]
    c.R[:] = R
    c.t[:] = [float(v) for v in torch.as_tensor(cam.t, dtype=torch.float32).reshape(3).tolist()]
    c.campos[:] = [float(v) for v in torch.as_tensor(cam.campos, dtype=torch.float32).reshape(3).tolist()]
    c.fx, c.fy, c.cx, c.cy = float(cam.fx), float(cam.fy), float(cam.cx), float(cam.cy)
    c.near_z = float(cam.near_z)
    c.width, c.height = int(cam.width), int(cam.height)
    return c


def projected(rec: dict) -> GsProjected:
    """gs_projected from a dict of record tensors (see Records in pipeline.py)."""
    return GsProjected(_p(rec["xyzo"]), _p(rec["conic"]), _p(rec["rgb"]), _p(rec["radius"]),
                       _p(rec["rect"]), _p(rec["tiles"]))


def version() -> int:
    return load().gs_version()


def gs_cull(means, importance, N, cam: GsCamera, lod_dist, importance_q, mask, active_idx,
            n_active, workspace, stream=None):
    nbytes = ctypes.c_size_t(0 if workspace is None else workspace.numel() * workspace.element_size())
    _check("gs_cull", load().gs_cull(_p(means), _p(importance), int(N), ctypes.byref(cam),
                                     float(lod_dist), float(importance_q), _p(mask), _p(active_idx),
                                     _p(n_active), _p(workspace), ctypes.byref(nbytes), _stream(stream)))
    return nbytes.value


def gs_cull_noalloc(means, importance, N, cam: GsCamera, lod_dist, importance_q, mask, active_idx,
                    n_active, stream=None):
    """gs_cull with the library's own static scratch (no workspace argument)."""
    _check("gs_cull_noalloc", load().gs_cull_noalloc(
        _p(means), _p(importance), int(N), ctypes.byref(cam), float(lod_dist), float(importance_q),
        _p(mask), _p(active_idx), _p(n_active), _stream(stream)))


def gs_cull_workspace(N, cam: GsCamera) -> int:
    nbytes = ctypes.c_size_t(0)
    _check("gs_cull", load().gs_cull(None, None, int(N), ctypes.byref(cam), 0.0, 0.0, None, None, None,
                                     None, ctypes.byref(nbytes), None))
    return nbytes.value


def gs_preprocess(means, log_scales, quats, opacity_logits, sh, sh_degree, N, active_idx, n_active,
                  cam: GsCamera, out: GsProjected, stream=None):
    _check("gs_preprocess", load().gs_preprocess(
        _p(means), _p(log_scales), _p(quats), _p(opacity_logits), _p(sh), int(sh_degree), int(N),
        _p(active_idx), _p(n_active), ctypes.byref(cam), ctypes.byref(out), _stream(stream)))


def gs_preprocess_multiview(means, log_scales, quats, opacity_logits, sh, sh_degree, N, cams, outs,
                            stream=None):
    """cams: list of GsCamera, outs: list of GsProjected (one per view)."""
    if len(cams) != len(outs):
        raise ValueError("one record set per camera")
    V = len(cams)
    cam_arr = (GsCamera * max(V, 1))(*cams)
    out_arr = (GsProjected * max(V, 1))(*outs)
    _check("gs_preprocess_multiview", load().gs_preprocess_multiview(
        _p(means), _p(log_scales), _p(quats), _p(opacity_logits), _p(sh), int(sh_degree), int(N),
        ctypes.cast(cam_arr, P), V, ctypes.cast(out_arr, P), _stream(stream)))


def gs_quant_encode(x, U, N, bits, codes, bounds, stream=None):
    _check("gs_quant_encode", load().gs_quant_encode(_p(x), int(U), int(N), int(bits), _p(codes), _p(bounds),
                                                     _stream(stream)))


def gs_quant_decode(codes, bounds, U, N, bits, x, stream=None):
    _check("gs_quant_decode", load().gs_quant_decode(_p(codes), _p(bounds), int(U), int(N), int(bits), _p(x),
                                                     _stream(stream)))


def gs_adam_sh_quant(grad, U, N, pc, pb, mc, mb, vc, vb, lr, beta1, beta2, eps, code_scale, step, stream=None):
    cfg = GsAdamConfig(float(lr), float(beta1), float(beta2), float(eps), float(code_scale), int(step))
    _check("gs_adam_sh_quant", load().gs_adam_sh_quant(
        _p(grad), int(U), int(N), _p(pc), _p(pb), _p(mc), _p(mb), _p(vc), _p(vb), ctypes.byref(cfg),
        _stream(stream)))


def gs_route_count(rec: GsProjected, n, n_ranks, tiles_y, mask, cta_counts, totals, band_starts=None,
                   dst_offsets=None, stream=None):
    """band_starts: host sequence of n_ranks + 1 tile rows (None: equal bands)."""
    bs = None
    if band_starts is not None:
        bs = (ctypes.c_int32 * len(band_starts))(*[int(v) for v in band_starts])
    _check("gs_route_count", load().gs_route_count(ctypes.byref(rec), int(n), int(n_ranks), int(tiles_y),
                                                   bs, _p(mask), _p(cta_counts), _p(totals), _p(dst_offsets),
                                                   _stream(stream)))


def gs_route_pack(rec: GsProjected, mask, n, n_ranks, rank, cta_offsets, dst_offsets, send, src_idx, stream=None):
    _check("gs_route_pack", load().gs_route_pack(ctypes.byref(rec), _p(mask), int(n), int(n_ranks), int(rank),
                                                 _p(cta_offsets), _p(dst_offsets), _p(send), _p(src_idx),
                                                 _stream(stream)))


def gs_merge_received(recv, seg_offsets, n_ranks, n_recv, row_lo, row_hi, out: GsProjected, perm, stream=None):
    _check("gs_merge_received", load().gs_merge_received(_p(recv), _p(seg_offsets), int(n_ranks), int(n_recv),
                                                         int(row_lo), int(row_hi), ctypes.byref(out), _p(perm),
                                                         _stream(stream)))


def gs_unmerge_grad2d(grad2d, perm, n, back, stream=None):
    _check("gs_unmerge_grad2d", load().gs_unmerge_grad2d(_p(grad2d), _p(perm), int(n), _p(back), _stream(stream)))


def gs_return_grad2d(ret, src_idx, n, grad2d, stream=None):
    _check("gs_return_grad2d", load().gs_return_grad2d(_p(ret), _p(src_idx), int(n), _p(grad2d), _stream(stream)))


def gs_accumulate_grad2d_norm(grad2d, tiles_touched, active_idx, n_active, n_records, norm_sum, view_count,
                              stream=None):
    _check("gs_accumulate_grad2d_norm", load().gs_accumulate_grad2d_norm(
        _p(grad2d), _p(tiles_touched), _p(active_idx), _p(n_active), int(n_records), _p(norm_sum),
        _p(view_count), _stream(stream)))


def gs_bin_sort_workspace(n, cam: GsCamera, capacity) -> int:
    nbytes = ctypes.c_size_t(0)
    ni = ctypes.c_int64(0)
    _check("gs_bin_sort", load().gs_bin_sort(None, int(n), ctypes.byref(cam), None, None, None,
                                             int(capacity), None, ctypes.byref(ni), None,
                                             ctypes.byref(nbytes), None))
    return nbytes.value


def gs_bin_sort(rec: GsProjected, n, cam: GsCamera, offsets, keys, vals, capacity, tile_ranges,
                workspace, stream=None, raise_on_capacity=True):
    """Returns (status, n_instances). Raises on errors other than GS_ERR_CAPACITY."""
    nbytes = ctypes.c_size_t(workspace.numel() * workspace.element_size())
    ni = ctypes.c_int64(0)
    st = load().gs_bin_sort(ctypes.byref(rec), int(n), ctypes.byref(cam), _p(offsets), _p(keys),
                            _p(vals), int(capacity), _p(tile_ranges), ctypes.byref(ni), _p(workspace),
                            ctypes.byref(nbytes), _stream(stream))
    if st == GS_ERR_CAPACITY and not raise_on_capacity:
        return st, ni.value
    _check("gs_bin_sort", st)
    return st, ni.value


def gs_bin_sort_async(rec: GsProjected, n, cam: GsCamera, offsets, keys, vals, capacity, tile_ranges,
                      result, workspace, stream=None):
    """Enqueues the bin/sort only; result [device] int64[2] receives (I, status).
    Raises on argument errors."""
    nbytes = ctypes.c_size_t(workspace.numel() * workspace.element_size())
    _check("gs_bin_sort_async", load().gs_bin_sort_async(
        ctypes.byref(rec), int(n), ctypes.byref(cam), _p(offsets), _p(keys), _p(vals), int(capacity),
        _p(tile_ranges), _p(result), _p(workspace), ctypes.byref(nbytes), _stream(stream)))


def gs_tile_order(tile_ranges, n_tiles, order, stream=None):
    _check("gs_tile_order", load().gs_tile_order(_p(tile_ranges), int(n_tiles), _p(order), _stream(stream)))


def gs_rasterize_fwd(rec: GsProjected, vals, tile_ranges, cam: GsCamera, bg, image, final_T,
                     n_contrib, last, stream=None, tile_order=None, hit_bits=None):
    bgv = (ctypes.c_float * 3)(*[float(b) for b in bg])
    _check("gs_rasterize_fwd", load().gs_rasterize_fwd(
        ctypes.byref(rec), _p(vals), _p(tile_ranges), _p(tile_order), ctypes.byref(cam), ctypes.cast(bgv, P),
        _p(image), _p(final_T), _p(n_contrib), _p(last), _p(hit_bits), _stream(stream)))


def gs_rasterize_fwd_importance(rec: GsProjected, vals, tile_ranges, cam: GsCamera, bg, active_idx, image,
                                final_T, n_contrib, last, importance, stream=None, tile_order=None, hit_bits=None):
    bgv = (ctypes.c_float * 3)(*[float(b) for b in bg])
    _check("gs_rasterize_fwd_importance", load().gs_rasterize_fwd_importance(
        ctypes.byref(rec), _p(vals), _p(tile_ranges), _p(tile_order), ctypes.byref(cam), ctypes.cast(bgv, P), _p(active_idx),
        _p(image), _p(final_T), _p(n_contrib), _p(last), _p(importance), _p(hit_bits), _stream(stream)))


def gs_rasterize_bwd(means, log_scales, quats, opacity_logits, sh, sh_degree, N, active_idx, n_active,
                     mask, cam: GsCamera, rec: GsProjected, vals, tile_ranges, bg, final_T, last,
                     dL_dimage, grad2d, d_means, d_log_scales, d_quats, d_opacity_logits, d_sh,
                     stream=None, tile_order=None, hit_bits=None):
    bgv = (ctypes.c_float * 3)(*[float(b) for b in bg])
    _check("gs_rasterize_bwd", load().gs_rasterize_bwd(
        _p(means), _p(log_scales), _p(quats), _p(opacity_logits), _p(sh), int(sh_degree), int(N),
        _p(active_idx), _p(n_active), _p(mask), ctypes.byref(cam), ctypes.byref(rec), _p(vals),
        _p(tile_ranges), _p(tile_order), _p(hit_bits), ctypes.cast(bgv, P), _p(final_T), _p(last), _p(dL_dimage),
        _p(grad2d), _p(d_means), _p(d_log_scales), _p(d_quats), _p(d_opacity_logits), _p(d_sh), _stream(stream)))


def gs_rasterize_bwd_2d(rec: GsProjected, n_records, vals, tile_ranges, cam: GsCamera, bg, final_T, last,
                        dL_dimage, grad2d, stream=None, tile_order=None, hit_bits=None):
    bgv = (ctypes.c_float * 3)(*[float(b) for b in bg])
    _check("gs_rasterize_bwd_2d", load().gs_rasterize_bwd_2d(
        ctypes.byref(rec), int(n_records), _p(vals), _p(tile_ranges), _p(tile_order), _p(hit_bits),
        ctypes.byref(cam),
        ctypes.cast(bgv, P), _p(final_T), _p(last), _p(dL_dimage), _p(grad2d), _stream(stream)))


def gs_debug_kernel_launches() -> int:
    return int(load().gs_debug_kernel_launches())


def gs_preprocess_bwd(means, log_scales, quats, opacity_logits, sh, sh_degree, N, active_idx, n_active,
                      mask, cam: GsCamera, rec: GsProjected, grad2d, d_means, d_log_scales, d_quats,
                      d_opacity_logits, d_sh, stream=None):
    _check("gs_preprocess_bwd", load().gs_preprocess_bwd(
        _p(means), _p(log_scales), _p(quats), _p(opacity_logits), _p(sh), int(sh_degree), int(N),
        _p(active_idx), _p(n_active), _p(mask), ctypes.byref(cam), ctypes.byref(rec), _p(grad2d),
        _p(d_means), _p(d_log_scales), _p(d_quats), _p(d_opacity_logits), _p(d_sh), _stream(stream)))


def gs_preprocess_bwd_accumulate(means, log_scales, quats, opacity_logits, sh, sh_degree, N, active_idx, n_active,
                                 cam: GsCamera, rec: GsProjected, grad2d, d_means, d_log_scales, d_quats,
                                 d_opacity_logits, d_sh, stream=None):
    _check("gs_preprocess_bwd_accumulate", load().gs_preprocess_bwd_accumulate(
        _p(means), _p(log_scales), _p(quats), _p(opacity_logits), _p(sh), int(sh_degree), int(N),
        _p(active_idx), _p(n_active), ctypes.byref(cam), ctypes.byref(rec), _p(grad2d),
        _p(d_means), _p(d_log_scales), _p(d_quats), _p(d_opacity_logits), _p(d_sh), _stream(stream)))


def gs_preprocess_bwd_multiview(means, log_scales, quats, opacity_logits, sh, sh_degree, N, cams, recs, grad2ds,
                                d_means, d_log_scales, d_quats, d_opacity_logits, d_sh, stream=None):
    """cams: list of GsCamera, recs: list of GsProjected, grad2ds: list of
    [N][12] float32 device tensors (one per view)."""
    if not len(cams) == len(recs) == len(grad2ds):
        raise ValueError("one record set and one 2-D gradient per camera")
    V = len(cams)
    cam_arr = (GsCamera * max(V, 1))(*cams)
    rec_arr = (GsProjected * max(V, 1))(*recs)
    g_arr = (ctypes.c_void_p * max(V, 1))(*[_p(t) for t in grad2ds])
    _check("gs_preprocess_bwd_multiview", load().gs_preprocess_bwd_multiview(
        _p(means), _p(log_scales), _p(quats), _p(opacity_logits), _p(sh), int(sh_degree), int(N),
        ctypes.cast(cam_arr, P), V, ctypes.cast(rec_arr, P), ctypes.cast(g_arr, P),
        _p(d_means), _p(d_log_scales), _p(d_quats), _p(d_opacity_logits), _p(d_sh), _stream(stream)))


def gs_debug_set_stalled_sort_tile(tile: int):
    load().gs_debug_set_stalled_sort_tile(int(tile))


def gs_debug_is_checked_build() -> bool:
    return bool(load().gs_debug_is_checked_build())


def gs_debug_checked_status() -> int:
    """First failed device-side check since the last call (0: none)."""
    return int(load().gs_debug_checked_status())
