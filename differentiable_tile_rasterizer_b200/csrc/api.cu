// C ABI entry points of libgs.so: argument validation, workspace carving and
// kernel launches. No entry point allocates device memory.

#include <atomic>
#include <cmath>

#include "checked.cuh"
#include "gs.h"
#include "gs_internal.cuh"

using namespace gs;

namespace {

int64_t g_stall_tile = -1;

bool records_ok(const gs_projected* r) {
  return r && r->xyzo && r->conic && r->rgb && r->radius && r->rect && r->tiles_touched;
}

Records to_records(const gs_projected* r) {
  Records o;
  o.xyzo = reinterpret_cast<float4*>(r->xyzo);
  o.conic = reinterpret_cast<float4*>(r->conic);
  o.rgb = reinterpret_cast<float4*>(r->rgb);
  o.radius = r->radius;
  o.rect = reinterpret_cast<ushort4*>(r->rect);
  o.tiles = r->tiles_touched;
  return o;
}

bool params_ok(const float* means, const float* log_scales, const float* quats, const float* logits,
               const float* sh, int64_t N) {
  if (N < 0 || N >= (int64_t(1) << 31)) return false;
  if (N == 0) return true;
  return means && log_scales && quats && logits && sh;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? GS_OK : GS_ERR_CUDA; }

}  // namespace

extern "C" {

GS_API int gs_version(void) { return 1; }

GS_API const char* gs_status_string(int status) {
  switch (status) {
    case GS_OK: return "ok";
    case GS_ERR_INVALID_ARGUMENT: return "invalid argument";
    case GS_ERR_CAPACITY: return "instance capacity exceeded";
    case GS_ERR_CUDA: return "CUDA runtime error";
    case GS_ERR_DEVICE_TIMEOUT: return "bounded device-side wait timed out";
    case GS_ERR_UNSUPPORTED: return "unsupported argument value";
    default: return "unknown status";
  }
}

GS_API void gs_debug_set_stalled_sort_tile(int64_t tile) { g_stall_tile = tile < 0 ? -1 : tile; }

GS_API int64_t gs_debug_kernel_launches(void) { return kernel_launches(); }

GS_API int gs_debug_is_checked_build(void) {
#ifdef GS_CHECKED
  return 1;
#else
  return 0;
#endif
}

GS_API uint32_t gs_debug_checked_status(void) {
  const uint32_t s[3] = {checked_status_raster(), checked_status_binsort(), checked_status_preprocess()};
  for (uint32_t v : s)
    if (v) return v;
  return 0;
}

GS_API int gs_cull(const float* means, const float* importance, int64_t N, const gs_camera* cam,
                   float lod_dist, float importance_q, uint8_t* mask, int32_t* active_idx,
                   int32_t* n_active, void* workspace, size_t* workspace_bytes, void* stream) {
  if (!workspace_bytes || N < 0 || N >= (int64_t(1) << 31) || !camera_ok(cam)) return GS_ERR_INVALID_ARGUMENT;
  if (!(importance_q >= 0.0f) || !(importance_q < 1.0f) || !std::isfinite(lod_dist))
    return GS_ERR_INVALID_ARGUMENT;
  const size_t need = cull_workspace_bytes(N);
  if (!workspace) {
    *workspace_bytes = need;
    return GS_OK;
  }
  if (*workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GS_ERR_INVALID_ARGUMENT;
  if (!n_active || (N > 0 && (!means || !mask || !active_idx))) return GS_ERR_INVALID_ARGUMENT;
  if (importance_q > 0.0f && N > 0 && !importance) return GS_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_cull(means, importance, N, make_devcam(*cam), lod_dist, importance_q, mask,
                                 active_idx, n_active, workspace, static_cast<cudaStream_t>(stream)));
}

GS_API int gs_preprocess(const float* means, const float* log_scales, const float* quats,
                         const float* opacity_logits, const float* sh, int sh_degree, int64_t N,
                         const int32_t* active_idx, const int32_t* n_active, const gs_camera* cam,
                         const gs_projected* out, void* stream) {
  if (sh_degree < 0) return GS_ERR_INVALID_ARGUMENT;
  if (sh_degree > 3) return GS_ERR_UNSUPPORTED;
  if (!params_ok(means, log_scales, quats, opacity_logits, sh, N) || !camera_ok(cam) || !records_ok(out))
    return GS_ERR_INVALID_ARGUMENT;
  Params p{means, log_scales, quats, opacity_logits, sh, N, sh_degree, active_idx, n_active};
  return cuda_status(launch_preprocess(p, make_devcam(*cam), to_records(out), static_cast<cudaStream_t>(stream)));
}

GS_API int gs_preprocess_multiview(const float* means, const float* log_scales, const float* quats,
                                   const float* opacity_logits, const float* sh, int sh_degree, int64_t N,
                                   const gs_camera* cams, int n_views, const gs_projected* outs, void* stream) {
  if (sh_degree < 0 || n_views < 0 || n_views > GS_MAX_VIEWS || (n_views > 0 && (!cams || !outs)))
    return GS_ERR_INVALID_ARGUMENT;
  if (sh_degree > 3) return GS_ERR_UNSUPPORTED;
  if (!params_ok(means, log_scales, quats, opacity_logits, sh, N)) return GS_ERR_INVALID_ARGUMENT;
  MultiViewArgs mv;
  mv.n_views = n_views;
  for (int v = 0; v < n_views; ++v) {
    if (!camera_ok(&cams[v]) || !records_ok(&outs[v])) return GS_ERR_INVALID_ARGUMENT;
    mv.cam[v] = make_devcam(cams[v]);
    mv.out[v] = to_records(&outs[v]);
  }
  Params p{means, log_scales, quats, opacity_logits, sh, N, sh_degree, nullptr, nullptr};
  return cuda_status(launch_preprocess_multiview(p, mv, static_cast<cudaStream_t>(stream)));
}

namespace {
// Shared by gs_bin_sort and gs_bin_sort_async: checks the arguments and
// enqueues the whole bin/sort on the stream (no host round trip). Returns
// GS_OK with *plan_out set, GS_OK with only *workspace_bytes set on a size
// query (*enqueued = false), or an argument/launch error.
int bin_sort_enqueue(const gs_projected* in, int64_t n, const gs_camera* cam, int32_t* offsets, uint64_t* keys,
                     uint32_t* vals, int64_t capacity, uint32_t* tile_ranges, void* workspace,
                     size_t* workspace_bytes, void* stream, BinSortPlan* plan_out, bool* enqueued) {
  *enqueued = false;
  if (!workspace_bytes || !camera_ok(cam) || n < 0 || n >= (int64_t(1) << 31) || capacity < 0 ||
      capacity >= (int64_t(1) << 30))
    return GS_ERR_INVALID_ARGUMENT;
  const DevCam dc = make_devcam(*cam);
  const BinSortPlan plan = binsort_plan(n, capacity, (int64_t)dc.TW * dc.TH);
  if (!workspace) {
    *workspace_bytes = plan.bytes;
    return GS_OK;
  }
  if (*workspace_bytes < plan.bytes || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return GS_ERR_INVALID_ARGUMENT;
  if (!records_ok(in) || !tile_ranges || (capacity > 0 && (!keys || !vals))) return GS_ERR_INVALID_ARGUMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Records rec = to_records(in);
  cudaError_t e = launch_depth_order(rec, n, offsets, workspace, plan, g_stall_tile, s);
  if (e == cudaSuccess) e = launch_emit_sort_ranges(rec, n, dc, keys, vals, tile_ranges, workspace, plan, g_stall_tile, s);
  if (e != cudaSuccess) return GS_ERR_CUDA;
  *plan_out = plan;
  *enqueued = true;
  return GS_OK;
}
}  // namespace

GS_API int gs_bin_sort(const gs_projected* in, int64_t n, const gs_camera* cam, int32_t* offsets,
                       uint64_t* keys, uint32_t* vals, int64_t capacity, uint32_t* tile_ranges,
                       int64_t* n_instances, void* workspace, size_t* workspace_bytes, void* stream) {
  if (workspace && !n_instances) return GS_ERR_INVALID_ARGUMENT;
  BinSortPlan plan;
  bool enqueued;
  const int st = bin_sort_enqueue(in, n, cam, offsets, keys, vals, capacity, tile_ranges, workspace,
                                  workspace_bytes, stream, &plan, &enqueued);
  if (st != GS_OK || !enqueued) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int64_t total = 0;
  int32_t status = 0;
  cudaError_t e = cudaMemcpyAsync(&total, binsort_total_ptr(workspace, plan), sizeof(int64_t),
                                  cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(&status, binsort_status_ptr(workspace, plan), sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return GS_ERR_CUDA;
  *n_instances = total;
  return status;  // GS_OK, GS_ERR_CAPACITY or GS_ERR_DEVICE_TIMEOUT
}

GS_API int gs_bin_sort_async(const gs_projected* in, int64_t n, const gs_camera* cam, int32_t* offsets,
                             uint64_t* keys, uint32_t* vals, int64_t capacity, uint32_t* tile_ranges,
                             int64_t* result, void* workspace, size_t* workspace_bytes, void* stream) {
  BinSortPlan plan;
  bool enqueued;
  const int st = bin_sort_enqueue(in, n, cam, offsets, keys, vals, capacity, tile_ranges, workspace,
                                  workspace_bytes, stream, &plan, &enqueued);
  if (st != GS_OK || !enqueued || !result) return st;
  return cuda_status(launch_publish(workspace, plan, result, static_cast<cudaStream_t>(stream)));
}

GS_API int gs_tile_order(const uint32_t* tile_ranges, int64_t n_tiles, uint32_t* order, void* stream) {
  if (n_tiles < 0 || n_tiles >= (int64_t(1) << 31) || (n_tiles > 0 && (!tile_ranges || !order)))
    return GS_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_tile_order(tile_ranges, n_tiles, order, static_cast<cudaStream_t>(stream)));
}

GS_API int gs_rasterize_fwd(const gs_projected* in, const uint32_t* vals, const uint32_t* tile_ranges,
                            const uint32_t* tile_order, const gs_camera* cam, const float* bg, float* image, float* final_T,
                            int32_t* n_contrib, int32_t* last, uint8_t* hit_bits, void* stream) {
  if (!records_ok(in) || !camera_ok(cam) || !tile_ranges || !bg || !image || !final_T || !n_contrib || !last)
    return GS_ERR_INVALID_ARGUMENT;
  if (reinterpret_cast<uintptr_t>(hit_bits) & 3u) return GS_ERR_INVALID_ARGUMENT;  // word atomics
  const float b[3] = {bg[0], bg[1], bg[2]};
  return cuda_status(launch_raster_fwd(to_records(in), vals, tile_ranges, make_devcam(*cam), b, image, final_T,
                                       n_contrib, last, nullptr, nullptr, tile_order, hit_bits,
                                       static_cast<cudaStream_t>(stream)));
}

GS_API int gs_rasterize_fwd_importance(const gs_projected* in, const uint32_t* vals, const uint32_t* tile_ranges,
                                       const uint32_t* tile_order, const gs_camera* cam, const float* bg, const int32_t* active_idx,
                                       float* image, float* final_T, int32_t* n_contrib, int32_t* last,
                                       float* importance, uint8_t* hit_bits, void* stream) {
  if (!records_ok(in) || !camera_ok(cam) || !tile_ranges || !bg || !image || !final_T || !n_contrib || !last ||
      !importance)
    return GS_ERR_INVALID_ARGUMENT;
  const float b[3] = {bg[0], bg[1], bg[2]};
  return cuda_status(launch_raster_fwd(to_records(in), vals, tile_ranges, make_devcam(*cam), b, image, final_T,
                                       n_contrib, last, importance, active_idx, tile_order, hit_bits,
                                       static_cast<cudaStream_t>(stream)));
}

GS_API int gs_rasterize_bwd_2d(const gs_projected* in, int64_t n_records, const uint32_t* vals,
                               const uint32_t* tile_ranges, const uint32_t* tile_order, const uint8_t* hit_bits,
                               const gs_camera* cam, const float* bg, const float* final_T, const int32_t* last,
                               const float* dL_dimage, float* grad2d, void* stream) {
  if (!records_ok(in) || !camera_ok(cam) || n_records < 0 || n_records >= (int64_t(1) << 31) || !tile_ranges ||
      !bg || !final_T || !last || !dL_dimage || (n_records > 0 && !grad2d))
    return GS_ERR_INVALID_ARGUMENT;
  if (n_records == 0) return GS_OK;
  const float b[3] = {bg[0], bg[1], bg[2]};
  return cuda_status(launch_raster_bwd(to_records(in), vals, tile_ranges, make_devcam(*cam), b, final_T, last,
                                       dL_dimage, reinterpret_cast<float4*>(grad2d), n_records, tile_order, hit_bits,
                                       static_cast<cudaStream_t>(stream)));
}

GS_API int gs_accumulate_grad2d_norm(const float* grad2d, const int32_t* tiles_touched, const int32_t* active_idx,
                                     const int32_t* n_active, int64_t n_records, float* norm_sum,
                                     int32_t* view_count, void* stream) {
  if (n_records < 0 || n_records >= (int64_t(1) << 31) ||
      (n_records > 0 && (!grad2d || !tiles_touched || !norm_sum || !view_count)))
    return GS_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_grad2d_norm(reinterpret_cast<const float4*>(grad2d), tiles_touched, active_idx,
                                        n_active, n_records, norm_sum, view_count,
                                        static_cast<cudaStream_t>(stream)));
}

GS_API int gs_quant_encode(const float* x, int64_t U, int64_t N, int bits, void* codes, float* bounds,
                           void* stream) {
  if (U < 0 || N < 0 || (bits != 8 && bits != 16) || (U * N > 0 && (!x || !codes || !bounds)))
    return GS_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_quant_encode(x, U, N, bits, codes, bounds, static_cast<cudaStream_t>(stream)));
}

GS_API int gs_quant_decode(const void* codes, const float* bounds, int64_t U, int64_t N, int bits, float* x,
                           void* stream) {
  if (U < 0 || N < 0 || (bits != 8 && bits != 16) || (U * N > 0 && (!x || !codes || !bounds)))
    return GS_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_quant_decode(codes, bounds, U, N, bits, x, static_cast<cudaStream_t>(stream)));
}

GS_API int gs_adam_sh_quant(const float* grad, int64_t U, int64_t N, uint16_t* value_codes, float* value_bounds,
                            uint8_t* m_codes, float* m_bounds, uint8_t* v_codes, float* v_bounds,
                            const gs_adam_config* cfg, void* stream) {
  if (!cfg || U < 0 || N < 0 || cfg->step < 1 || !(cfg->code_scale > 0.0) ||
      (U * N > 0 && (!grad || !value_codes || !value_bounds || !m_codes || !m_bounds || !v_codes || !v_bounds)))
    return GS_ERR_INVALID_ARGUMENT;
  // the fp32 constants of the step, each rounded from double
  const double t = (double)cfg->step;
  const float hp[10] = {(float)cfg->lr,
                       (float)cfg->beta1,
                       (float)(1.0 - cfg->beta1),
                       (float)cfg->beta2,
                       (float)(1.0 - cfg->beta2),
                       (float)(1.0 / (1.0 - std::pow(cfg->beta1, t))),
                       (float)(1.0 / (1.0 - std::pow(cfg->beta2, t))),
                       (float)cfg->eps,
                       (float)cfg->code_scale,
                       (float)(1.0 / cfg->code_scale)};
  return cuda_status(launch_adam_sh_quant(grad, U, N, value_codes, value_bounds, m_codes, m_bounds, v_codes,
                                          v_bounds, hp, static_cast<cudaStream_t>(stream)));
}

GS_API int64_t gs_route_ctas(int64_t n) { return n < 0 ? 0 : route_ctas(n); }

GS_API int gs_route_count(const gs_projected* rec, int64_t n, int n_ranks, int tiles_y, const int32_t* band_starts,
                          uint32_t* mask, uint32_t* cta_counts, int64_t* totals, int64_t* dst_offsets, void* stream) {
  if (!records_ok(rec) || n < 0 || n >= (int64_t(1) << 31) || n_ranks < 1 || n_ranks > GS_MAX_RANKS ||
      tiles_y < 1 || !totals || (n > 0 && (!mask || !cta_counts)))
    return GS_ERR_INVALID_ARGUMENT;
  BandStarts b;
  for (int q = 0; q <= n_ranks; ++q) {
    b.row[q] = band_starts ? band_starts[q] : (int32_t)(((int64_t)q * tiles_y) / n_ranks);
    if (q > 0 && b.row[q] < b.row[q - 1]) return GS_ERR_INVALID_ARGUMENT;
  }
  if (b.row[0] != 0 || b.row[n_ranks] != tiles_y) return GS_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_route_count(to_records(rec), n, n_ranks, b, mask, cta_counts, totals, dst_offsets,
                                        static_cast<cudaStream_t>(stream)));
}

GS_API int gs_route_pack(const gs_projected* rec, const uint32_t* mask, int64_t n, int n_ranks, int rank,
                         const uint32_t* cta_offsets, const int64_t* dst_offsets, void* send, int32_t* src_idx,
                         void* stream) {
  if (!records_ok(rec) || n < 0 || n >= (int64_t(1) << 31) || n_ranks < 1 || n_ranks > GS_MAX_RANKS || rank < 0 ||
      rank >= n_ranks || (n > 0 && (!mask || !cta_offsets || !dst_offsets || !send || !src_idx)))
    return GS_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_route_pack(to_records(rec), mask, n, n_ranks, rank, cta_offsets, dst_offsets,
                                       static_cast<WireRecord*>(send), src_idx, static_cast<cudaStream_t>(stream)));
}

GS_API int gs_merge_received(const void* recv, const int64_t* seg_offsets, int n_ranks, int64_t n_recv,
                             int tile_row_lo, int tile_row_hi, const gs_projected* out, int32_t* perm,
                             void* stream) {
  if (!records_ok(out) || n_recv < 0 || n_recv >= (int64_t(1) << 31) || n_ranks < 1 || n_ranks > GS_MAX_RANKS ||
      tile_row_lo < 0 || tile_row_hi < tile_row_lo || (n_recv > 0 && (!recv || !seg_offsets || !perm)))
    return GS_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_merge(static_cast<const WireRecord*>(recv), seg_offsets, n_ranks, n_recv, tile_row_lo,
                                  tile_row_hi, to_records(out), perm, static_cast<cudaStream_t>(stream)));
}

GS_API int gs_unmerge_grad2d(const float* grad2d, const int32_t* perm, int64_t n, float* back, void* stream) {
  if (n < 0 || (n > 0 && (!grad2d || !perm || !back))) return GS_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_unmerge_grad(reinterpret_cast<const float4*>(grad2d), perm, n,
                                         reinterpret_cast<float4*>(back), static_cast<cudaStream_t>(stream)));
}

GS_API int gs_return_grad2d(const float* ret, const int32_t* src_idx, int64_t n, float* grad2d, void* stream) {
  if (n < 0 || (n > 0 && (!ret || !src_idx || !grad2d))) return GS_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_return_grad(reinterpret_cast<const float4*>(ret), src_idx, n,
                                        reinterpret_cast<float4*>(grad2d), static_cast<cudaStream_t>(stream)));
}

GS_API int gs_preprocess_bwd(const float* means, const float* log_scales, const float* quats,
                             const float* opacity_logits, const float* sh, int sh_degree, int64_t N,
                             const int32_t* active_idx, const int32_t* n_active, const uint8_t* mask,
                             const gs_camera* cam, const gs_projected* in, const float* grad2d,
                             float* d_means, float* d_log_scales, float* d_quats, float* d_opacity_logits,
                             float* d_sh, void* stream) {
  if (sh_degree < 0) return GS_ERR_INVALID_ARGUMENT;
  if (sh_degree > 3) return GS_ERR_UNSUPPORTED;
  if (!params_ok(means, log_scales, quats, opacity_logits, sh, N) || !camera_ok(cam) || !records_ok(in))
    return GS_ERR_INVALID_ARGUMENT;
  if (active_idx && !mask) return GS_ERR_INVALID_ARGUMENT;
  if (N > 0 && (!grad2d || !d_means || !d_log_scales || !d_quats || !d_opacity_logits || !d_sh))
    return GS_ERR_INVALID_ARGUMENT;
  Params p{means, log_scales, quats, opacity_logits, sh, N, sh_degree, active_idx, n_active};
  Grads g{d_means, d_log_scales, d_quats, d_opacity_logits, d_sh};
  return cuda_status(launch_preprocess_bwd(p, mask, make_devcam(*cam), to_records(in),
                                           reinterpret_cast<const float4*>(grad2d), g, false,
                                           static_cast<cudaStream_t>(stream)));
}

GS_API int gs_preprocess_bwd_multiview(const float* means, const float* log_scales, const float* quats,
                                       const float* opacity_logits, const float* sh, int sh_degree, int64_t N,
                                       const gs_camera* cams, int n_views, const gs_projected* ins,
                                       const float* const* grad2ds, float* d_means, float* d_log_scales,
                                       float* d_quats, float* d_opacity_logits, float* d_sh, void* stream) {
  if (sh_degree < 0 || n_views < 1 || n_views > GS_MAX_VIEWS || !cams || !ins || !grad2ds)
    return GS_ERR_INVALID_ARGUMENT;
  if (sh_degree > 3) return GS_ERR_UNSUPPORTED;
  if (!params_ok(means, log_scales, quats, opacity_logits, sh, N)) return GS_ERR_INVALID_ARGUMENT;
  if (N > 0 && (!d_means || !d_log_scales || !d_quats || !d_opacity_logits || !d_sh)) return GS_ERR_INVALID_ARGUMENT;
  MultiViewBwdArgs mv;
  mv.n_views = n_views;
  for (int v = 0; v < n_views; ++v) {
    if (!camera_ok(&cams[v]) || !records_ok(&ins[v]) || (N > 0 && !grad2ds[v])) return GS_ERR_INVALID_ARGUMENT;
    mv.cam[v] = make_devcam(cams[v]);
    mv.rec[v] = to_records(&ins[v]);
    mv.grad2d[v] = reinterpret_cast<const float4*>(grad2ds[v]);
  }
  Params p{means, log_scales, quats, opacity_logits, sh, N, sh_degree, nullptr, nullptr};
  Grads g{d_means, d_log_scales, d_quats, d_opacity_logits, d_sh};
  return cuda_status(launch_preprocess_bwd_multiview(p, mv, g, static_cast<cudaStream_t>(stream)));
}

GS_API int gs_preprocess_bwd_accumulate(const float* means, const float* log_scales, const float* quats,
                                        const float* opacity_logits, const float* sh, int sh_degree, int64_t N,
                                        const int32_t* active_idx, const int32_t* n_active, const gs_camera* cam,
                                        const gs_projected* in, const float* grad2d, float* d_means,
                                        float* d_log_scales, float* d_quats, float* d_opacity_logits, float* d_sh,
                                        void* stream) {
  if (sh_degree < 0) return GS_ERR_INVALID_ARGUMENT;
  if (sh_degree > 3) return GS_ERR_UNSUPPORTED;
  if (!params_ok(means, log_scales, quats, opacity_logits, sh, N) || !camera_ok(cam) || !records_ok(in))
    return GS_ERR_INVALID_ARGUMENT;
  if (N > 0 && (!grad2d || !d_means || !d_log_scales || !d_quats || !d_opacity_logits || !d_sh))
    return GS_ERR_INVALID_ARGUMENT;
  Params p{means, log_scales, quats, opacity_logits, sh, N, sh_degree, active_idx, n_active};
  Grads g{d_means, d_log_scales, d_quats, d_opacity_logits, d_sh};
  return cuda_status(launch_preprocess_bwd(p, nullptr, make_devcam(*cam), to_records(in),
                                           reinterpret_cast<const float4*>(grad2d), g, true,
                                           static_cast<cudaStream_t>(stream)));
}

GS_API int gs_rasterize_bwd(const float* means, const float* log_scales, const float* quats,
                            const float* opacity_logits, const float* sh, int sh_degree, int64_t N,
                            const int32_t* active_idx, const int32_t* n_active, const uint8_t* mask,
                            const gs_camera* cam, const gs_projected* in, const uint32_t* vals,
                            const uint32_t* tile_ranges, const uint32_t* tile_order, const uint8_t* hit_bits,
                            const float* bg,
                            const float* final_T, const int32_t* last, const float* dL_dimage,
                            float* grad2d, float* d_means,
                            float* d_log_scales, float* d_quats, float* d_opacity_logits, float* d_sh,
                            void* stream) {
  if (sh_degree < 0) return GS_ERR_INVALID_ARGUMENT;
  if (sh_degree > 3) return GS_ERR_UNSUPPORTED;
  if (!params_ok(means, log_scales, quats, opacity_logits, sh, N) || !camera_ok(cam) || !records_ok(in))
    return GS_ERR_INVALID_ARGUMENT;
  if (!tile_ranges || !bg || !final_T || !last || !dL_dimage || (N > 0 && !grad2d)) return GS_ERR_INVALID_ARGUMENT;
  if (active_idx && !mask) return GS_ERR_INVALID_ARGUMENT;
  if (N > 0 && (!d_means || !d_log_scales || !d_quats || !d_opacity_logits || !d_sh)) return GS_ERR_INVALID_ARGUMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const DevCam dc = make_devcam(*cam);
  const Records rec = to_records(in);
  const float b[3] = {bg[0], bg[1], bg[2]};
  if (N > 0) {
    cudaError_t e = launch_raster_bwd(rec, vals, tile_ranges, dc, b, final_T, last, dL_dimage,
                                      reinterpret_cast<float4*>(grad2d), N, tile_order, hit_bits, s);
    if (e != cudaSuccess) return GS_ERR_CUDA;
  }
  Params p{means, log_scales, quats, opacity_logits, sh, N, sh_degree, active_idx, n_active};
  Grads g{d_means, d_log_scales, d_quats, d_opacity_logits, d_sh};
  return cuda_status(launch_preprocess_bwd(p, mask, dc, rec, reinterpret_cast<const float4*>(grad2d), g, false, s));
}

}  // extern "C"

namespace gs {
namespace {
std::atomic<int64_t> g_launches{0};
}
void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
int64_t kernel_launches() { return g_launches.load(std::memory_order_relaxed); }
}  // namespace gs
