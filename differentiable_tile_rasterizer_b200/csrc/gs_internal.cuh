// Internal launch interface shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>

#include <cmath>
#include <cstddef>
#include <cstdint>

#include "gs.h"

namespace gs {

// Camera as passed by value to kernels.
struct DevCam {
  float W[9], t[3], campos[3];
  float fx, fy, cx, cy, near_z;
  int width, height, TW, TH;
};

// Host-side camera validation shared by every entry point that takes a camera:
// a positive image size whose tile grid fits the 16-bit rect fields, finite
// pose and intrinsics, and near_z >= 0 (so depth bits sort like depths).
inline bool camera_ok(const gs_camera* c) {
  if (!c) return false;
  if (c->width < 1 || c->height < 1 || c->width > 65535 * 16 || c->height > 65535 * 16) return false;
  for (int k = 0; k < 9; ++k)
    if (!std::isfinite(c->R[k])) return false;
  for (int k = 0; k < 3; ++k)
    if (!std::isfinite(c->t[k]) || !std::isfinite(c->campos[k])) return false;
  if (!std::isfinite(c->fx) || !std::isfinite(c->fy) || !std::isfinite(c->cx) || !std::isfinite(c->cy)) return false;
  return std::isfinite(c->near_z) && c->near_z >= 0.0f;
}

inline DevCam make_devcam(const gs_camera& c) {
  DevCam d;
  for (int k = 0; k < 9; ++k) d.W[k] = c.R[k];
  for (int k = 0; k < 3; ++k) d.t[k] = c.t[k];
  for (int k = 0; k < 3; ++k) d.campos[k] = c.campos[k];
  d.fx = c.fx; d.fy = c.fy; d.cx = c.cx; d.cy = c.cy; d.near_z = c.near_z;
  d.width = c.width; d.height = c.height;
  d.TW = (c.width + 15) / 16;
  d.TH = (c.height + 15) / 16;
  return d;
}

struct Params {
  const float* means;
  const float* log_scales;
  const float* quats;
  const float* logits;
  const float* sh;
  int64_t N;
  int sh_degree;
  const int32_t* active_idx;  // may be null
  const int32_t* n_active;    // may be null
};

struct Records {
  float4* xyzo;
  float4* conic;
  float4* rgb;
  int32_t* radius;
  ushort4* rect;
  int32_t* tiles;
};

struct Grads {
  float* d_means;
  float* d_log_scales;
  float* d_quats;
  float* d_logits;
  float* d_sh;
};

inline unsigned grid_for(int64_t n, int block) { return (unsigned)((n + block - 1) / block); }

// Process-wide count of kernel launches (see gs_debug_kernel_launches).
void count_launches(int n);
int64_t kernel_launches();

// preprocess.cu
cudaError_t launch_preprocess(const Params& p, const DevCam& cam, const Records& out,
                              cudaStream_t s);
// accumulate: add the visible records' chains to the gradient rows and touch
// nothing else; otherwise overwrite every row (zero for culled and invisible).
cudaError_t launch_preprocess_bwd(const Params& p, const uint8_t* mask, const DevCam& cam,
                                  const Records& in, const float4* grad2d, const Grads& g,
                                  bool accumulate, cudaStream_t s);

// cull.cu
size_t cull_workspace_bytes(int64_t N);
cudaError_t launch_cull(const float* means, const float* importance, int64_t N, const DevCam& cam,
                        float lod_dist, float q, uint8_t* mask, int32_t* active_idx,
                        int32_t* n_active, void* ws, cudaStream_t s);

// Several views of one preprocess pass (all N Gaussians, no cull).
constexpr int kMaxViews = 16;
struct MultiViewArgs {
  DevCam cam[kMaxViews];
  Records out[kMaxViews];
  int n_views;
};
cudaError_t launch_preprocess_multiview(const Params& p, const MultiViewArgs& mv, cudaStream_t s);
struct MultiViewBwdArgs {
  DevCam cam[kMaxViews];
  Records rec[kMaxViews];
  const float4* grad2d[kMaxViews];  // [N][3] per view
  int n_views;
};
// The parameter gradients summed over the views (every row written).
cudaError_t launch_preprocess_bwd_multiview(const Params& p, const MultiViewBwdArgs& mv, const Grads& g,
                                            cudaStream_t s);

// stats.cu: norm_sum[g] += |(dpx, dpy)|, view_count[g] += 1 for every
// visible record of the view (Gaussian g = active_idx[i] or i).
cudaError_t launch_grad2d_norm(const float4* grad2d, const int32_t* tiles, const int32_t* active_idx,
                               const int32_t* n_active, int64_t n_records, float* norm_sum, int32_t* view_count,
                               cudaStream_t s);

// adam.cu: block codes (256 units per block, row stride quant_blocks(N) * 256)
int64_t quant_blocks(int64_t N);
cudaError_t launch_quant_encode(const float* x, int64_t U, int64_t N, int bits, void* codes, float* bounds,
                                cudaStream_t s);
cudaError_t launch_quant_decode(const void* codes, const float* bounds, int64_t U, int64_t N, int bits, float* x,
                                cudaStream_t s);
// hp = {lr, b1, 1 - b1, b2, 1 - b2, c1, c2, eps, code scale e, 1 / e}
cudaError_t launch_adam_sh_quant(const float* grad, int64_t U, int64_t N, uint16_t* pc, float* pb, uint8_t* mc,
                                 float* mb, uint8_t* vc, float* vb, const float hp[10], cudaStream_t s);

// exchange.cu: index-interleaved ranks and the one exchange of projected
// records (bands of tile rows per rank).
constexpr int kMaxRanks = 32;
struct WireRecord {   // 64 bytes on the wire
  float4 xyzo;
  float4 conic;       // w: global Gaussian index (int bits)
  float4 rgb;         // w: radius (int bits)
  ushort4 rect;
  uint2 pad;
};
static_assert(sizeof(WireRecord) == 64, "wire record layout");
// First tile row of every rank's band (row[G] = tile rows), by value.
struct BandStarts {
  int32_t row[kMaxRanks + 1];
};
int64_t route_ctas(int64_t n);
cudaError_t launch_route_count(const Records& rec, int64_t n, int G, const BandStarts& bands, uint32_t* mask,
                               uint32_t* cta_counts, int64_t* totals, int64_t* dst_off, cudaStream_t s);
cudaError_t launch_route_pack(const Records& rec, const uint32_t* mask, int64_t n, int G, int rank,
                              const uint32_t* cta_offsets, const int64_t* dst_off, WireRecord* send,
                              int32_t* src_idx, cudaStream_t s);
cudaError_t launch_merge(const WireRecord* recv, const int64_t* seg_off, int G, int64_t n_recv, int y_lo, int y_hi,
                         const Records& out, int32_t* perm, cudaStream_t s);
cudaError_t launch_unmerge_grad(const float4* grad2d, const int32_t* perm, int64_t n, float4* back,
                                cudaStream_t s);
cudaError_t launch_return_grad(const float4* ret, const int32_t* src_idx, int64_t n, float4* grad2d,
                               cudaStream_t s);

// binsort.cu
struct BinSortPlan {
  int64_t n, capacity, tiles;
  int passes, tile_bits;
  size_t bytes;
};
BinSortPlan binsort_plan(int64_t n, int64_t capacity, int64_t tiles);
// Sorts the records by (depth, index) and scans their tiles_touched in that
// order (total at binsort_total_ptr); also the record-order offsets if given.
cudaError_t launch_depth_order(const Records& rec, int64_t n, int32_t* offsets, void* ws,
                               const BinSortPlan& plan, int64_t stall_tile, cudaStream_t s);
const int64_t* binsort_total_ptr(void* ws, const BinSortPlan& plan);
const int32_t* binsort_status_ptr(void* ws, const BinSortPlan& plan);
// Emits the instances in depth order, sorts them by tile and writes the tile
// ranges; the instance count is read on the device (none are emitted when it
// exceeds plan.capacity: status GS_ERR_CAPACITY). Enqueue only.
cudaError_t launch_emit_sort_ranges(const Records& rec, int64_t n, const DevCam& cam, uint64_t* keys,
                                    uint32_t* vals, uint32_t* ranges, void* ws, const BinSortPlan& plan,
                                    int64_t stall_tile, cudaStream_t s);
// result[0] = instance count, result[1] = status, on the device.
cudaError_t launch_publish(void* ws, const BinSortPlan& plan, int64_t* result, cudaStream_t s);

// raster.cu
// importance == nullptr: the plain forward. Otherwise also adds each
// Gaussian's sum over pixels of alpha * T to importance[active_idx[i] or i].
cudaError_t launch_raster_fwd(const Records& rec, const uint32_t* vals, const uint32_t* ranges,
                              const DevCam& cam, const float bg[3], float* image, float* final_T,
                              int32_t* n_contrib, int32_t* last, float* importance, const int32_t* active_idx,
                              const uint32_t* order, uint8_t* hits, cudaStream_t s);
// Tiles by descending log2 of their list length (order [TT]); the raster
// launches take their CTAs' tiles in this order (order == nullptr: tile b).
cudaError_t launch_tile_order(const uint32_t* ranges, int64_t TT, uint32_t* order, cudaStream_t s);
cudaError_t launch_raster_bwd(const Records& rec, const uint32_t* vals, const uint32_t* ranges,
                              const DevCam& cam, const float bg[3], const float* final_T,
                              const int32_t* last, const float* dL_dimage, float4* grad2d,
                              int64_t n_records, const uint32_t* order, const uint8_t* hits, cudaStream_t s);

}  // namespace gs
