// Per-view statistics over the 2-D gradients: for every Gaussian visible in
// the view, the norm of the gradient of the loss with respect to its
// projected mean, summed over views, and the number of views in which it was
// visible (the mean of the two is the usual densification criterion of
// Gaussian splatting training).

#include "gs_device.cuh"
#include "gs_internal.cuh"

namespace gs {
namespace {

// One thread per record; each Gaussian has at most one record per view, so
// the accumulation needs no atomics.
__global__ void __launch_bounds__(256) grad2d_norm_kernel(const float4* grad2d, const int32_t* tiles,
                                                          const int32_t* active_idx, const int32_t* n_active,
                                                          int64_t n_records, float* norm_sum,
                                                          int32_t* view_count) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t na = n_active ? (int64_t)*n_active : n_records;
  if (i >= n_records || i >= na || tiles[i] <= 0) return;
  const float4 g = grad2d[3 * i];  // (dpx, dpy, dopacity, 0)
  const float nrm = __fsqrt_rn(__fmaf_rn(g.x, g.x, __fmul_rn(g.y, g.y)));
  const int64_t gid = active_idx ? (int64_t)active_idx[i] : i;
  norm_sum[gid] = __fadd_rn(norm_sum[gid], nrm);
  view_count[gid] += 1;
}

}  // namespace

cudaError_t launch_grad2d_norm(const float4* grad2d, const int32_t* tiles, const int32_t* active_idx,
                               const int32_t* n_active, int64_t n_records, float* norm_sum, int32_t* view_count,
                               cudaStream_t s) {
  if (n_records == 0) return cudaSuccess;
  grad2d_norm_kernel<<<grid_for(n_records, 256), 256, 0, s>>>(grad2d, tiles, active_idx, n_active, n_records,
                                                               norm_sum, view_count);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace gs
