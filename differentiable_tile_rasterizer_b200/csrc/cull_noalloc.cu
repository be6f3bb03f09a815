// gs_cull_noalloc: the per-view cull for callers that cannot hand the library
// any device memory for scratch.
//
// Some callers cannot allocate device memory at all. A plugin running inside
// a host application (a game or visualisation engine, a driver-level layer)
// often does not own the device allocator and gets no workspace from it, and
// a hard real-time loop may not call cudaMalloc, whose implicit device-wide
// synchronisation would stall the frame. For them this entry point keeps the
// cull's scratch (radix-select histogram, select state, per-block counts) in
// a file-scope device array that is part of the loaded library image, so the
// call allocates nothing: no cudaMalloc, no cudaFree, no allocating library
// routine. The caller still passes all inputs and outputs.
//
// Costs and limits, stated in gs.h as well:
//  - every GPU that loads the library holds kNoAllocScratchBytes (32 KiB) of
//    this array until the process exits;
//  - N is limited to GS_CULL_NOALLOC_MAX_N (2^24) Gaussians;
//  - all calls share the one array. Each call clears what must start at zero
//    (histogram and select state) before use, but two calls whose work
//    overlaps on the GPU (different streams, or different host threads) race
//    on it and corrupt each other's results.

#include <cmath>
#include <mutex>

#include "gs.h"
#include "gs_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = 32 * 1024;

// The scratch itself. In host code this name is only a stand-in for the symbol,
// not a device address: the address is obtained once per device with
// cudaGetSymbolAddress (see scratch_for_current_device) and passed to the
// kernels like any workspace pointer.
static __device__ __align__(256) unsigned char g_cull_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device; looked up on the first
// call made with that device current, then cached.
cudaError_t scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_cull_scratch);
    if (e != cudaSuccess) return e;
    if (p == nullptr) return cudaErrorInvalidSymbol;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

// The same camera checks as gs_cull.
bool camera_usable(const gs_camera* c) {
  if (!c) return false;
  if (c->width < 1 || c->height < 1 || c->width > 65535 * 16 || c->height > 65535 * 16) return false;
  for (int k = 0; k < 9; ++k)
    if (!std::isfinite(c->R[k])) return false;
  for (int k = 0; k < 3; ++k)
    if (!std::isfinite(c->t[k]) || !std::isfinite(c->campos[k])) return false;
  if (!std::isfinite(c->fx) || !std::isfinite(c->fy) || !std::isfinite(c->cx) || !std::isfinite(c->cy))
    return false;
  return std::isfinite(c->near_z) && c->near_z >= 0.0f;
}

}  // namespace

extern "C" GS_API int gs_cull_noalloc(const float* means, const float* importance, int64_t N,
                                      const gs_camera* cam, float lod_dist, float importance_q, uint8_t* mask,
                                      int32_t* active_idx, int32_t* n_active, void* stream) {
  if (N < 0 || N > GS_CULL_NOALLOC_MAX_N || !camera_usable(cam)) return GS_ERR_INVALID_ARGUMENT;
  if (!(importance_q >= 0.0f) || !(importance_q < 1.0f) || !std::isfinite(lod_dist))
    return GS_ERR_INVALID_ARGUMENT;
  if (gs::cull_workspace_bytes(N) > kNoAllocScratchBytes) return GS_ERR_INVALID_ARGUMENT;
  if (!n_active || (N > 0 && (!means || !mask || !active_idx))) return GS_ERR_INVALID_ARGUMENT;
  if (importance_q > 0.0f && N > 0 && !importance) return GS_ERR_INVALID_ARGUMENT;
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return GS_ERR_CUDA;
  const cudaError_t e = gs::launch_cull(means, importance, N, gs::make_devcam(*cam), lod_dist, importance_q, mask,
                                        active_idx, n_active, scratch, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GS_OK : GS_ERR_CUDA;
}
