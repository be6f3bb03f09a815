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

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "gs.h"
#include "gs_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = 32 * 1024;

// The scratch itself. In host code this name is only a stand-in for the symbol,
// not a device address: the address is obtained with cudaGetSymbolAddress
// (see scratch_for_current_context) and passed to the kernels like any
// workspace pointer.
static __device__ __align__(256) unsigned char g_cull_scratch[kNoAllocScratchBytes];

// The address of g_cull_scratch belongs to one CUDA context: every context
// that loads the library (the device's primary context, a context the host
// application created itself with cuCtxCreate, or the primary context
// re-created after cudaDeviceReset) holds its own copy of the array at its own
// address. The address is therefore cached per context, keyed by the
// context's unique id (cuCtxGetId), which, unlike a context handle, is never
// reused within a process. The two driver calls are reached through the
// runtime's entry-point query, so the library does not link libcuda itself.
constexpr int kMaxContexts = 64;
struct ScratchSlot {
  unsigned long long ctx_id;
  void* ptr;
};
std::mutex g_mu;
ScratchSlot g_slots[kMaxContexts] = {};
int g_n_slots = 0, g_next_evict = 0;
PFN_cuCtxGetCurrent_v4000 g_get_current = nullptr;
PFN_cuCtxGetId_v12000 g_get_id = nullptr;

cudaError_t resolve_driver_calls() {  // under g_mu
  if (g_get_current && g_get_id) return cudaSuccess;
  void* f = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !f) return e != cudaSuccess ? e : cudaErrorNotSupported;
  g_get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
  f = nullptr;
  e = cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !f) return e != cudaSuccess ? e : cudaErrorNotSupported;
  g_get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
  return cudaSuccess;
}

// Device address of the scratch in the context current on this thread; looked
// up with cudaGetSymbolAddress on the first call made in that context, then
// cached. If no context is current yet, the lookup itself binds the current
// device's primary context, as any runtime call would.
cudaError_t scratch_for_current_context(void** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  cudaError_t e = resolve_driver_calls();
  if (e != cudaSuccess) return e;
  CUcontext ctx = nullptr;
  if (g_get_current(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  void* fresh = nullptr;
  if (ctx == nullptr) {
    e = cudaGetSymbolAddress(&fresh, g_cull_scratch);
    if (e != cudaSuccess) return e;
    if (g_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
  }
  unsigned long long id = 0;
  if (g_get_id(ctx, &id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  for (int k = 0; k < g_n_slots; ++k)
    if (g_slots[k].ctx_id == id) {
      *out = g_slots[k].ptr;
      return cudaSuccess;
    }
  if (fresh == nullptr) {
    e = cudaGetSymbolAddress(&fresh, g_cull_scratch);
    if (e != cudaSuccess) return e;
  }
  if (fresh == nullptr) return cudaErrorInvalidSymbol;
  // ids of destroyed contexts never come back, so an old slot can be reused
  const int k = g_n_slots < kMaxContexts ? g_n_slots++ : (g_next_evict++ % kMaxContexts);
  g_slots[k] = {id, fresh};
  *out = fresh;
  return cudaSuccess;
}

}  // namespace

extern "C" GS_API int gs_cull_noalloc(const float* means, const float* importance, int64_t N,
                                      const gs_camera* cam, float lod_dist, float importance_q, uint8_t* mask,
                                      int32_t* active_idx, int32_t* n_active, void* stream) {
  if (N < 0 || N > GS_CULL_NOALLOC_MAX_N || !gs::camera_ok(cam)) return GS_ERR_INVALID_ARGUMENT;
  if (!(importance_q >= 0.0f) || !(importance_q < 1.0f) || !std::isfinite(lod_dist))
    return GS_ERR_INVALID_ARGUMENT;
  if (gs::cull_workspace_bytes(N) > kNoAllocScratchBytes) return GS_ERR_INVALID_ARGUMENT;
  if (!n_active || (N > 0 && (!means || !mask || !active_idx))) return GS_ERR_INVALID_ARGUMENT;
  if (importance_q > 0.0f && N > 0 && !importance) return GS_ERR_INVALID_ARGUMENT;
  void* scratch = nullptr;
  if (scratch_for_current_context(&scratch) != cudaSuccess) return GS_ERR_CUDA;
  const cudaError_t e = gs::launch_cull(means, importance, N, gs::make_devcam(*cam), lod_dist, importance_q, mask,
                                        active_idx, n_active, scratch, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GS_OK : GS_ERR_CUDA;
}
