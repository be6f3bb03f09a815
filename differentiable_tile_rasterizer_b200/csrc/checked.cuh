// Device-side index checks of the checked build (GS_CHECKED defined at
// compile time). A failed check records its code in the status word of the
// translation unit it sits in (the first failure wins) and the guarded access
// is skipped: nothing traps, so the context stays usable and the host reads
// the word afterwards. Unchecked builds compile every check to `true`.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace gs {

enum CheckCode : uint32_t {
  kCheckRecordIndex = 1,  // a list value or active index past the record count
  kCheckSortSlot = 2,     // a radix-sort scatter destination past the key count
  kCheckTileRange = 3,    // a tile range that runs backwards
};

#ifdef GS_CHECKED
static __device__ uint32_t g_checked_status;
__device__ __forceinline__ bool check(bool ok, uint32_t code) {
  if (!ok) atomicCAS(&g_checked_status, 0u, code);
  return ok;
}
// This translation unit's status word, cleared after reading (host side).
static inline uint32_t take_checked_status() {
  uint32_t v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_checked_status, sizeof v) != cudaSuccess) return 0xffffffffu;
  if (cudaMemcpyToSymbol(g_checked_status, &z, sizeof z) != cudaSuccess) return 0xffffffffu;
  return v;
}
#else
__device__ __forceinline__ bool check(bool, uint32_t) { return true; }
static inline uint32_t take_checked_status() { return 0; }
#endif

// Readers of the translation units that hold checks.
uint32_t checked_status_raster();
uint32_t checked_status_binsort();
uint32_t checked_status_preprocess();

}  // namespace gs
