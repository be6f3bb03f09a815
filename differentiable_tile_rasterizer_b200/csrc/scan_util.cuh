// Block-wide scans built from warp shuffles.
#pragma once

#include <cstdint>

namespace gs {

template <typename T>
__device__ __forceinline__ T warp_inclusive_scan(T v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Exclusive scan over the block; `total` receives the block sum. `scratch`
// needs one slot per warp. Every thread of the block must call it.
template <typename T, int BLOCK>
__device__ __forceinline__ T block_exclusive_scan(T v, T& total, T* scratch) {
  constexpr int kWarps = BLOCK / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const T inc = warp_inclusive_scan(v);
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    T w = lane < kWarps ? scratch[lane] : T(0);
    const T wi = warp_inclusive_scan(w);
    if (lane < kWarps) scratch[lane] = wi - w;  // exclusive warp offsets
    if (lane == kWarps - 1) scratch[kWarps] = wi;
  }
  __syncthreads();
  const T out = scratch[warp] + inc - v;
  total = scratch[kWarps];
  __syncthreads();
  return out;
}

template <typename T, int BLOCK>
__device__ __forceinline__ T block_sum(T v, T* scratch) {
  T total;
  block_exclusive_scan<T, BLOCK>(v, total, scratch);
  return total;
}

}  // namespace gs
