// Per-view active-set cull: distance-LOD gate, importance-quantile mask and
// order-preserving compaction (BlitzGS write-up, section 2.3).
//
// The importance threshold tau is the value of rank floor(q N) among all N
// weights. It is found by a three-pass radix select (11, 11 and 10 bits) over
// an order-preserving map of the fp32 bit patterns; each pass histograms the
// weights whose higher bits match the prefix chosen so far and a one-warp
// kernel picks the next digit. Nothing leaves the device, so the whole cull
// is asynchronous. Compaction is reduce-then-scan: per-block kept counts, one
// block scanning them, and a pass that writes the kept indices in order.

#include "gs_device.cuh"
#include "gs_internal.cuh"
#include "scan_util.cuh"

#include <algorithm>
#include <cmath>

namespace gs {
namespace {

constexpr int kBins = 2048;
constexpr int kMaskBlock = 256;
constexpr int kMaskItems = 16;
constexpr int kMaskTile = kMaskBlock * kMaskItems;

struct SelectState {
  uint32_t prefix;   // digits chosen so far
  uint32_t rank;     // rank still to find below the prefix
  uint32_t enabled;  // importance mask active
  uint32_t pad;
};

struct CullWs {
  uint32_t* hist;       // [kBins]
  SelectState* state;   // [1]
  uint32_t* partials;   // [nblocks + 1]
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

CullWs carve(void* ws, int64_t N) {
  char* p = static_cast<char*>(ws);
  CullWs w;
  w.hist = reinterpret_cast<uint32_t*>(p);
  p += align256(kBins * sizeof(uint32_t));
  w.state = reinterpret_cast<SelectState*>(p);
  p += align256(sizeof(SelectState));
  w.partials = reinterpret_cast<uint32_t*>(p);
  return w;
}

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_order_key(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

// pass 0: bits 31..21, pass 1: bits 20..10, pass 2: bits 9..0
__device__ __forceinline__ int digit_shift(int pass) { return pass == 0 ? 21 : (pass == 1 ? 10 : 0); }
__device__ __forceinline__ int digit_bits(int pass) { return pass == 2 ? 10 : 11; }

__global__ void __launch_bounds__(256) select_hist_kernel(const float* imp, int64_t N, int pass,
                                                          const SelectState* st, uint32_t* hist) {
  __shared__ uint32_t sh[kBins];
  for (int b = threadIdx.x; b < kBins; b += blockDim.x) sh[b] = 0;
  __syncthreads();
  const int sft = digit_shift(pass);
  const uint32_t dmask = (1u << digit_bits(pass)) - 1u;
  const int hi = sft + digit_bits(pass);
  const uint32_t prefix = st->prefix;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < N;
       g += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t k = order_key(imp[g]);
    if (pass == 0 || (k >> hi) == prefix) atomicAdd(&sh[(k >> sft) & dmask], 1u);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < kBins; b += blockDim.x)
    if (sh[b]) atomicAdd(&hist[b], sh[b]);
}

// One warp: find the bin holding the remaining rank, extend the prefix, clear
// the histogram for the next pass.
__global__ void select_pick_kernel(int pass, SelectState* st, uint32_t* hist) {
  const int lane = threadIdx.x;
  const int nb = 1 << digit_bits(pass);
  const int per = nb / 32;
  uint32_t local = 0;
  for (int b = 0; b < per; ++b) local += hist[lane * per + b];
  const uint32_t inc = warp_inclusive_scan(local);
  const uint32_t exc = inc - local;
  const uint32_t rank = st->rank;
  const bool mine = rank >= exc && rank < inc;
  const unsigned owner = __ballot_sync(0xffffffffu, mine);
  if (owner != 0 && lane == __ffs(owner) - 1) {
    uint32_t c = exc;
    int b = lane * per;
    for (; b < lane * per + per; ++b) {
      const uint32_t h = hist[b];
      if (rank < c + h) break;
      c += h;
    }
    st->prefix = (st->prefix << digit_bits(pass)) | (uint32_t)b;
    st->rank = rank - c;
  }
  __syncwarp();
  for (int b = lane; b < kBins; b += 32) hist[b] = 0;
}

__global__ void select_init_kernel(SelectState* st, uint32_t rank, uint32_t enabled, uint32_t* hist) {
  if (threadIdx.x == 0) {
    st->prefix = 0;
    st->rank = rank;
    st->enabled = enabled;
  }
  for (int b = threadIdx.x; b < kBins; b += blockDim.x) hist[b] = 0;
}

struct MaskArgs {
  const float* means;
  const float* imp;
  int64_t N;
  float cx, cy, cz, dd;
  int use_lod;
  const SelectState* st;
  uint8_t* mask;
  uint32_t* partials;
};

__device__ __forceinline__ bool keep_of(const MaskArgs& a, int64_t g, float tau) {
  bool keep = true;
  if (a.use_lod) {
    const float dx = __fsub_rn(a.means[g], a.cx);
    const float dy = __fsub_rn(a.means[a.N + g], a.cy);
    const float dz = __fsub_rn(a.means[2 * a.N + g], a.cz);
    const float s2 = __fadd_rn(__fadd_rn(__fmul_rn(dx, dx), __fmul_rn(dy, dy)), __fmul_rn(dz, dz));
    keep = s2 <= a.dd;
  }
  if (a.st->enabled) keep = keep && (a.imp[g] >= tau);
  return keep;
}

__global__ void __launch_bounds__(kMaskBlock) mask_kernel(MaskArgs a) {
  __shared__ uint32_t scratch[kMaskBlock / 32 + 1];
  const float tau = from_order_key(a.st->prefix);
  const int64_t base = (int64_t)blockIdx.x * kMaskTile;
  uint32_t cnt = 0;
#pragma unroll 4
  for (int j = 0; j < kMaskItems; ++j) {
    const int64_t g = base + j * kMaskBlock + threadIdx.x;
    if (g < a.N) {
      const bool k = keep_of(a, g, tau);
      a.mask[g] = k ? 1 : 0;
      cnt += k;
    }
  }
  const uint32_t total = block_sum<uint32_t, kMaskBlock>(cnt, scratch);
  if (threadIdx.x == 0) a.partials[blockIdx.x] = total;
}

// Exclusive scan of the per-block counts (single block); n_active = total.
__global__ void __launch_bounds__(1024) scan_partials_kernel(uint32_t* partials, int nb, int32_t* n_active) {
  __shared__ uint32_t scratch[1024 / 32 + 1];
  uint32_t carry = 0;
  for (int base = 0; base < nb; base += 1024) {
    const int b = base + threadIdx.x;
    const uint32_t v = b < nb ? partials[b] : 0u;
    uint32_t total;
    const uint32_t ex = block_exclusive_scan<uint32_t, 1024>(v, total, scratch);
    if (b < nb) partials[b] = carry + ex;
    carry += total;
  }
  if (threadIdx.x == 0) *n_active = (int32_t)carry;
}

__global__ void __launch_bounds__(kMaskBlock) compact_kernel(const uint8_t* mask, int64_t N,
                                                             const uint32_t* partials, int32_t* active) {
  __shared__ uint32_t scratch[kMaskBlock / 32 + 1];
  const int64_t base = (int64_t)blockIdx.x * kMaskTile;
  uint32_t offset = partials[blockIdx.x];
  for (int j = 0; j < kMaskItems; ++j) {
    const int64_t g = base + j * kMaskBlock + threadIdx.x;
    const uint32_t k = (g < N && mask[g]) ? 1u : 0u;
    uint32_t total;
    const uint32_t ex = block_exclusive_scan<uint32_t, kMaskBlock>(k, total, scratch);
    if (k) active[offset + ex] = (int32_t)g;
    offset += total;
  }
}

}  // namespace

size_t cull_workspace_bytes(int64_t N) {
  const int64_t nb = (N + kMaskTile - 1) / kMaskTile;
  return align256(kBins * sizeof(uint32_t)) + align256(sizeof(SelectState)) +
         align256((size_t)(nb + 1) * sizeof(uint32_t));
}

cudaError_t launch_cull(const float* means, const float* importance, int64_t N, const DevCam& cam,
                        float lod_dist, float q, uint8_t* mask, int32_t* active_idx,
                        int32_t* n_active, void* ws, cudaStream_t s) {
  CullWs w = carve(ws, N);
  const bool use_imp = q > 0.0f && N > 0;
  const uint32_t rank = use_imp ? (uint32_t)std::floor((double)q * (double)N) : 0u;
  select_init_kernel<<<1, 256, 0, s>>>(w.state, rank, use_imp ? 1u : 0u, w.hist);
  count_launches(1);
  if (use_imp) {
    const unsigned grid = (unsigned)std::min<int64_t>(grid_for(N, 256), 148 * 8);
    for (int pass = 0; pass < 3; ++pass) {
      select_hist_kernel<<<grid, 256, 0, s>>>(importance, N, pass, w.state, w.hist);
      select_pick_kernel<<<1, 32, 0, s>>>(pass, w.state, w.hist);
    }
    count_launches(6);
  }
  const int64_t nb = (N + kMaskTile - 1) / kMaskTile;
  if (nb > 0) {
    MaskArgs a;
    a.means = means; a.imp = importance; a.N = N;
    a.cx = cam.campos[0]; a.cy = cam.campos[1]; a.cz = cam.campos[2];
    a.dd = lod_dist * lod_dist;
    a.use_lod = lod_dist > 0.0f;
    a.st = w.state; a.mask = mask; a.partials = w.partials;
    mask_kernel<<<(unsigned)nb, kMaskBlock, 0, s>>>(a);
  }
  scan_partials_kernel<<<1, 1024, 0, s>>>(w.partials, (int)nb, n_active);
  if (nb > 0) compact_kernel<<<(unsigned)nb, kMaskBlock, 0, s>>>(mask, N, w.partials, active_idx);
  count_launches(nb > 0 ? 3 : 1);
  return cudaGetLastError();
}

}  // namespace gs
