// Tile binning: scan of tiles_touched, key emission, stable LSD radix sort of
// the 64-bit (tile_id << 32 | depth bits) keys, and per-tile ranges.
//
// Sort: one histogram kernel reads every key once and builds the 256-bin
// digit histograms of all passes; each pass is then a single "onesweep"
// kernel. A CTA takes the next 4096-key tile (atomic ticket, so all earlier
// tiles are already resident), ranks its keys per digit with warp match-any,
// publishes its per-digit counts and finds its global offsets by decoupled
// look-back over the predecessors' published counts, then scatters through
// shared memory so that writes of equal digits are contiguous. Every
// look-back wait is bounded: past the limit the CTA records
// GS_ERR_DEVICE_TIMEOUT in the status word and carries on without hanging.
// Only the bits [0, 32 + ceil(log2 tiles)) are sorted (8-bit digits).

#include "gs_internal.cuh"
#include "scan_util.cuh"

#include <algorithm>

namespace gs {
namespace {

constexpr int kScanBlock = 256;
constexpr int kScanItems = 16;
constexpr int kScanTile = kScanBlock * kScanItems;
constexpr int kSortBlock = 256;
constexpr int kSortItems = 16;
constexpr int kSortTile = kSortBlock * kSortItems;  // 4096
constexpr int kSortWarps = kSortBlock / 32;
constexpr int kRadix = 256;
constexpr int kMaxPasses = 8;
constexpr uint32_t kValMask = (1u << 30) - 1u;
constexpr uint32_t kFlagAgg = 1u << 30;
constexpr uint32_t kFlagInc = 2u << 30;
constexpr uint32_t kSpinLimit = 1u << 20;
constexpr size_t kSortSmem = (size_t)kSortTile * (sizeof(uint64_t) + sizeof(uint32_t));

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct SortWs {
  int64_t* partials;   // [n_scan_blocks + 1]
  int64_t* total;      // [1]
  int32_t* status;     // [1]
  uint32_t* hist;      // [kMaxPasses][kRadix]
  uint32_t* counters;  // [kMaxPasses], directly followed by lookback
  uint32_t* lookback;  // [passes][n_tiles][kRadix]
  uint64_t* keys_alt;  // [capacity]
  uint32_t* vals_alt;  // [capacity]
};

int64_t scan_blocks(int64_t n) { return (n + kScanTile - 1) / kScanTile; }
int64_t sort_tiles(int64_t n) { return (n + kSortTile - 1) / kSortTile; }

SortWs carve(void* ws, const BinSortPlan& p) {
  char* c = static_cast<char*>(ws);
  SortWs w;
  w.partials = reinterpret_cast<int64_t*>(c);
  c += align256((size_t)(scan_blocks(p.n) + 1) * sizeof(int64_t));
  w.total = reinterpret_cast<int64_t*>(c);
  c += 256;
  w.status = reinterpret_cast<int32_t*>(c);
  c += 256;
  w.hist = reinterpret_cast<uint32_t*>(c);
  c += align256(kMaxPasses * kRadix * sizeof(uint32_t));
  w.counters = reinterpret_cast<uint32_t*>(c);
  w.lookback = w.counters + 64;
  c += align256((64 + (size_t)p.passes * sort_tiles(p.capacity) * kRadix) * sizeof(uint32_t));
  w.keys_alt = reinterpret_cast<uint64_t*>(c);
  c += align256((size_t)p.capacity * sizeof(uint64_t));
  w.vals_alt = reinterpret_cast<uint32_t*>(c);
  return w;
}

__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------- scan
__global__ void __launch_bounds__(kScanBlock) scan_reduce_kernel(const int32_t* tiles, int64_t n,
                                                                 int64_t* partials) {
  __shared__ int64_t scratch[kScanBlock / 32 + 1];
  const int64_t base = (int64_t)blockIdx.x * kScanTile;
  int64_t s = 0;
#pragma unroll 4
  for (int j = 0; j < kScanItems; ++j) {
    const int64_t i = base + j * kScanBlock + threadIdx.x;
    if (i < n) s += tiles[i];
  }
  const int64_t tot = block_sum<int64_t, kScanBlock>(s, scratch);
  if (threadIdx.x == 0) partials[blockIdx.x] = tot;
}

__global__ void __launch_bounds__(1024) scan_partials_kernel(int64_t* partials, int64_t nb, int64_t* total) {
  __shared__ int64_t scratch[1024 / 32 + 1];
  int64_t carry = 0;
  for (int64_t base = 0; base < nb; base += 1024) {
    const int64_t b = base + threadIdx.x;
    const int64_t v = b < nb ? partials[b] : 0;
    int64_t t;
    const int64_t ex = block_exclusive_scan<int64_t, 1024>(v, t, scratch);
    if (b < nb) partials[b] = carry + ex;
    carry += t;
  }
  if (threadIdx.x == 0) *total = carry;
}

__global__ void __launch_bounds__(kScanBlock) scan_down_kernel(const int32_t* tiles, int64_t n,
                                                               const int64_t* partials, int32_t* offsets) {
  __shared__ int64_t scratch[kScanBlock / 32 + 1];
  const int64_t base = (int64_t)blockIdx.x * kScanTile;
  int64_t run = partials[blockIdx.x];
  for (int j = 0; j < kScanItems; ++j) {
    const int64_t i = base + j * kScanBlock + threadIdx.x;
    const int64_t v = i < n ? (int64_t)tiles[i] : 0;
    int64_t t;
    const int64_t ex = block_exclusive_scan<int64_t, kScanBlock>(v, t, scratch);
    if (i < n) offsets[i] = (int32_t)(run + ex);
    run += t;
  }
}

// ---------------------------------------------------------------- emission
__global__ void __launch_bounds__(256) emit_kernel(const float4* xyzo, const ushort4* rect,
                                                   const int32_t* tiles, const int32_t* offsets,
                                                   int64_t n, int TW, uint64_t* keys, uint32_t* vals) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n || tiles[i] <= 0) return;
  int64_t off = offsets[i];
  const uint64_t dbits = __float_as_uint(xyzo[i].z);
  const ushort4 r = rect[i];
  for (int ty = r.y; ty < r.w; ++ty)
    for (int tx = r.x; tx < r.z; ++tx) {
      keys[off] = ((uint64_t)(ty * TW + tx) << 32) | dbits;
      vals[off] = (uint32_t)i;
      ++off;
    }
}

// ---------------------------------------------------------------- histogram
__global__ void __launch_bounds__(256) digit_hist_kernel(const uint64_t* keys, int64_t n, int passes,
                                                         uint32_t* hist) {
  __shared__ uint32_t sh[kMaxPasses * kRadix];
  for (int b = threadIdx.x; b < kMaxPasses * kRadix; b += blockDim.x) sh[b] = 0;
  __syncthreads();
  for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n;
       k += (int64_t)gridDim.x * blockDim.x) {
    const uint64_t key = keys[k];
    for (int p = 0; p < passes; ++p) atomicAdd(&sh[p * kRadix + (uint32_t)((key >> (8 * p)) & 255u)], 1u);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < passes * kRadix; b += blockDim.x)
    if (sh[b]) atomicAdd(&hist[b], sh[b]);
}

__global__ void __launch_bounds__(kRadix) digit_offsets_kernel(uint32_t* hist) {
  __shared__ uint32_t scratch[kRadix / 32 + 1];
  uint32_t* h = hist + blockIdx.x * kRadix;
  const uint32_t v = h[threadIdx.x];
  uint32_t t;
  const uint32_t ex = block_exclusive_scan<uint32_t, kRadix>(v, t, scratch);
  h[threadIdx.x] = ex;
}

// ---------------------------------------------------------------- onesweep
struct PassArgs {
  const uint64_t* kin;
  const uint32_t* vin;
  uint64_t* kout;
  uint32_t* vout;
  int64_t n;
  int shift;
  const uint32_t* digit_off;  // [256] exclusive global digit offsets
  uint32_t* lookback;         // [n_tiles][256]
  uint32_t* counter;
  int32_t* status;
  int64_t stall_tile;
};

__global__ void __launch_bounds__(kSortBlock) onesweep_kernel(PassArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint64_t* s_keys = reinterpret_cast<uint64_t*>(smem);
  uint32_t* s_vals = reinterpret_cast<uint32_t*>(smem + (size_t)kSortTile * sizeof(uint64_t));
  __shared__ uint32_t s_whist[kSortWarps][kRadix];
  __shared__ uint32_t s_dstart[kRadix];
  __shared__ uint32_t s_gbase[kRadix];
  __shared__ uint32_t s_scan[kSortWarps + 1];
  __shared__ uint32_t s_tile;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) s_tile = atomicAdd(a.counter, 1u);
  for (int b = tid; b < kSortWarps * kRadix; b += kSortBlock) (&s_whist[0][0])[b] = 0;
  __syncthreads();
  const int64_t tile = s_tile;
  const int64_t base = tile * kSortTile;

  uint64_t key[kSortItems];
  uint32_t val[kSortItems];
  uint32_t dig[kSortItems];
  uint32_t rank[kSortItems];
#pragma unroll
  for (int j = 0; j < kSortItems; ++j) {
    const int64_t idx = base + warp * (kSortItems * 32) + j * 32 + lane;
    const bool ok = idx < a.n;
    key[j] = ok ? a.kin[idx] : 0ull;
    val[j] = ok ? a.vin[idx] : 0u;
    dig[j] = ok ? (uint32_t)((key[j] >> a.shift) & 255u) : (uint32_t)kRadix;
  }
  // Rank within the warp, in (j, lane) order = original order.
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < kSortItems; ++j) {
    const uint32_t d = dig[j];
    const uint32_t peers = __match_any_sync(0xffffffffu, d);
    const uint32_t pre = d < kRadix ? s_whist[warp][d] : 0u;
    __syncwarp();
    if (d < kRadix && lane == 31 - __clz(peers)) s_whist[warp][d] = pre + __popc(peers);
    __syncwarp();
    rank[j] = pre + __popc(peers & lt);
  }
  __syncthreads();
  // Per digit (thread d): exclusive offsets of the warps, block count.
  const int d = tid;
  uint32_t cnt = 0;
#pragma unroll
  for (int w = 0; w < kSortWarps; ++w) {
    const uint32_t c = s_whist[w][d];
    s_whist[w][d] = cnt;
    cnt += c;
  }
  uint32_t blk_total;
  const uint32_t dstart = block_exclusive_scan<uint32_t, kSortBlock>(cnt, blk_total, s_scan);
  s_dstart[d] = dstart;
  // Decoupled look-back for digit d.
  const bool stall = tile == a.stall_tile;
  uint32_t* row = a.lookback + (size_t)tile * kRadix;
  uint32_t excl = 0;
  if (tile == 0) {
    if (!stall) st_relaxed(row + d, kFlagInc | cnt);
  } else {
    if (!stall) st_relaxed(row + d, kFlagAgg | cnt);
    int64_t k = tile - 1;
    uint32_t spins = 0;
    while (true) {
      const uint32_t s = ld_relaxed(a.lookback + (size_t)k * kRadix + d);
      const uint32_t flag = s & ~kValMask;
      if (flag == 0u) {
        if (++spins > kSpinLimit) {
          atomicExch(a.status, (int32_t)GS_ERR_DEVICE_TIMEOUT);
          break;
        }
        __nanosleep(64);
        continue;
      }
      excl += s & kValMask;
      if (flag == kFlagInc || k == 0) break;
      --k;
    }
    if (!stall) st_relaxed(row + d, kFlagInc | ((excl + cnt) & kValMask));
  }
  s_gbase[d] = a.digit_off[d] + excl;
  __syncthreads();
  // Scatter into shared memory in digit order.
#pragma unroll
  for (int j = 0; j < kSortItems; ++j) {
    const uint32_t dj = dig[j];
    if (dj < kRadix) {
      const uint32_t pos = s_dstart[dj] + s_whist[warp][dj] + rank[j];
      s_keys[pos] = key[j];
      s_vals[pos] = val[j];
    }
  }
  __syncthreads();
  const int64_t rem = a.n - base;
  const int items = rem < kSortTile ? (int)rem : kSortTile;
  for (int s = tid; s < items; s += kSortBlock) {
    const uint64_t k = s_keys[s];
    const uint32_t dd = (uint32_t)((k >> a.shift) & 255u);
    const uint32_t out = s_gbase[dd] + ((uint32_t)s - s_dstart[dd]);
    a.kout[out] = k;
    a.vout[out] = s_vals[s];
  }
}

// ---------------------------------------------------------------- ranges
__global__ void __launch_bounds__(256) ranges_kernel(const uint64_t* keys, int64_t n, int64_t TT,
                                                     uint2* ranges) {
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= n) return;
  const uint64_t tile = keys[k] >> 32;
  if (tile >= (uint64_t)TT) return;
  const uint64_t prev = k > 0 ? (keys[k - 1] >> 32) : ~0ull;
  const uint64_t next = k + 1 < n ? (keys[k + 1] >> 32) : ~0ull;
  if (prev != tile) ranges[tile].x = (uint32_t)k;
  if (next != tile) ranges[tile].y = (uint32_t)(k + 1);
}

}  // namespace

BinSortPlan binsort_plan(int64_t n, int64_t capacity, int64_t tiles) {
  BinSortPlan p;
  p.n = n;
  p.capacity = capacity;
  p.tiles = tiles;
  int tb = 0;
  while ((int64_t(1) << tb) < tiles) ++tb;
  p.tile_bits = tb;
  p.passes = (32 + tb + 7) / 8;
  p.bytes = align256((size_t)(scan_blocks(n) + 1) * sizeof(int64_t)) + 256 + 256 +
            align256(kMaxPasses * kRadix * sizeof(uint32_t)) +
            align256((64 + (size_t)p.passes * sort_tiles(capacity) * kRadix) * sizeof(uint32_t)) +
            align256((size_t)capacity * sizeof(uint64_t)) + align256((size_t)capacity * sizeof(uint32_t));
  return p;
}

const int64_t* binsort_total_ptr(void* ws, const BinSortPlan& plan) { return carve(ws, plan).total; }
const int32_t* binsort_status_ptr(void* ws, const BinSortPlan& plan) { return carve(ws, plan).status; }

cudaError_t launch_scan_tiles(const int32_t* tiles, int64_t n, int32_t* offsets, void* ws,
                              const BinSortPlan& plan, cudaStream_t s) {
  SortWs w = carve(ws, plan);
  const int64_t nb = scan_blocks(n);
  cudaError_t e = cudaMemsetAsync(w.status, 0, sizeof(int32_t), s);
  if (e != cudaSuccess) return e;
  if (nb > 0) scan_reduce_kernel<<<(unsigned)nb, kScanBlock, 0, s>>>(tiles, n, w.partials);
  scan_partials_kernel<<<1, 1024, 0, s>>>(w.partials, nb, w.total);
  if (nb > 0) scan_down_kernel<<<(unsigned)nb, kScanBlock, 0, s>>>(tiles, n, w.partials, offsets);
  count_launches(nb > 0 ? 3 : 1);
  return cudaGetLastError();
}

cudaError_t launch_emit_sort_ranges(const Records& rec, int64_t n, const int32_t* offsets,
                                    const DevCam& cam, int64_t n_inst, uint64_t* keys,
                                    uint32_t* vals, uint32_t* ranges, void* ws,
                                    const BinSortPlan& plan, int64_t stall_tile, cudaStream_t s) {
  SortWs w = carve(ws, plan);
  const int64_t TT = (int64_t)cam.TW * cam.TH;
  cudaError_t e = cudaMemsetAsync(ranges, 0, (size_t)TT * 2 * sizeof(uint32_t), s);
  if (e != cudaSuccess || n_inst == 0) return e;
  const int P = plan.passes;
  uint64_t* kb[2];
  uint32_t* vb[2];
  kb[0] = (P % 2 == 0) ? keys : w.keys_alt;
  vb[0] = (P % 2 == 0) ? vals : w.vals_alt;
  kb[1] = (P % 2 == 0) ? w.keys_alt : keys;
  vb[1] = (P % 2 == 0) ? w.vals_alt : vals;
  emit_kernel<<<grid_for(n, 256), 256, 0, s>>>(rec.xyzo, rec.rect, rec.tiles, offsets, n, cam.TW, kb[0], vb[0]);
  e = cudaMemsetAsync(w.hist, 0, kMaxPasses * kRadix * sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;
  const unsigned hgrid = (unsigned)std::min<int64_t>(grid_for(n_inst, 256), 148 * 4);
  digit_hist_kernel<<<hgrid, 256, 0, s>>>(kb[0], n_inst, P, w.hist);
  digit_offsets_kernel<<<P, kRadix, 0, s>>>(w.hist);
  const int64_t ntiles = sort_tiles(n_inst);
  // counters and the look-back words of this call's passes: [P][ntiles][256]
  e = cudaMemsetAsync(w.counters, 0, (64 + (size_t)P * ntiles * kRadix) * sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(onesweep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSortSmem);
  if (e != cudaSuccess) return e;
  for (int p = 0; p < P; ++p) {
    PassArgs a;
    a.kin = kb[p & 1];
    a.vin = vb[p & 1];
    a.kout = kb[(p + 1) & 1];
    a.vout = vb[(p + 1) & 1];
    a.n = n_inst;
    a.shift = 8 * p;
    a.digit_off = w.hist + p * kRadix;
    a.lookback = w.lookback + (size_t)p * ntiles * kRadix;
    a.counter = w.counters + p;
    a.status = w.status;
    a.stall_tile = stall_tile;
    onesweep_kernel<<<(unsigned)ntiles, kSortBlock, kSortSmem, s>>>(a);
  }
  ranges_kernel<<<grid_for(n_inst, 256), 256, 0, s>>>(keys, n_inst, TT, reinterpret_cast<uint2*>(ranges));
  count_launches(4 + P);
  return cudaGetLastError();
}

}  // namespace gs
