// Tile binning: the (tile_id << 32 | depth bits) keys of every (Gaussian,
// tile) instance, stably sorted, and per-tile ranges.
//
// An LSD radix sort of the 64-bit keys first sorts by the 32 depth bits and
// then by the tile bits. All instances of one Gaussian share its depth bits,
// so the depth passes are run on the Gaussians (one 32-bit key each) before
// the instances are expanded; instances are then emitted in (depth, index)
// order and only the ceil(log2 tiles) tile bits are sorted over the
// instances. Stability makes the result identical to the full 64-bit sort:
// ascending (tile, depth, record index). At 1080p with ~6 instances per
// Gaussian this moves ~1/4 of the bytes of sorting all key bits per instance.
//
// Stages: the visible records' depth keys, compacted in record order (so a
// cull that leaves few records visible sorts few keys); 4 depth passes; a
// scan of tiles_touched in depth order, which also records the Gaussian of
// every 256-instance chunk's first instance; the emission, partitioned by
// instance so that Gaussians touching thousands of tiles are shared by many
// warps; the tile passes over 32-bit tile ids; and the ranges kernel, which
// finds each tile's run and writes the final 64-bit keys.
//
// Each sort pass is one "onesweep" kernel: a CTA takes the next 4096-key tile
// (atomic ticket, so all earlier tiles are already resident), ranks its keys
// per digit with warp ballots, publishes its per-digit counts and finds its
// global offsets by decoupled look-back over its predecessors' counts, then
// scatters through shared memory so that writes of equal digits are
// contiguous. Every look-back wait is bounded: past the limit the CTA records
// GS_ERR_DEVICE_TIMEOUT in the status word and carries on without hanging.
// A single histogram kernel per sort builds the digit counts of all passes.

#include "checked.cuh"
#include "gs_internal.cuh"
#include "scan_util.cuh"

#include <algorithm>

namespace gs {
namespace {

constexpr int kScanBlock = 256;
constexpr int kScanItems = 16;
constexpr int kScanTile = kScanBlock * kScanItems;
constexpr int kVisTile = 1024;  // records per CTA of the visible-record compaction
constexpr int kVisRows = kVisTile / kScanBlock;
constexpr int kEmitChunk = 256;  // instances per warp of the emission
constexpr int kSortBlock = 512;
constexpr int kSortItems = 8;
constexpr int kSortTile = kSortBlock * kSortItems;  // 4096
constexpr int kSortWarps = kSortBlock / 32;
constexpr int kRadix = 256;
constexpr int kMaxPasses = 8;
constexpr int kDepthPasses = 4;
constexpr uint32_t kValMask = (1u << 30) - 1u;
constexpr uint32_t kFlagAgg = 1u << 30;
constexpr uint32_t kFlagInc = 2u << 30;
constexpr uint32_t kSpinLimit = 1u << 20;
constexpr int kLookAhead = 4;  // look-back words read per poll
constexpr uint32_t kInvisibleKey = 0xffffffffu;

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int64_t scan_blocks(int64_t n) { return (n + kScanTile - 1) / kScanTile; }
int64_t vis_blocks(int64_t n) { return (n + kVisTile - 1) / kVisTile; }
int64_t emit_chunks(int64_t capacity) { return (capacity + kEmitChunk - 1) / kEmitChunk + 1; }
// entries of the partials buffer: the scans' and the compaction's blocks
int64_t partial_slots(int64_t n) { return std::max(scan_blocks(n), vis_blocks(n)) + 1; }
int64_t sort_tiles(int64_t n) { return (n + kSortTile - 1) / kSortTile; }

struct SortWs {
  int64_t* partials;   // [scan blocks + 1]
  int64_t* total;      // [2]: instances, then visible records
  int32_t* status;     // [1]
  uint32_t* hist;      // [kMaxPasses][kRadix]
  uint32_t* counters;  // [64], directly followed by the look-back words
  uint32_t* lookback;  // [passes][sort tiles][kRadix]
  uint32_t* dkey[2];   // [n] depth keys
  uint32_t* dval[2];   // [n] record indices
  int32_t* doff;       // [n] instance offsets in depth order
  int32_t* dtiles;     // [n] tiles_touched in depth order
  int32_t* chunk_g;    // [emit chunks] depth position of each emit chunk's first instance
  uint32_t* tkey[2];   // [capacity] tile ids
  uint32_t* tval[2];   // [capacity] record indices
};

size_t lookback_words(const BinSortPlan& p) {
  const size_t a = (size_t)kDepthPasses * sort_tiles(p.n);
  const size_t b = (size_t)std::max(p.passes, 1) * sort_tiles(p.capacity);
  return 64 + std::max(a, b) * kRadix;
}

SortWs carve(void* ws, const BinSortPlan& p) {
  char* c = static_cast<char*>(ws);
  SortWs w;
  w.partials = reinterpret_cast<int64_t*>(c);
  c += align256((size_t)partial_slots(p.n) * sizeof(int64_t));
  w.total = reinterpret_cast<int64_t*>(c);
  c += 256;
  w.status = reinterpret_cast<int32_t*>(c);
  c += 256;
  w.hist = reinterpret_cast<uint32_t*>(c);
  c += align256(kMaxPasses * kRadix * sizeof(uint32_t));
  w.counters = reinterpret_cast<uint32_t*>(c);
  w.lookback = w.counters + 64;
  c += align256(lookback_words(p) * sizeof(uint32_t));
  for (int k = 0; k < 2; ++k) {
    w.dkey[k] = reinterpret_cast<uint32_t*>(c);
    c += align256((size_t)p.n * sizeof(uint32_t));
    w.dval[k] = reinterpret_cast<uint32_t*>(c);
    c += align256((size_t)p.n * sizeof(uint32_t));
  }
  w.doff = reinterpret_cast<int32_t*>(c);
  c += align256((size_t)p.n * sizeof(int32_t));
  w.dtiles = reinterpret_cast<int32_t*>(c);
  c += align256((size_t)p.n * sizeof(int32_t));
  w.chunk_g = reinterpret_cast<int32_t*>(c);
  c += align256((size_t)emit_chunks(p.capacity) * sizeof(int32_t));
  for (int k = 0; k < 2; ++k) {
    w.tkey[k] = reinterpret_cast<uint32_t*>(c);
    c += align256((size_t)p.capacity * sizeof(uint32_t));
    w.tval[k] = reinterpret_cast<uint32_t*>(c);
    c += align256((size_t)p.capacity * sizeof(uint32_t));
  }
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

// Instances to emit and sort, read on the device so that no host round trip
// sits between the count and the sort: the scan's total, or none when it
// exceeds the capacity (the emit kernel then records GS_ERR_CAPACITY).
__device__ __forceinline__ int64_t live_instances(const int64_t* total, int64_t capacity) {
  const int64_t t = *total;
  return t <= capacity ? t : 0;
}

// ---------------------------------------------------------------- scans
// Exclusive scan of tiles[order[r]] (order == nullptr: identity).
__global__ void __launch_bounds__(kScanBlock) scan_reduce_kernel(const int32_t* tiles, const uint32_t* order,
                                                                 int64_t n, const int64_t* n_dev,
                                                                 int64_t* partials) {
  __shared__ int64_t scratch[kScanBlock / 32 + 1];
  if (n_dev && *n_dev < n) n = *n_dev;  // elements past the device count are 0
  const int64_t base = (int64_t)blockIdx.x * kScanTile;
  int64_t s = 0;
#pragma unroll 4
  for (int j = 0; j < kScanItems; ++j) {
    const int64_t r = base + j * kScanBlock + threadIdx.x;
    if (r < n) s += tiles[order ? order[r] : r];
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

// Row j of a CTA's tile holds elements base + j kScanBlock + [0, kScanBlock):
// every load and store is coalesced. Each warp scans its 32 elements of every
// row with shuffles; one warp then scans the (row, warp) totals in element
// order, so the whole tile needs two CTA barriers.
__global__ void __launch_bounds__(kScanBlock) scan_down_kernel(const int32_t* tiles, const uint32_t* order,
                                                               int64_t n, const int64_t* partials,
                                                               int32_t* offsets, int32_t* chunk_g,
                                                               int64_t n_chunks, const int64_t* n_dev) {
  constexpr int kWarps = kScanBlock / 32;
  constexpr int kParts = kScanItems * kWarps;  // (row, warp) pieces in element order
  static_assert(kParts == 4 * 32, "one warp scans the pieces, four per lane");
  __shared__ int64_t s_part[kParts];
  if (n_dev && *n_dev < n) n = *n_dev;  // elements past the device count are 0 (and not written)
  const int64_t base = (int64_t)blockIdx.x * kScanTile;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t ex[kScanItems];  // the element first, then its exclusive prefix in the warp's row
#pragma unroll
  for (int j = 0; j < kScanItems; ++j) {
    const int64_t r = base + j * kScanBlock + threadIdx.x;
    ex[j] = r < n ? tiles[order ? order[r] : r] : 0;
  }
#pragma unroll
  for (int j = 0; j < kScanItems; ++j) {
    int32_t x = ex[j];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    ex[j] = x - ex[j];
    if (lane == 31) s_part[j * kWarps + warp] = x;
  }
  __syncthreads();
  if (warp == 0) {
    const int64_t a0 = s_part[4 * lane], a1 = s_part[4 * lane + 1], a2 = s_part[4 * lane + 2],
                  a3 = s_part[4 * lane + 3];
    int64_t x = a0 + a1 + a2 + a3;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    const int64_t e = x - (a0 + a1 + a2 + a3) + partials[blockIdx.x];
    s_part[4 * lane] = e;
    s_part[4 * lane + 1] = e + a0;
    s_part[4 * lane + 2] = e + a0 + a1;
    s_part[4 * lane + 3] = e + a0 + a1 + a2;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kScanItems; ++j) {
    const int64_t r = base + j * kScanBlock + threadIdx.x;
    if (r < n) {
      const int64_t off = s_part[j * kWarps + warp] + ex[j];
      offsets[r] = (int32_t)off;
      if (chunk_g) {  // element r holds the first instance of every emit chunk that starts in its range
        const int64_t end = off + tiles[order ? order[r] : r];
        for (int64_t b = (off + kEmitChunk - 1) / kEmitChunk; b * kEmitChunk < end && b < n_chunks; ++b)
          chunk_g[b] = (int32_t)r;
      }
    }
  }
}

// ---------------------------------------------------------------- keys
// The depth sort takes the visible records only (tiles_touched > 0),
// compacted in record order: equal depths then keep record order, so the
// sorted order equals that of a stable sort of all records with the
// invisible ones keyed last, and a cull that leaves few records visible
// sorts few keys. Two passes over tiles_touched: visible records per scan
// block (then scan_partials_kernel), and the compacted keys and values.
__global__ void __launch_bounds__(kScanBlock) vis_count_kernel(const int32_t* tiles, int64_t n, int64_t* partials) {
  __shared__ int64_t scratch[kScanBlock / 32 + 1];
  const int64_t base = (int64_t)blockIdx.x * kVisTile;
  int64_t c = 0;
#pragma unroll
  for (int j = 0; j < kVisRows; ++j) {
    const int64_t r = base + j * kScanBlock + threadIdx.x;
    if (r < n && tiles[r] > 0) ++c;
  }
  const int64_t tot = block_sum<int64_t, kScanBlock>(c, scratch);
  if (threadIdx.x == 0) partials[blockIdx.x] = tot;
}

// Row j of a CTA holds records base + j kScanBlock + [0, kScanBlock): a
// ballot per warp row, then one warp scans the (row, warp) counts, one per
// lane.
__global__ void __launch_bounds__(kScanBlock) vis_compact_kernel(const float4* xyzo, const int32_t* tiles, int64_t n,
                                                                 const int64_t* partials, uint32_t* key,
                                                                 uint32_t* val) {
  constexpr int kWarps = kScanBlock / 32;
  static_assert(kVisRows * kWarps == 32, "one warp scans the pieces, one per lane");
  __shared__ int64_t s_part[32];
  const int64_t base = (int64_t)blockIdx.x * kVisTile;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t vis[kVisRows];  // ballot of the warp's row j
#pragma unroll
  for (int j = 0; j < kVisRows; ++j) {
    const int64_t r = base + j * kScanBlock + threadIdx.x;
    vis[j] = __ballot_sync(0xffffffffu, r < n && tiles[r] > 0);
    if (lane == 0) s_part[j * kWarps + warp] = __popc(vis[j]);
  }
  __syncthreads();
  if (warp == 0) {
    const int64_t a = s_part[lane];
    int64_t x = a;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    s_part[lane] = x - a + partials[blockIdx.x];
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kVisRows; ++j) {
    if ((vis[j] >> lane) & 1u) {
      const int64_t r = base + j * kScanBlock + threadIdx.x;
      const int64_t pos = s_part[j * kWarps + warp] + __popc(vis[j] & lt);
      key[pos] = __float_as_uint(xyzo[r].z);
      val[pos] = (uint32_t)r;
    }
  }
}

// Instances of the Gaussians in depth order, tiles row-major in each rect,
// partitioned by instance: warp w writes instances [w C, (w + 1) C) with
// C = kEmitChunk, so a Gaussian that touches thousands of tiles is shared by
// many warps (near-camera Gaussians sort next to each other, and giving each
// warp whole Gaussians left a few warps with most of the instances). The
// scan of the depth-order counts records the Gaussian of every chunk's first
// instance; the warp walks windows of 32 consecutive Gaussians from it, each
// lane finding the Gaussian of its instance by a binary search over the
// window's offsets; the stores of every step are 32 consecutive slots.
__global__ void __launch_bounds__(256) emit_kernel(const uint32_t* order, const int32_t* doff,
                                                   const int32_t* dtiles, const int32_t* chunk_g,
                                                   const ushort4* rect, int64_t n, const int64_t* nvis, int TW,
                                                   const int64_t* total,
                                                   int64_t capacity, int32_t* status, uint32_t* tkey,
                                                   uint32_t* tval) {
  if (*status != 0) return;  // the depth order is not valid
  const int64_t I = *total;
  if (I > capacity) {  // nothing is emitted or sorted
    if (blockIdx.x == 0 && threadIdx.x == 0) *status = GS_ERR_CAPACITY;
    return;
  }
  const int lane = threadIdx.x & 31;
  const int64_t chunk = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t q0 = chunk * kEmitChunk;
  if (q0 >= I) return;  // warp-uniform
  const int64_t q1 = q0 + kEmitChunk < I ? q0 + kEmitChunk : I;
  const int64_t nd = *nvis < n ? *nvis : n;  // depth positions past the visible records hold nothing
  // the depth position whose instances hold q0 (written by the scan)
  int64_t q = q0;
  for (int64_t g = chunk_g[chunk]; q < q1; g += 32) {
    const int64_t gl = g + lane;
    int32_t off = INT32_MAX;  // lanes past the records never match
    int t = 0, x0 = 0, y0 = 0, bw = 1;
    uint32_t i = 0;
    if (gl < nd) {
      off = doff[gl];
      t = dtiles[gl];
      i = order[gl];
      if (t > 0 && i < n) {
        const ushort4 b = rect[i];
        x0 = b.x;
        y0 = b.y;
        bw = (int)b.z - (int)b.x;
      }
    }
    // the window's instances end where its last Gaussian's end (or all end)
    const int64_t end = __shfl_sync(0xffffffffu, gl < nd ? (int64_t)off + t : I, 31);
    const int64_t qe = end < q1 ? end : q1;
    for (int64_t qs = q; qs < qe; qs += 32) {
      const int64_t qq = qs + lane;
      int L = 0;
#pragma unroll
      for (int st = 16; st > 0; st >>= 1) {
        const int c = L + st;
        if ((int64_t)__shfl_sync(0xffffffffu, off, c) <= qq) L = c;
      }
      const int32_t offL = __shfl_sync(0xffffffffu, off, L);
      const uint32_t iL = __shfl_sync(0xffffffffu, i, L);
      const int x0L = __shfl_sync(0xffffffffu, x0, L);
      const int y0L = __shfl_sync(0xffffffffu, y0, L);
      const int bwL = __shfl_sync(0xffffffffu, bw, L);
      if (qq < qe) {
        const int li = (int)(qq - offL);
        const int row = li / bwL;
        tkey[qq] = (uint32_t)((y0L + row) * TW + x0L + (li - row * bwL));
        tval[qq] = iL;
      }
    }
    q = qe;  // the next window starts where this one's instances end
  }
}

// Digit histograms of `passes` passes (digit p = bits [8p, 8p + 8)).
__global__ void __launch_bounds__(256) digit_hist_kernel(const uint32_t* keys, int64_t n, const int64_t* n_dev,
                                                         int64_t cap, int passes, uint32_t* hist) {
  __shared__ uint32_t sh[kMaxPasses * kRadix];
  if (n_dev) n = live_instances(n_dev, cap);
  for (int b = threadIdx.x; b < kMaxPasses * kRadix; b += blockDim.x) sh[b] = 0;
  __syncthreads();
  // eight keys per thread and step, as two 16-byte loads issued together
  // (the key buffers are 256-byte aligned), so their latencies overlap
  auto count = [&](uint32_t key) {
    for (int p = 0; p < passes; ++p) atomicAdd(&sh[p * kRadix + ((key >> (8 * p)) & 255u)], 1u);
  };
  const int64_t stride = (int64_t)gridDim.x * blockDim.x * 8;
  for (int64_t k = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; k < n; k += stride) {
    if (k + 8 <= n) {
      const uint4 a = *reinterpret_cast<const uint4*>(keys + k);
      const uint4 b = *reinterpret_cast<const uint4*>(keys + k + 4);
      count(a.x); count(a.y); count(a.z); count(a.w);
      count(b.x); count(b.y); count(b.z); count(b.w);
    } else {
      for (int64_t j = k; j < n; ++j) count(keys[j]);
    }
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
  const uint32_t* kin;
  const uint32_t* vin;
  uint32_t* kout;             // next-pass keys
  uint32_t* vout;
  int64_t n_records;          // values index records [0, n_records)
  const int32_t* tiles_in;    // optional: also write tiles_out[out] = tiles_in[value]
  int32_t* tiles_out;
  int64_t n;                  // keys, or (n_dev set) an upper bound on them
  const int64_t* n_dev;       // optional: the key count on the device ...
  int64_t cap;                // ... used only if it is <= cap (else none)
  int shift;
  const uint32_t* digit_off;  // [256] exclusive global digit offsets
  uint32_t* lookback;         // [n_tiles][256]
  uint32_t* counter;
  int32_t* status;
  int64_t stall_tile;
};

// 512 threads of 8 keys each, two CTAs per SM (64 registers): twice the
// resident warps of 256 threads of 16 keys, for the same 4096-key tile and
// look-back. A warp's count of one digit is at most 256 and a digit's
// exclusive offset inside the tile below 4096, so the per-warp counts are
// 16-bit (the CTA's shared memory stays under the 48 KB static limit).
__global__ void __launch_bounds__(kSortBlock, 2) onesweep_kernel(PassArgs a) {
  __shared__ uint32_t s_keys[kSortTile];
  __shared__ uint32_t s_vals[kSortTile];
  __shared__ uint16_t s_whist[kSortWarps][kRadix];
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
  const int64_t n = a.n_dev ? live_instances(a.n_dev, a.cap) : a.n;
  // CTAs past the keys leave (tickets are taken in order, so none that
  // stays waits on them)
  if (base >= n) return;

  uint32_t key[kSortItems], val[kSortItems], dig[kSortItems], rank[kSortItems];
#pragma unroll
  for (int j = 0; j < kSortItems; ++j) {
    const int64_t idx = base + warp * (kSortItems * 32) + j * 32 + lane;
    const bool ok = idx < n;
    key[j] = ok ? a.kin[idx] : 0u;
    val[j] = ok ? a.vin[idx] : 0u;
    dig[j] = ok ? ((key[j] >> a.shift) & 255u) : (uint32_t)kRadix;
  }
  // Rank within the warp, in (j, lane) order = original order. The lanes
  // holding the same digit are found with one ballot per digit bit (plus
  // one for the out-of-range lanes): a fixed cost, where a match-any grows
  // with the number of distinct digits in the warp.
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < kSortItems; ++j) {
    const uint32_t d = dig[j];
    const uint32_t vm = __ballot_sync(0xffffffffu, d < kRadix);
    uint32_t peers = d < kRadix ? vm : ~vm;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const uint32_t bb = __ballot_sync(0xffffffffu, (d >> b) & 1u);
      peers &= ((d >> b) & 1u) ? bb : ~bb;
    }
    const uint32_t pre = d < kRadix ? (uint32_t)s_whist[warp][d] : 0u;
    __syncwarp();
    if (d < kRadix && lane == 31 - __clz(peers)) s_whist[warp][d] = (uint16_t)(pre + __popc(peers));
    __syncwarp();
    rank[j] = pre + __popc(peers & lt);
  }
  __syncthreads();
  // Per digit (thread d < kRadix): exclusive offsets of the warps, block count.
  const int d = tid;
  const bool owner = d < kRadix;
  uint32_t cnt = 0;
  if (owner) {
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) {
      const uint32_t c = s_whist[w][d];
      s_whist[w][d] = (uint16_t)cnt;
      cnt += c;
    }
  }
  uint32_t blk_total;
  const uint32_t dstart = block_exclusive_scan<uint32_t, kSortBlock>(cnt, blk_total, s_scan);
  if (owner) s_dstart[d] = dstart;
  // Decoupled look-back for digit d.
  const bool stall = tile == a.stall_tile;
  uint32_t* row = a.lookback + (size_t)tile * kRadix;
  uint32_t excl = 0;
  if (!owner) {
  } else if (tile == 0) {
    if (!stall) st_relaxed(row + d, kFlagInc | cnt);
  } else {
    if (!stall) st_relaxed(row + d, kFlagAgg | cnt);
    // kLookAhead predecessor words per poll, in flight together; they are
    // taken in order as before: aggregates are added, the first inclusive
    // prefix (or tile 0) ends the walk, and the first word not yet published
    // is polled again, from where the walk stopped.
    int64_t k = tile - 1;
    uint32_t spins = 0;
    while (true) {
      uint32_t w[kLookAhead];
#pragma unroll
      for (int i = 0; i < kLookAhead; ++i)
        w[i] = k - i >= 0 ? ld_relaxed(a.lookback + (size_t)(k - i) * kRadix + d) : 0u;
      int i = 0;
      bool stop = false, pending = false;
#pragma unroll
      for (; i < kLookAhead; ++i) {
        const uint32_t flag = w[i] & ~kValMask;
        if (flag == 0u) {
          pending = true;
          break;
        }
        excl += w[i] & kValMask;
        if (flag == kFlagInc || k - i == 0) {
          stop = true;
          break;
        }
      }
      if (stop) break;
      k -= i;  // past the aggregates taken; at the unpublished word if pending
      if (pending) {
        if (++spins > kSpinLimit) {
          atomicExch(a.status, (int32_t)GS_ERR_DEVICE_TIMEOUT);
          break;
        }
        __nanosleep(64);
      }
    }
    if (!stall) st_relaxed(row + d, kFlagInc | ((excl + cnt) & kValMask));
  }
  if (owner) s_gbase[d] = a.digit_off[d] + excl;
  __syncthreads();
  // Scatter into shared memory in digit order.
#pragma unroll
  for (int j = 0; j < kSortItems; ++j) {
    const uint32_t dj = dig[j];
    if (dj < kRadix) {
      const uint32_t pos = s_dstart[dj] + (uint32_t)s_whist[warp][dj] + rank[j];
      s_keys[pos] = key[j];
      s_vals[pos] = val[j];
    }
  }
  __syncthreads();
  const int64_t rem = n - base;
  const int items = rem < kSortTile ? (int)rem : kSortTile;
  for (int s = tid; s < items; s += kSortBlock) {
    const uint32_t k = s_keys[s];
    const uint32_t dd = (k >> a.shift) & 255u;
    const uint32_t out = s_gbase[dd] + ((uint32_t)s - s_dstart[dd]);
    const uint32_t v = s_vals[s];
    // (values are record indices; the bound only matters after a look-back
    // timeout, when a slot can hold a stale value)
    const bool vok = v < a.n_records;
    if (!check(out < (uint64_t)n, kCheckSortSlot)) continue;
    a.kout[out] = k;
    a.vout[out] = v;
    if (a.tiles_out) a.tiles_out[out] = vok ? a.tiles_in[v] : 0;
  }
}

// Final keys when no tile pass runs (a single tile): (0 << 32) | depth bits.
__global__ void __launch_bounds__(256) finalize_kernel(const uint32_t* tkey, const uint32_t* tval,
                                                       const int64_t* n_dev, int64_t cap, const float4* xyzo,
                                                       uint64_t* keys, uint32_t* vals) {
  const int64_t n = live_instances(n_dev, cap);
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= n) return;
  const uint32_t v = tval[k];
  keys[k] = ((uint64_t)tkey[k] << 32) | __float_as_uint(xyzo[v].z);
  vals[k] = v;
}

// ---------------------------------------------------------------- results
// Copies the instance count and the status word to the caller's result[2].
__global__ void publish_kernel(const int64_t* total, const int32_t* status, int64_t* result) {
  result[0] = *total;
  result[1] = *status;
}

// ---------------------------------------------------------------- ranges
// Tiles stay empty when the sort failed (status set), so a raster call on
// these buffers reads nothing.
// Also writes the final 64-bit keys, (tile << 32) | depth bits of the
// instance's record, from the sorted tile ids and values: a streaming loop
// hides the record gathers better than the last sort pass's scatter would.
__global__ void __launch_bounds__(256) ranges_kernel(const uint32_t* tk, const uint32_t* tv, const float4* xyzo,
                                                     int64_t n_records, uint64_t* keys, const int64_t* n_dev,
                                                     int64_t cap, const int32_t* status, int64_t TT,
                                                     uint2* ranges) {
  if (*status != 0) return;
  const int64_t n = live_instances(n_dev, cap);
  // grid-stride: the grid is sized for a bound, the count is on the device
  for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t tile = tk[k];
    const uint32_t v = tv[k];
    // (the bound only matters after a look-back timeout, when a slot can
    // hold a stale value)
    keys[k] = ((uint64_t)tile << 32) |
              (check(v < n_records, kCheckRecordIndex) ? __float_as_uint(xyzo[v].z) : kInvisibleKey);
    if (tile >= (uint64_t)TT) continue;
    const uint32_t prev = k > 0 ? tk[k - 1] : ~0u;
    const uint32_t next = k + 1 < n ? tk[k + 1] : ~0u;
    if (prev != tile) ranges[tile].x = (uint32_t)k;
    if (next != tile) ranges[tile].y = (uint32_t)(k + 1);
  }
}

// One LSD sort over `passes` 8-bit digits starting at bit 0, keys/values
// ping-ponging between (k0, v0) and (k1, v1); the last pass writes to
// (last_k, last_v). n keys, or with n_dev at most n keys, their
// number read on the device (live_instances(n_dev, n)). Returns the kernels
// launched, -1 on error.
int sort_passes(const SortWs& w, uint32_t* k0, uint32_t* v0, uint32_t* k1, uint32_t* v1, int64_t n,
                const int64_t* n_dev, int passes, uint32_t* last_k, uint32_t* last_v, int64_t n_records,
                const int32_t* tiles_in, int32_t* tiles_out, int64_t stall,
                cudaStream_t s) {
  if (cudaMemsetAsync(w.hist, 0, kMaxPasses * kRadix * sizeof(uint32_t), s) != cudaSuccess) return -1;
  const int64_t nt = sort_tiles(n);
  if (cudaMemsetAsync(w.counters, 0, (64 + (size_t)passes * nt * kRadix) * sizeof(uint32_t), s) != cudaSuccess)
    return -1;
  const unsigned hgrid = (unsigned)std::min<int64_t>(grid_for(n, 256), 148 * 4);
  digit_hist_kernel<<<hgrid, 256, 0, s>>>(k0, n, n_dev, n, passes, w.hist);
  digit_offsets_kernel<<<passes, kRadix, 0, s>>>(w.hist);
  uint32_t* kb[2] = {k0, k1};
  uint32_t* vb[2] = {v0, v1};
  for (int p = 0; p < passes; ++p) {
    const bool last = p == passes - 1;
    PassArgs a;
    a.kin = kb[p & 1];
    a.vin = vb[p & 1];
    a.kout = last ? last_k : kb[(p + 1) & 1];
    a.vout = last ? last_v : vb[(p + 1) & 1];
    a.n_records = n_records;
    a.tiles_in = tiles_in;
    a.tiles_out = last ? tiles_out : nullptr;
    a.n = n;
    a.n_dev = n_dev;
    a.cap = n;
    a.shift = 8 * p;
    a.digit_off = w.hist + p * kRadix;
    a.lookback = w.lookback + (size_t)p * nt * kRadix;
    a.counter = w.counters + p;
    a.status = w.status;
    a.stall_tile = stall;
    onesweep_kernel<<<(unsigned)nt, kSortBlock, 0, s>>>(a);
  }
  if (cudaGetLastError() != cudaSuccess) return -1;
  return 2 + passes;
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
  p.passes = (tb + 7) / 8;  // tile-digit passes over the instances
  p.bytes = align256((size_t)partial_slots(n) * sizeof(int64_t)) + 256 + 256 +
            align256(kMaxPasses * kRadix * sizeof(uint32_t)) + align256(lookback_words(p) * sizeof(uint32_t)) +
            4 * align256((size_t)n * sizeof(uint32_t)) + 2 * align256((size_t)n * sizeof(int32_t)) +
            align256((size_t)emit_chunks(capacity) * sizeof(int32_t)) +
            4 * align256((size_t)capacity * sizeof(uint32_t));
  return p;
}

const int64_t* binsort_total_ptr(void* ws, const BinSortPlan& plan) { return carve(ws, plan).total; }

cudaError_t launch_publish(void* ws, const BinSortPlan& plan, int64_t* result, cudaStream_t s) {
  const SortWs w = carve(ws, plan);
  publish_kernel<<<1, 1, 0, s>>>(w.total, w.status, result);
  count_launches(1);
  return cudaGetLastError();
}
const int32_t* binsort_status_ptr(void* ws, const BinSortPlan& plan) { return carve(ws, plan).status; }

cudaError_t launch_depth_order(const Records& rec, int64_t n, int32_t* offsets, void* ws,
                               const BinSortPlan& plan, int64_t stall_tile, cudaStream_t s) {
  SortWs w = carve(ws, plan);
  cudaError_t e = cudaMemsetAsync(w.status, 0, sizeof(int32_t), s);
  if (e != cudaSuccess) return e;
  const int64_t nb = scan_blocks(n);
  int launched = 0;
  if (offsets && nb > 0) {  // record-order offsets, on request
    scan_reduce_kernel<<<(unsigned)nb, kScanBlock, 0, s>>>(rec.tiles, nullptr, n, nullptr, w.partials);
    scan_partials_kernel<<<1, 1024, 0, s>>>(w.partials, nb, w.total);
    scan_down_kernel<<<(unsigned)nb, kScanBlock, 0, s>>>(rec.tiles, nullptr, n, w.partials, offsets, nullptr, 0,
                                                         nullptr);
    launched += 3;
  }
  if (n > 0) {
    // the visible records' depth keys, compacted; their count in nvis
    int64_t* nvis = w.total + 1;
    const int64_t nv = vis_blocks(n);
    vis_count_kernel<<<(unsigned)nv, kScanBlock, 0, s>>>(rec.tiles, n, w.partials);
    scan_partials_kernel<<<1, 1024, 0, s>>>(w.partials, nv, nvis);
    vis_compact_kernel<<<(unsigned)nv, kScanBlock, 0, s>>>(rec.xyzo, rec.tiles, n, w.partials, w.dkey[0], w.dval[0]);
    // 4 passes over the nvis keys: dkey[0] -> [1] -> [0] -> [1] -> [0]
    // the last pass also writes tiles_touched in depth order (dtiles)
    const int k = sort_passes(w, w.dkey[0], w.dval[0], w.dkey[1], w.dval[1], n, nvis, kDepthPasses, w.dkey[0],
                              w.dval[0], n, rec.tiles, w.dtiles, stall_tile, s);
    if (k < 0) return cudaErrorLaunchFailure;
    launched += 3 + k;
    scan_reduce_kernel<<<(unsigned)nb, kScanBlock, 0, s>>>(w.dtiles, nullptr, n, w.total + 1, w.partials);
    launched += 1;
  }
  scan_partials_kernel<<<1, 1024, 0, s>>>(w.partials, nb, w.total);
  launched += 1;
  if (nb > 0) {
    scan_down_kernel<<<(unsigned)nb, kScanBlock, 0, s>>>(w.dtiles, nullptr, n, w.partials, w.doff, w.chunk_g,
                                                         emit_chunks(plan.capacity), w.total + 1);
    launched += 1;
  }
  count_launches(launched);
  return cudaGetLastError();
}

cudaError_t launch_emit_sort_ranges(const Records& rec, int64_t n, const DevCam& cam, uint64_t* keys,
                                    uint32_t* vals, uint32_t* ranges, void* ws, const BinSortPlan& plan,
                                    int64_t stall_tile, cudaStream_t s) {
  SortWs w = carve(ws, plan);
  const int64_t TT = (int64_t)cam.TW * cam.TH;
  const int64_t cap = plan.capacity;
  cudaError_t e = cudaMemsetAsync(ranges, 0, (size_t)TT * 2 * sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;
  int launched = 0;
  if (n > 0) {
    emit_kernel<<<grid_for((cap + kEmitChunk - 1) / kEmitChunk * 32, 256), 256, 0, s>>>(
        w.dval[0], w.doff, w.dtiles, w.chunk_g, rec.rect, n, w.total + 1, cam.TW, w.total, cap,
                                                 w.status, w.tkey[0], w.tval[0]);
    ++launched;
  }
  if (cap > 0) {
    if (plan.passes == 0) {
      finalize_kernel<<<grid_for(cap, 256), 256, 0, s>>>(w.tkey[0], w.tval[0], w.total, cap, rec.xyzo, keys,
                                                         vals);
      ++launched;
    } else {
      // the last pass leaves tile ids (the ranges kernel writes the keys)
      const int k = sort_passes(w, w.tkey[0], w.tval[0], w.tkey[1], w.tval[1], cap, w.total, plan.passes,
                                w.tkey[plan.passes & 1], vals, n, nullptr, nullptr, stall_tile, s);
      if (k < 0) return cudaErrorLaunchFailure;
      launched += k;
    }
    const uint32_t* tiles_sorted = plan.passes == 0 ? w.tkey[0] : w.tkey[plan.passes & 1];
    ranges_kernel<<<(unsigned)std::min<int64_t>(grid_for(cap, 256), 148 * 16), 256, 0, s>>>(
        tiles_sorted, vals, rec.xyzo, n, keys, w.total, cap, w.status, TT, reinterpret_cast<uint2*>(ranges));
    ++launched;
  }
  count_launches(launched);
  return cudaGetLastError();
}

uint32_t checked_status_binsort() { return take_checked_status(); }

}  // namespace gs
