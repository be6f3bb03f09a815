// Tile compositing: forward (front to back) and backward (back to front).
//
// A 16x16 tile is four 8x8 pixel blocks, each the work of one warp, whose
// lanes hold two pixels (the same column, rows r and r + 4) run as packed
// fp32 pairs. The forward's warps, and the backward's when the forward's hit
// bytes are given, walk the tile's sorted list independently, with the
// entries' records gathered by cp.async into the warp's own shared-memory
// slots one chunk ahead; no CTA barrier stands between them. The backward
// without hit bytes stages batches of records for the tile's four warps in
// shared memory. The forward's warps leave the walk as soon as their pixels
// have stopped.
//
// The per-pair arithmetic is the fixed fp32 specification: the conic is
// scaled by -log2(e)/2 (and -log2(e) for the cross term) when it is staged,
// p2 = dx (a dx + b dy) + (c dy) dy, alpha = min(0.99, o * exp2(p2)). The
// backward recomputes alpha with the same operations, so its skip decisions
// match the forward's exactly, and recovers T by division.

#include "checked.cuh"
#include "gs_device.cuh"
#include "gs_internal.cuh"

namespace gs {
namespace {

constexpr int kTile = 16;
constexpr int kBlock = kTile * kTile;
// Backward CTA: 4 warps, two pixels per thread.
constexpr int kBlockB = kBlock / 2;
// List entries staged in shared memory per CTA-wide step of the backward
// without hit bytes: one per thread.
constexpr int kBatchB = kBlockB;

// 16-byte asynchronous global -> shared copy (L2 only), its commit and the
// wait for all of this thread's outstanding copies.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }
// cp.async groups: wait until at most one (the newest) is still in flight.
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }


// Conservative screen box of the pixel centres at which the fp32 pair
// arithmetic can give alpha >= 1/255 (a warp whose pixels all lie outside
// may skip the Gaussian: the per-pixel result is the same).
// With d = (px - x, py - y) the exact quadratic is p2(d) = -d^T M d,
// M = [[-a2, -b2/2], [-b2/2, -c2]] positive definite. Evaluated in fp32 as
// specified it is off by at most ~7 eps (|a2| dx^2 + |b2| |dx dy| + |c2| dy^2)
// <= sl |d|^2 with sl = 1e-6 K, K = max(|a2|, |c2|) + |b2|/2, so the
// computed value is <= -d^T (M - sl I) d. A blend needs o exp2(p2) >= 1/255
// up to ~2 ulp, i.e. p2 >= -log2(255 o) - 1e-3. Hence every blending pixel
// lies in the ellipse d^T (M - sl I) d <= log2(255 o) + 1e-3, whose bounding
// box is returned, widened by 2% plus 0.05 px to cover the rounding of this
// computation. For an ellipse that is not elongated (lambda_min >
// lambda_max / 100, where the quadratic form is accurate in fp32 to ~1e-4
// relative) the test is exact instead: the minimum of d^T (M - sl I) d over
// the warp's rectangle of pixel centres (widened by the same pad) against
// rho2 * 1.01. Returned: box = (px, py, hx, hy); q1 = (m00, m01, m11,
// threshold), threshold +inf when only the box applies; q2 = (m01 / m00,
// m01 / m11, pad, 0). An empty box (negative half-widths) if the Gaussian
// can never blend, an unbounded one if (M - sl I) is not safely positive
// definite.
// The region's square roots and quotients use the hardware approximations
// (sqrt.approx, div.approx: a few ulp, ~1e-6 relative at most) instead of
// correctly rounded ones: the box is widened by 2% and the threshold by 1%,
// four orders of magnitude more than those errors, and the minimum of the
// quadratic form moves only to second order with the edge point the ratios
// give, so the region stays conservative.
__device__ __forceinline__ float sqrt_approx(float x) {
  float r;
  asm("sqrt.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
struct BlendRegion {
  float4 box;
  float4 q1;
  float4 q2;
};

__device__ __forceinline__ BlendRegion blend_region(float px, float py, float a2, float b2, float c2, float o) {
  const float kInf = __int_as_float(0x7f800000);
  const float rho2 = __log2f(255.0f * o) + 1e-3f;
  const float4 none = make_float4(0.f, 0.f, 0.f, 0.f);
  if (!(rho2 > 0.0f)) return BlendRegion{make_float4(px, py, -kInf, -kInf), make_float4(1.f, 0.f, 1.f, kInf), none};
  const float K = fmaxf(fabsf(a2), fabsf(c2)) + 0.5f * fabsf(b2);
  const float sl = 1e-6f * K;
  const float m00 = -a2 - sl, m11 = -c2 - sl, m01 = -0.5f * b2;
  const float det = m00 * m11 - m01 * m01;
  if (!(m00 > 0.0f) || !(m11 > 0.0f) || !(det > 1e-3f * (m00 * m11)))
    return BlendRegion{make_float4(px, py, kInf, kInf), make_float4(1.f, 0.f, 1.f, kInf), none};
  const float pad = 0.05f + 1e-6f * (fabsf(px) + fabsf(py));
  const float idet = __fdividef(rho2, det);
  const float hx = sqrt_approx(idet * m11) * 1.02f + pad;
  const float hy = sqrt_approx(idet * m00) * 1.02f + pad;
  const float half_tr = 0.5f * (m00 + m11);
  const float disc = sqrt_approx(0.25f * (m00 - m11) * (m00 - m11) + m01 * m01);
  const float lmin = half_tr - disc;
  const float thr = lmin > 0.01f * (half_tr + disc) ? rho2 * 1.01f : kInf;
  return BlendRegion{make_float4(px, py, hx, hy), make_float4(m00, m01, m11, thr),
                     make_float4(__fdividef(m01, m00), __fdividef(m01, m11), pad, 0.f)};
}

// Can the Gaussian blend at a pixel centre of the warp block with centre
// (wcx, wcy) and half extents (hwx, hwy)? Box test, then (when enabled) the
// minimum of the quadratic form over the rectangle of offsets d = (px, py) -
// pixel centre: 0 if the rectangle holds the centre, else the least of the
// four edges' one-dimensional minima.
__device__ __forceinline__ bool region_hits(const float4 b, const float4 q1, const float4 q2, float wcx,
                                            float wcy, float hwx, float hwy) {
  const float ux = b.x - wcx, uy = b.y - wcy;
  if (!(fabsf(ux) - hwx <= b.z && fabsf(uy) - hwy <= b.w)) return false;
  if (!(q1.w < __int_as_float(0x7f800000))) return true;
  const float dx0 = ux - hwx - q2.z, dx1 = ux + hwx + q2.z;
  const float dy0 = uy - hwy - q2.z, dy1 = uy + hwy + q2.z;
  if (dx0 <= 0.0f && dx1 >= 0.0f && dy0 <= 0.0f && dy1 >= 0.0f) return true;
  const float m00 = q1.x, m01 = q1.y, m11 = q1.z;
  auto qf = [&](float dx, float dy) { return fmaf(m00 * dx, dx, fmaf(2.0f * m01 * dx, dy, m11 * dy * dy)); };
  const float xa = fminf(fmaxf(-q2.x * dy0, dx0), dx1), xb = fminf(fmaxf(-q2.x * dy1, dx0), dx1);
  const float ya = fminf(fmaxf(-q2.y * dx0, dy0), dy1), yb = fminf(fmaxf(-q2.y * dx1, dy0), dy1);
  const float best = fminf(fminf(qf(xa, dy0), qf(xb, dy1)), fminf(qf(dx0, ya), qf(dx1, yb)));
  return best <= q1.w;
}


// Tiles in descending order of log2 of their list length: a launch that takes
// its CTAs' tiles in this order starts the longest lists first, so few long
// CTAs are left running alone at the end. One CTA; counting sort over 33
// buckets, the order inside a bucket unspecified (it does not change results).
__global__ void __launch_bounds__(1024) tile_order_kernel(const uint2* ranges, int64_t TT, uint32_t* order) {
  __shared__ uint32_t cnt[33];
  if (threadIdx.x < 33) cnt[threadIdx.x] = 0;
  __syncthreads();
  for (int64_t t = threadIdx.x; t < TT; t += 1024) {
    const uint32_t len = ranges[t].y - ranges[t].x;
    atomicAdd(&cnt[len ? 32 - __clz(len) : 0], 1u);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t run = 0;
    for (int b = 32; b >= 0; --b) {
      const uint32_t c = cnt[b];
      cnt[b] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int64_t t = threadIdx.x; t < TT; t += 1024) {
    const uint32_t len = ranges[t].y - ranges[t].x;
    order[atomicAdd(&cnt[len ? 32 - __clz(len) : 0], 1u)] = (uint32_t)t;
  }
}

struct FwdArgs {
  const float4* xyzo;
  const float4* conic;
  const float4* rgb;
  const uint32_t* vals;
  const uint2* ranges;
  const uint32_t* order;  // tile of CTA b (null: tile b)
  int W, H, TW;
  float bg0, bg1, bg2;
  float* image;
  float* final_T;
  int32_t* n_contrib;
  int32_t* last;
  float* importance;           // kImp: [N] += sum over pixels of alpha * T
  const int32_t* active_idx;   // record -> Gaussian, or null (identity)
  uint8_t* hits;               // [entries] or null: bit w = the entry blended in warp w's block
};

// Zeroes the hit bytes of every tile's list entries ([range.x, range.y) of
// each tile, one CTA per tile) before a forward whose warps OR their bits in.
__global__ void __launch_bounds__(256) zero_hits_kernel(const uint2* ranges, uint8_t* hits) {
  const uint2 r = ranges[blockIdx.x];
  for (uint32_t k = r.x + threadIdx.x; k < r.y; k += 256) hits[k] = 0;
}

// Forward with independent warps and no CTA barrier: warp w of a tile (warp
// 4 slot + w of the grid) owns the 8x8 pixel block at ((w & 1) * 8, (w >> 1) * 8), lane l
// its pixels (l & 7, l >> 3) and (l & 7, (l >> 3) + 4), both run as packed
// fp32 pairs (each half rounded as the scalar operation, so every pixel's
// values are those of the specification). The warp walks its tile's list
// front to back in chunks of 32 entries (lane l: entry 32 c + l): the
// entries' records arrive by cp.async in the warp's own double-buffered
// slots, one chunk ahead, and their indices two chunks ahead. Each lane tests
// its entry's blend region against the warp's block; the warp then blends the
// entries that can reach it, in list order. A warp leaves as soon as its 64
// pixels have stopped, independently of the tile's other blocks.
// Hit bytes: bit f (pixel rows 0-3 of the block, the 8x4 block f of the
// eight-warp layout) and bit f + 2 (rows 4-7), f = (w & 1) | (w >> 1) << 2,
// are OR-ed into the entry's byte with one word atomic per 4 entries; the
// bytes are zeroed first (zero_hits_kernel).
// kFwdWarps independent warps per CTA (blocks of the same tile, sharing
// nothing): more resident warps than one-warp CTAs allow (32 per SM), within
// the register bound below.
// kImp also adds each Gaussian's importance weight (the sum over the view's
// pixels of its blend weights alpha * T): per blended entry the warp sums its
// 64 pixels' weights (the lane's pair, then a 5-level butterfly) into the
// entry's slot, and after the chunk each lane adds its entry's slot to the
// Gaussian's total with one atomic: one atomic per (Gaussian, 8x8 block).
constexpr int kFwdWarps = 2;
static_assert(4 % kFwdWarps == 0, "a tile's four blocks split evenly over the CTAs");
template <bool kImp>
__global__ void __launch_bounds__(32 * kFwdWarps, 18) raster_fwd_warp_kernel(FwdArgs a) {
  __shared__ float4 s_raw_all[kFwdWarps][2][3][32];  // per warp: xyzo, conic, rgb of two chunks of entries
  __shared__ float s_imp_all[kImp ? kFwdWarps : 1][32];  // per warp: the chunk's importance sums
  const int lane = threadIdx.x & 31;
  float4(*s_raw)[3][32] = s_raw_all[threadIdx.x >> 5];
  float* s_imp = s_imp_all[kImp ? threadIdx.x >> 5 : 0];
  const int64_t gw = (int64_t)blockIdx.x * kFwdWarps + (threadIdx.x >> 5);  // (tile slot, 8x8 block)
  const uint32_t slot4 = (uint32_t)(gw >> 2);
  const int warp = (int)(gw & 3);
  const uint32_t tile_u = a.order ? a.order[slot4] : slot4;
  if (tile_u >= gridDim.x * (uint32_t)kFwdWarps / 4u) return;  // not a tile: a schedule that is no permutation
  const int tile = (int)tile_u;
  const int tx0 = (tile % a.TW) * kTile, ty0 = (tile / a.TW) * kTile;
  const int u = tx0 + (warp & 1) * 8 + (lane & 7), v0 = ty0 + (warp >> 1) * 8 + (lane >> 3);
  const bool in0 = u < a.W && v0 < a.H, in1 = u < a.W && v0 + 4 < a.H;
  const float xc = __fadd_rn((float)u, 0.5f);
  const float2 yc = make_float2(__fadd_rn((float)v0, 0.5f), __fadd_rn((float)(v0 + 4), 0.5f));
  const float bcx = (float)(tx0 + (warp & 1) * 8) + 4.0f, bcy = (float)(ty0 + (warp >> 1) * 8) + 4.0f;
  const uint2 range = a.ranges[tile];
  const int n = check(range.y >= range.x, kCheckTileRange) ? (int)(range.y - range.x) : 0;
  const int f = (warp & 1) | ((warp >> 1) << 2);
  float2 T = make_float2(1.0f, 1.0f), C0 = make_float2(0.f, 0.f), C1 = C0, C2 = C0;
  int cnt0 = 0, cnt1 = 0, lst0 = 0, lst1 = 0;
  bool done0 = !in0, done1 = !in1;
  const uint32_t* lv = a.vals + range.x;
  auto meta = [&](int c) { return 32 * c + lane < n ? lv[32 * c + lane] : 0u; };
  auto fetch = [&](int buf, int c, uint32_t idx) {
    if (32 * c + lane < n) {
      cp_async16(&s_raw[buf][0][lane], a.xyzo + idx);
      cp_async16(&s_raw[buf][1][lane], a.conic + idx);
      cp_async16(&s_raw[buf][2][lane], a.rgb + idx);
    }
    cp_async_commit();
  };
  const int nchunks = (n + 31) >> 5;
  uint32_t i_cur = meta(0);
  fetch(0, 0, i_cur);
  uint32_t i_nxt = meta(1);
  for (int c = 0; c < nchunks; ++c) {
    if (__all_sync(0xffffffffu, done0 && done1)) break;
    const int buf = c & 1;
    fetch(buf ^ 1, c + 1, i_nxt);  // chunk c + 1 in flight (its buffer was released after chunk c - 1)
    const uint32_t i_this = i_cur;  // this lane's entry of chunk c
    i_cur = i_nxt;
    i_nxt = meta(c + 2);
    cp_async_wait_1();  // this lane's copies of chunk c have landed
    __syncwarp();       // and every lane's
    const int j = 32 * c + lane;
    bool rel = false;
    if (j < n) {
      const float4 g = s_raw[buf][0][lane];
      const float4 q = s_raw[buf][1][lane];
      const float a2 = __fmul_rn(q.x, kHalfNegLog2e), b2 = __fmul_rn(q.y, kNegLog2e),
                  c2 = __fmul_rn(q.z, kHalfNegLog2e);
      const BlendRegion r = blend_region(g.x, g.y, a2, b2, c2, g.w);
      rel = region_hits(r.box, r.q1, r.q2, bcx, bcy, 3.5f, 3.5f);
      s_raw[buf][1][lane] = make_float4(a2, b2, c2, 0.0f);  // the scaled conic, once per entry
    }
    unsigned msk = __ballot_sync(0xffffffffu, rel);
    __syncwarp();                 // the scaled conics are visible to every lane
    uint32_t bl0 = 0u, bl1 = 0u;  // bit k: entry 32 c + k blended at this lane's pixel 0 / 1
    uint32_t imp_msk = 0u;        // kImp: bit k: entry 32 c + k has a sum in its slot
    while (msk) {
      const int k = __ffs(msk) - 1;
      msk &= msk - 1;
      const float4 g = s_raw[buf][0][k];
      const float4 q = s_raw[buf][1][k];
      const float a2 = q.x, b2 = q.y, c2 = q.z;
      const float dx = __fsub_rn(g.x, xc);
      const float2 dy = sub2(splat2(g.y), yc);
      const float2 qv = fma2(splat2(b2), dy, splat2(__fmul_rn(a2, dx)));
      float2 p2 = mul2(splat2(dx), qv);
      p2 = fma2(mul2(splat2(c2), dy), dy, p2);
      const float2 e = exp2_raster2(p2);
      const float2 va = mul2(splat2(g.w), e);
      const float al0 = fminf(va.x, kAlphaMax), al1 = fminf(va.y, kAlphaMax);
      // a pixel that skips the entry or has stopped blends with alpha 0, which
      // leaves its colour, T and counts exactly as they were
      const bool b0 = !done0 && al0 >= kAlphaMin, b1 = !done1 && al1 >= kAlphaMin;
      if (!__any_sync(0xffffffffu, b0 || b1)) continue;
      const float4 col = s_raw[buf][2][k];
      const float2 ab = make_float2(b0 ? al0 : 0.0f, b1 ? al1 : 0.0f);
      const float2 wgt = mul2(ab, T);
      if (kImp) {
        float ws = wgt.x + wgt.y;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, o);
        if (lane == 0) s_imp[k] = ws;
        imp_msk |= 1u << k;
      }
      C0 = fma2(wgt, splat2(col.x), C0);
      C1 = fma2(wgt, splat2(col.y), C1);
      C2 = fma2(wgt, splat2(col.z), C2);
      T = mul2(T, sub2(splat2(1.0f), ab));
      done0 = done0 || T.x < kTMin;
      done1 = done1 || T.y < kTMin;
      bl0 |= (b0 ? 1u : 0u) << k;
      bl1 |= (b1 ? 1u : 0u) << k;
    }
    if (kImp) {
      __syncwarp();  // lane 0's sums are visible
      if ((imp_msk >> lane) & 1u) {
        const float w = s_imp[lane];
        if (w != 0.0f) atomicAdd(a.importance + (a.active_idx ? a.active_idx[i_this] : (int32_t)i_this), w);
      }
    }
    // contributor counts and last blends of the chunk, from its blend masks
    cnt0 += __popc(bl0);
    cnt1 += __popc(bl1);
    if (bl0) lst0 = 32 * c + (32 - __clz(bl0));
    if (bl1) lst1 = 32 * c + (32 - __clz(bl1));
    if (a.hits) {
      // lane k: the byte bits of entry 32 c + k; one atomic OR per 4 entries
      const uint32_t h0 = __reduce_or_sync(0xffffffffu, bl0), h1 = __reduce_or_sync(0xffffffffu, bl1);
      const uint32_t e = range.x + (uint32_t)j;  // global entry index
      uint32_t byte = (((h0 >> lane) & 1u) << f) | (((h1 >> lane) & 1u) << (f + 2));
      if (j >= n) byte = 0u;
      uint32_t word = byte << (8 * (e & 3u));
#pragma unroll
      for (int d = 1; d < 4; ++d) {  // the following lanes of the same 4-entry word
        const uint32_t o = __shfl_down_sync(0xffffffffu, word, d);
        const uint32_t oe = __shfl_down_sync(0xffffffffu, e, d);
        if (lane + d < 32 && (oe >> 2) == (e >> 2)) word |= o;
      }
      const bool leads = lane == 0 || (e & 3u) == 0u;
      if (leads && word != 0u && j < n)
        atomicOr(reinterpret_cast<unsigned int*>(a.hits + (e & ~3u)), word);
    }
    __syncwarp();  // every lane is done with buffer buf before it is refilled
  }
  cp_async_wait_all();  // no copy outlives the CTA
  const size_t P = (size_t)a.W * a.H;
  if (in0) {
    const size_t pix = (size_t)v0 * a.W + u;
    a.image[pix] = __fmaf_rn(T.x, a.bg0, C0.x);
    a.image[P + pix] = __fmaf_rn(T.x, a.bg1, C1.x);
    a.image[2 * P + pix] = __fmaf_rn(T.x, a.bg2, C2.x);
    a.final_T[pix] = T.x;
    a.n_contrib[pix] = cnt0;
    a.last[pix] = lst0;
  }
  if (in1) {
    const size_t pix = (size_t)(v0 + 4) * a.W + u;
    a.image[pix] = __fmaf_rn(T.y, a.bg0, C0.y);
    a.image[P + pix] = __fmaf_rn(T.y, a.bg1, C1.y);
    a.image[2 * P + pix] = __fmaf_rn(T.y, a.bg2, C2.y);
    a.final_T[pix] = T.y;
    a.n_contrib[pix] = cnt1;
    a.last[pix] = lst1;
  }
}

struct BwdArgs {
  const float4* xyzo;
  const float4* conic;
  const float4* rgb;
  const uint32_t* vals;
  const uint2* ranges;
  const uint32_t* order;  // tile of CTA b (null: tile b)
  int W, H, TW;
  float bg0, bg1, bg2;
  const float* final_T;
  const int32_t* last;
  const float* dL_dimage;
  float4* grad2d;  // [n][3]
  const uint8_t* hits;  // [entries] from the forward, or null
  int64_t n_records;    // records (bound of the list values)
};

// Where the multi-value butterfly below leaves its results: lane `lane` ends
// up holding the warp total of value `idx`, and it is the lane that reports
// it if `owner` (one lane per value 0..8).
struct Reduce9Slot {
  int idx;
  bool owner;
};
__device__ __forceinline__ Reduce9Slot reduce9_slot(int lane) {
  // Split tree over the value index range: 9 -> (5 | 4), 5 -> (3 | 2), 3 -> (2 | 1),
  // 2 -> (1 | 1); lanes with the offset bit set take the upper part.
  int b = 0, hi = 9;
  const int n1[4] = {5, 3, 2, 1};
  const int off[4] = {16, 8, 4, 2};
#pragma unroll
  for (int l = 0; l < 4; ++l) {
    if (lane & off[l]) b += n1[l];
    else hi = min(hi, b + n1[l]);
  }
  return Reduce9Slot{b, b < hi && (lane & 1) == 0};
}

// Sum v[0..8] over the warp with 12 shuffles (instead of 45): at each level a
// lane keeps one half of its values and trades the other half with its
// partner. Returns the total of value reduce9_slot(lane).idx.
__device__ __forceinline__ float warp_reduce9(const float v[9], int lane) {
  const bool u1 = lane & 16, u2 = lane & 8, u3 = lane & 4, u4 = lane & 2;
  float w1[5];
#pragma unroll
  for (int j = 0; j < 5; ++j) {
    const float lo = v[j], up = j + 5 < 9 ? v[j + 5] : 0.0f;
    const float r = __shfl_xor_sync(0xffffffffu, u1 ? lo : up, 16);
    w1[j] = (u1 ? up : lo) + r;
  }
  float w2[3];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const float lo = w1[j], up = j + 3 < 5 ? w1[j + 3] : 0.0f;
    const float r = __shfl_xor_sync(0xffffffffu, u2 ? lo : up, 8);
    w2[j] = (u2 ? up : lo) + r;
  }
  float w3[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float lo = w2[j], up = j + 2 < 3 ? w2[j + 2] : 0.0f;
    const float r = __shfl_xor_sync(0xffffffffu, u3 ? lo : up, 4);
    w3[j] = (u3 ? up : lo) + r;
  }
  const float r4 = __shfl_xor_sync(0xffffffffu, u4 ? w3[0] : w3[1], 2);
  const float w4 = (u4 ? w3[1] : w3[0]) + r4;
  return w4 + __shfl_xor_sync(0xffffffffu, w4, 1);
}

// State of a lane's two pixels in the backward walk: the same column, rows
// r and r + 4, so dx is shared and everything else is a pair (packed fp32).
struct BwdPair {
  float xc;          // pixel centre column
  float2 yc;         // pixel centre rows
  float2 T;          // transmittance in front of the current entry
  float2 R0, R1, R2; // colour accumulated behind it (background included)
  float2 g0, g1, g2; // dL/dimage
  int last0, last1;  // 1 + list offset of the last blend (0: none)
};

__device__ __forceinline__ BwdPair load_bwd_pair(const BwdArgs& a, int u, int v, size_t P) {
  BwdPair q;
  q.xc = __fadd_rn((float)u, 0.5f);
  q.yc = make_float2(__fadd_rn((float)v, 0.5f), __fadd_rn((float)(v + 4), 0.5f));
  q.R0 = splat2(a.bg0);
  q.R1 = splat2(a.bg1);
  q.R2 = splat2(a.bg2);
  float T[2] = {1.0f, 1.0f}, g[2][3] = {{0.f, 0.f, 0.f}, {0.f, 0.f, 0.f}};
  int last[2] = {0, 0};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int vv = v + 4 * h;
    if (u < a.W && vv < a.H) {
      const size_t pix = (size_t)vv * a.W + u;
      T[h] = a.final_T[pix];
      last[h] = a.last[pix];
      g[h][0] = a.dL_dimage[pix];
      g[h][1] = a.dL_dimage[P + pix];
      g[h][2] = a.dL_dimage[2 * P + pix];
    }
  }
  q.T = make_float2(T[0], T[1]);
  q.g0 = make_float2(g[0][0], g[1][0]);
  q.g1 = make_float2(g[0][1], g[1][1]);
  q.g2 = make_float2(g[0][2], g[1][2]);
  q.last0 = last[0];
  q.last1 = last[1];
  return q;
}

// Backward CTA: 4 warps per tile, warp w owns the 8x8 block at
// ((w & 1) * 8, (w >> 1) * 8) and lane l its pixels (l & 7, l >> 3) and
// (l & 7, (l >> 3) + 4). One warp step handles one entry for 64 pixels, so
// the warp sum of the gradient terms is paid once per 64 pixels.
__global__ void __launch_bounds__(kBlockB, 8) raster_bwd_kernel(BwdArgs a) {
  __shared__ float4 s_raw[3][kBatchB];  // xyzo, conic, rgb of the next batch, in flight
  __shared__ float4 s_geo[kBatchB];     // px, py, a2, b2
  __shared__ float4 s_co[kBatchB];      // c2, opacity, A, B
  __shared__ float4 s_rgb[kBatchB];     // r, g, b, C
  __shared__ uint8_t s_hit[kBatchB];    // bit w: the entry can blend in warp w's block
  __shared__ float s_acc[kBatchB][9];   // per-batch gradient sums of the CTA ([slot][value]: conflict-free)
  __shared__ int s_maxlast;
  const uint32_t tile_u = a.order ? a.order[blockIdx.x] : blockIdx.x;
  if (tile_u >= gridDim.x) return;  // not a tile: a schedule that is no permutation
  const int tile = (int)tile_u;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tx0 = (tile % a.TW) * kTile, ty0 = (tile / a.TW) * kTile;
  const int u = tx0 + (warp & 1) * 8 + (lane & 7), v = ty0 + (warp >> 1) * 8 + (lane >> 3);
  const uint2 range = a.ranges[tile];
  const size_t P = (size_t)a.W * a.H;
  BwdPair px = load_bwd_pair(a, u, v, P);
  const int warp_last = __reduce_max_sync(0xffffffffu, max(px.last0, px.last1));
  const Reduce9Slot slot = reduce9_slot(lane);
  if (tid == 0) s_maxlast = 0;
  __syncthreads();
  if (lane == 0 && warp_last > 0) atomicMax(&s_maxlast, warp_last);
  __syncthreads();
  const int n = s_maxlast;  // list offsets [0, n) can hold a blend
  // Slot k of the batch that starts at `done` holds list offset
  // n - 1 - done - k (back to front); thread tid owns slot tid. The records
  // of the next batch are copied into s_raw while this one is processed and
  // the indices of the batch after it are loaded into a register.
  const uint32_t* lv = a.vals + range.x;
  auto index_of = [&](int d) {
    const uint32_t i = n - 1 - d - tid >= 0 ? lv[n - 1 - d - tid] : 0u;
    return check(i < (uint64_t)a.n_records, kCheckRecordIndex) ? i : 0u;
  };
  auto fetch = [&](int d, uint32_t i) {
    if (n - 1 - d - tid >= 0) {
      cp_async16(&s_raw[0][tid], a.xyzo + i);
      cp_async16(&s_raw[1][tid], a.conic + i);
      cp_async16(&s_raw[2][tid], a.rgb + i);
    }
    cp_async_commit();
  };
  uint32_t icur = index_of(0);
  fetch(0, icur);
  uint32_t inext = index_of(kBatchB);
  for (int done = 0; done < n; done += kBatchB) {
    cp_async_wait_all();
    const bool have = n - 1 - done - tid >= 0;
    if (have) {
      const int e = tid;
      const float4 g = s_raw[0][e];
      const float4 q = s_raw[1][e];
      const float4 c = s_raw[2][e];
      const float a2 = __fmul_rn(q.x, kHalfNegLog2e), b2 = __fmul_rn(q.y, kNegLog2e),
                  c2 = __fmul_rn(q.z, kHalfNegLog2e);
      s_geo[e] = make_float4(g.x, g.y, a2, b2);
      s_co[e] = make_float4(c2, g.w, q.x, q.y);
      s_rgb[e] = make_float4(c.x, c.y, c.z, q.z);
      const BlendRegion r = blend_region(g.x, g.y, a2, b2, c2, g.w);
      uint32_t hit = 0;
#pragma unroll
      for (int w = 0; w < kBlockB / 32; ++w) {
        const float bcx = (float)(tx0 + (w & 1) * 8) + 4.0f, bcy = (float)(ty0 + (w >> 1) * 8) + 4.0f;
        if (region_hits(r.box, r.q1, r.q2, bcx, bcy, 3.5f, 3.5f)) hit |= 1u << w;
      }
      s_hit[e] = (uint8_t)hit;
    }
#pragma unroll
    for (int j = 0; j < 9; ++j) s_acc[tid][j] = 0.0f;
    const uint32_t ithis = icur;
    icur = inext;
    fetch(done + kBatchB, icur);
    inext = index_of(done + 2 * kBatchB);
    __syncthreads();
    const int m = min(kBatchB, n - done);
    for (int c0 = 0; c0 < m; c0 += 32) {
      const int j = c0 + lane;
      const bool rel = j < m && (n - 1 - done - j) < warp_last && ((s_hit[j] >> warp) & 1u);
      unsigned msk = __ballot_sync(0xffffffffu, rel);
      while (msk) {
        const int k = c0 + __ffs(msk) - 1;
        msk &= msk - 1;
        const int offk = n - 1 - done - k;
        const float4 g = s_geo[k];   // px, py, a2, b2
        const float4 co = s_co[k];   // c2, opacity, A, B
        // alpha of both pixels, recomputed exactly as the forward computed
        // it (the same operations; dx is common to the pair)
        const float dx = __fsub_rn(g.x, px.xc);
        const float2 dy = sub2(splat2(g.y), px.yc);
        const float2 qv = fma2(splat2(g.w), dy, splat2(__fmul_rn(g.z, dx)));
        float2 p2 = mul2(splat2(dx), qv);
        p2 = fma2(mul2(splat2(co.x), dy), dy, p2);
        const float2 e = exp2_raster2(p2);
        const float2 vv = mul2(splat2(co.y), e);
        const float al0 = fminf(vv.x, kAlphaMax), al1 = fminf(vv.y, kAlphaMax);
        // a pair that was not a blend of the forward (past the pixel's last
        // blend, or alpha < 1/255) runs with alpha 0: T and R stay, no terms
        const bool b0 = offk < px.last0 && al0 >= kAlphaMin, b1 = offk < px.last1 && al1 >= kAlphaMin;
        if (!__any_sync(0xffffffffu, b0 || b1)) continue;
        const float2 ab = make_float2(b0 ? al0 : 0.0f, b1 ? al1 : 0.0f);
        const float2 oma = sub2(splat2(1.0f), ab);
        // transmittance in front of this entry (gradient values only)
        px.T = make_float2(b0 ? __fdividef(px.T.x, oma.x) : px.T.x, b1 ? __fdividef(px.T.y, oma.y) : px.T.y);
        const float2 wgt = mul2(ab, px.T);
        const float4 c = s_rgb[k];   // r, g, b, C
        float2 sg = mul2(px.g0, sub2(splat2(c.x), px.R0));
        sg = fma2(px.g1, sub2(splat2(c.y), px.R1), sg);
        sg = fma2(px.g2, sub2(splat2(c.z), px.R2), sg);
        const float2 Gk = mul2(px.T, sg);
        // no gradient through a clamped alpha
        const float2 Gm = make_float2((b0 && vv.x < kAlphaMax) ? Gk.x : 0.0f, (b1 && vv.y < kAlphaMax) ? Gk.y : 0.0f);
        const float2 dp = mul2(Gm, ab);
        const float2 dpdy = mul2(dp, dy);
        const float2 dpdy2 = mul2(dpdy, dy);
        const float2 ge = mul2(Gm, e);
        const float2 w0 = mul2(px.g0, wgt), w1 = mul2(px.g1, wgt), w2 = mul2(px.g2, wgt);
        // the nine terms summed over the pair (mean2D x, y, opacity, conic
        // A, B, C, colour r, g, b); dp/dpx = -(A dx + B dy), dp/dA = -dx^2/2,
        // dp/dB = -dx dy, dp/dC = -dy^2/2
        const float sdp = dp.x + dp.y, sdpdy = dpdy.x + dpdy.y;
        const float A = co.z, B = co.w, Cc = c.w, dxs = dx * sdp;
        float gv[9];
        gv[0] = -fmaf(A, dxs, B * sdpdy);
        gv[1] = -fmaf(B, dxs, Cc * sdpdy);
        gv[2] = ge.x + ge.y;
        gv[3] = -0.5f * dx * dxs;
        gv[4] = -dx * sdpdy;
        gv[5] = -0.5f * (dpdy2.x + dpdy2.y);
        gv[6] = w0.x + w0.y;
        gv[7] = w1.x + w1.y;
        gv[8] = w2.x + w2.y;
        px.R0 = fma2(splat2(c.x), ab, mul2(oma, px.R0));
        px.R1 = fma2(splat2(c.y), ab, mul2(oma, px.R1));
        px.R2 = fma2(splat2(c.z), ab, mul2(oma, px.R2));
        const float tot = warp_reduce9(gv, lane);
        if (slot.owner) atomicAdd(&s_acc[k][slot.idx], tot);
      }
    }
    __syncthreads();
    // flush this thread's slot (only this thread touches it until the next
    // batch's barrier)
    if (have) {
      float r[9];
      bool any = false;
#pragma unroll
      for (int j = 0; j < 9; ++j) {
        r[j] = s_acc[tid][j];
        any |= r[j] != 0.0f;
      }
      if (any) {
        float4* dst = a.grad2d + 3 * (size_t)ithis;
        atomicAdd(dst, make_float4(r[0], r[1], r[2], 0.f));
        atomicAdd(dst + 1, make_float4(r[3], r[4], r[5], 0.f));
        atomicAdd(dst + 2, make_float4(r[6], r[7], r[8], 0.f));
      }
    }
  }
  cp_async_wait_all();  // no copy outlives the CTA
}

// Warps (8x8 blocks) per CTA of the hit-byte backward. Its warps share
// nothing, so a CTA of one warp frees its slot as soon as its block is done
// instead of waiting for the tile's other three blocks.
constexpr int kHitsWarps = 1;
static_assert(4 % kHitsWarps == 0, "a tile's four blocks split evenly over the CTAs");


// Backward with the forward's hit bytes: warp w (the 8x8 block of forward
// warps f and f + 2, f = (w & 1) | (w >> 1) << 2) walks its own list
// entries back to front from the last blend of its pixels, 32 per chunk
// (lane l: offset warp_last - 1 - 32 c - l). Only the entries whose byte has
// bit f or f + 2 set are fetched: by cp.async into the warp's own
// double-buffered slots, one chunk ahead. The warps of a CTA share no data
// and never wait for each other. Per pixel the operations, and the entries
// that blend, are those of raster_bwd_kernel, so every pixel's terms are
// the same values; the warp sums go to the global gradient rows directly.
__global__ void __launch_bounds__(32 * kHitsWarps) raster_bwd_hits_kernel(BwdArgs a) {
  __shared__ float4 s_raw[kHitsWarps][2][3][32];  // xyzo, conic, rgb of the hit entries of two chunks
  __shared__ float s_acc[kHitsWarps][32][9];      // the chunk's warp sums ([slot][value])
  const int wc = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gw = (int64_t)blockIdx.x * kHitsWarps + wc;  // (tile slot, 8x8 block)
  const uint32_t slot4 = (uint32_t)(gw >> 2);
  const uint32_t tile_u = a.order ? a.order[slot4] : slot4;
  if (tile_u >= gridDim.x * (uint32_t)kHitsWarps / 4u) return;  // not a tile: a schedule that is no permutation
  const int tile = (int)tile_u;
  const int warp = (int)(gw & 3);
  const int tx0 = (tile % a.TW) * kTile, ty0 = (tile / a.TW) * kTile;
  const int u = tx0 + (warp & 1) * 8 + (lane & 7), v = ty0 + (warp >> 1) * 8 + (lane >> 3);
  const uint2 range = a.ranges[tile];
  const size_t P = (size_t)a.W * a.H;
  BwdPair px = load_bwd_pair(a, u, v, P);
  const int warp_last = __reduce_max_sync(0xffffffffu, max(px.last0, px.last1));
  if (warp_last == 0) return;  // no pixel of the block blended anything
  const Reduce9Slot slot = reduce9_slot(lane);
  const int f = (warp & 1) | ((warp >> 1) << 2);
  const uint32_t fbits = (1u << f) | (1u << (f + 2));
  const uint32_t* lv = a.vals + range.x;
  const uint8_t* hb = a.hits + range.x;
  float4(*raw)[3][32] = s_raw[wc];
  float(*acc)[9] = s_acc[wc];
  // lane's entry of chunk c: its record index and whether the block can blend it
  auto meta = [&](int c, uint32_t& idx, bool& hit) {
    const int off = warp_last - 1 - 32 * c - lane;
    const bool in = off >= 0;
    const uint32_t b = in ? (uint32_t)hb[off] : 0u;
    idx = in ? lv[off] : 0u;
    hit = (b & fbits) != 0u && check(idx < (uint64_t)a.n_records, kCheckRecordIndex);
  };
  auto fetch = [&](int buf, uint32_t idx, bool hit) {
    if (hit) {
      cp_async16(&raw[buf][0][lane], a.xyzo + idx);
      cp_async16(&raw[buf][1][lane], a.conic + idx);
      cp_async16(&raw[buf][2][lane], a.rgb + idx);
    }
    cp_async_commit();
  };
  const int nchunks = (warp_last + 31) >> 5;
  uint32_t i_cur, i_nxt;
  bool h_cur, h_nxt;
  meta(0, i_cur, h_cur);
  fetch(0, i_cur, h_cur);
  meta(1, i_nxt, h_nxt);
  for (int c = 0; c < nchunks; ++c) {
    const int buf = c & 1;
    fetch(buf ^ 1, i_nxt, h_nxt);  // chunk c + 1 in flight (its buffer was freed after chunk c - 1)
    const uint32_t i_this = i_cur;
    const bool h_this = h_cur;
    i_cur = i_nxt;
    h_cur = h_nxt;
    meta(c + 2, i_nxt, h_nxt);
    cp_async_wait_1();  // this lane's copies of chunk c have landed
    __syncwarp();       // and every lane's
    unsigned msk = __ballot_sync(0xffffffffu, h_this);
    unsigned summed = 0u;
    while (msk) {
      const int k = __ffs(msk) - 1;
      msk &= msk - 1;
      const int offk = warp_last - 1 - 32 * c - k;
      const float4 G = raw[buf][0][k];  // px, py, depth, opacity
      const float4 Q = raw[buf][1][k];  // A, B, C
      const float a2 = __fmul_rn(Q.x, kHalfNegLog2e), b2 = __fmul_rn(Q.y, kNegLog2e),
                  c2 = __fmul_rn(Q.z, kHalfNegLog2e);
      const float dx = __fsub_rn(G.x, px.xc);
      const float2 dy = sub2(splat2(G.y), px.yc);
      const float2 qv = fma2(splat2(b2), dy, splat2(__fmul_rn(a2, dx)));
      float2 p2 = mul2(splat2(dx), qv);
      p2 = fma2(mul2(splat2(c2), dy), dy, p2);
      const float2 e = exp2_raster2(p2);
      const float2 vv = mul2(splat2(G.w), e);
      const float al0 = fminf(vv.x, kAlphaMax), al1 = fminf(vv.y, kAlphaMax);
      const bool b0 = offk < px.last0 && al0 >= kAlphaMin, b1 = offk < px.last1 && al1 >= kAlphaMin;
      if (!__any_sync(0xffffffffu, b0 || b1)) continue;
      const float2 ab = make_float2(b0 ? al0 : 0.0f, b1 ? al1 : 0.0f);
      const float2 oma = sub2(splat2(1.0f), ab);
      px.T = make_float2(b0 ? __fdividef(px.T.x, oma.x) : px.T.x, b1 ? __fdividef(px.T.y, oma.y) : px.T.y);
      const float2 wgt = mul2(ab, px.T);
      const float4 cc = raw[buf][2][k];  // r, g, b
      float2 sg = mul2(px.g0, sub2(splat2(cc.x), px.R0));
      sg = fma2(px.g1, sub2(splat2(cc.y), px.R1), sg);
      sg = fma2(px.g2, sub2(splat2(cc.z), px.R2), sg);
      const float2 Gk = mul2(px.T, sg);
      const float2 Gm = make_float2((b0 && vv.x < kAlphaMax) ? Gk.x : 0.0f, (b1 && vv.y < kAlphaMax) ? Gk.y : 0.0f);
      const float2 dp = mul2(Gm, ab);
      const float2 dpdy = mul2(dp, dy);
      const float2 dpdy2 = mul2(dpdy, dy);
      const float2 ge = mul2(Gm, e);
      const float2 w0 = mul2(px.g0, wgt), w1 = mul2(px.g1, wgt), w2 = mul2(px.g2, wgt);
      const float sdp = dp.x + dp.y, sdpdy = dpdy.x + dpdy.y;
      const float A = Q.x, B = Q.y, Cc = Q.z, dxs = dx * sdp;
      float gv[9];
      gv[0] = -fmaf(A, dxs, B * sdpdy);
      gv[1] = -fmaf(B, dxs, Cc * sdpdy);
      gv[2] = ge.x + ge.y;
      gv[3] = -0.5f * dx * dxs;
      gv[4] = -dx * sdpdy;
      gv[5] = -0.5f * (dpdy2.x + dpdy2.y);
      gv[6] = w0.x + w0.y;
      gv[7] = w1.x + w1.y;
      gv[8] = w2.x + w2.y;
      px.R0 = fma2(splat2(cc.x), ab, mul2(oma, px.R0));
      px.R1 = fma2(splat2(cc.y), ab, mul2(oma, px.R1));
      px.R2 = fma2(splat2(cc.z), ab, mul2(oma, px.R2));
      const float tot = warp_reduce9(gv, lane);
      if (slot.owner) acc[k][slot.idx] = tot;
      summed |= 1u << k;
    }
    __syncwarp();
    if ((summed >> lane) & 1u) {
      float r[9];
      bool any = false;
#pragma unroll
      for (int j = 0; j < 9; ++j) {
        r[j] = acc[lane][j];
        any |= r[j] != 0.0f;
      }
      if (any) {
        float4* dst = a.grad2d + 3 * (size_t)i_this;
        atomicAdd(dst, make_float4(r[0], r[1], r[2], 0.f));
        atomicAdd(dst + 1, make_float4(r[3], r[4], r[5], 0.f));
        atomicAdd(dst + 2, make_float4(r[6], r[7], r[8], 0.f));
      }
    }
    __syncwarp();  // the chunk's slots and sums are free again
  }
  cp_async_wait_all();  // no copy outlives the warp
}

}  // namespace

cudaError_t launch_raster_fwd(const Records& rec, const uint32_t* vals, const uint32_t* ranges,
                              const DevCam& cam, const float bg[3], float* image, float* final_T,
                              int32_t* n_contrib, int32_t* last, float* importance, const int32_t* active_idx,
                              const uint32_t* order, uint8_t* hits, cudaStream_t s) {
  FwdArgs a;
  a.xyzo = rec.xyzo; a.conic = rec.conic; a.rgb = rec.rgb;
  a.vals = vals; a.ranges = reinterpret_cast<const uint2*>(ranges); a.order = order;
  a.W = cam.width; a.H = cam.height; a.TW = cam.TW;
  a.bg0 = bg[0]; a.bg1 = bg[1]; a.bg2 = bg[2];
  a.image = image; a.final_T = final_T; a.n_contrib = n_contrib; a.last = last;
  a.importance = importance; a.active_idx = active_idx; a.hits = hits;
  const int TT = cam.TW * cam.TH;
  int launched = 1;
  if (hits) {
    zero_hits_kernel<<<TT, 256, 0, s>>>(a.ranges, hits);
    ++launched;
  }
  if (importance)
    raster_fwd_warp_kernel<true><<<TT * 4 / kFwdWarps, 32 * kFwdWarps, 0, s>>>(a);
  else
    raster_fwd_warp_kernel<false><<<TT * 4 / kFwdWarps, 32 * kFwdWarps, 0, s>>>(a);
  count_launches(launched);
  return cudaGetLastError();
}

cudaError_t launch_raster_bwd(const Records& rec, const uint32_t* vals, const uint32_t* ranges,
                              const DevCam& cam, const float bg[3], const float* final_T,
                              const int32_t* last, const float* dL_dimage, float4* grad2d,
                              int64_t n_records, const uint32_t* order, const uint8_t* hits, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(grad2d, 0, (size_t)n_records * 3 * sizeof(float4), s);
  if (e != cudaSuccess) return e;
  BwdArgs a;
  a.xyzo = rec.xyzo; a.conic = rec.conic; a.rgb = rec.rgb;
  a.vals = vals; a.ranges = reinterpret_cast<const uint2*>(ranges); a.order = order;
  a.W = cam.width; a.H = cam.height; a.TW = cam.TW;
  a.bg0 = bg[0]; a.bg1 = bg[1]; a.bg2 = bg[2];
  a.final_T = final_T; a.last = last; a.dL_dimage = dL_dimage; a.grad2d = grad2d; a.hits = hits;
  a.n_records = n_records;
  if (hits)
    raster_bwd_hits_kernel<<<cam.TW * cam.TH * 4 / kHitsWarps, 32 * kHitsWarps, 0, s>>>(a);
  else
    raster_bwd_kernel<<<cam.TW * cam.TH, kBlockB, 0, s>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_tile_order(const uint32_t* ranges, int64_t TT, uint32_t* order, cudaStream_t s) {
  if (TT == 0) return cudaSuccess;
  tile_order_kernel<<<1, 1024, 0, s>>>(reinterpret_cast<const uint2*>(ranges), TT, order);
  count_launches(1);
  return cudaGetLastError();
}

uint32_t checked_status_raster() { return take_checked_status(); }

}  // namespace gs
