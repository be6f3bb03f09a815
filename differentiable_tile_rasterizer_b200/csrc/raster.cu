// Tile compositing: forward (front to back) and backward (back to front).
//
// One CTA per 16x16 tile, one thread per pixel; each warp owns an 8x4 pixel
// block so that its lanes sit close together in the image. The tile's sorted
// list is walked in batches of 256 records that the CTA stages cooperatively
// in shared memory (one gathered 16-byte load per record field per batch),
// after which every thread reads them as shared-memory broadcasts. The CTA
// leaves the walk as soon as all its pixels have stopped.
//
// The per-pair arithmetic is the fixed fp32 specification: the conic is
// scaled by -log2(e)/2 (and -log2(e) for the cross term) when it is staged,
// p2 = dx (a dx + b dy) + (c dy) dy, alpha = min(0.99, o * exp2(p2)). The
// backward recomputes alpha with the same operations, so its skip decisions
// match the forward's exactly, and recovers T by division.

#include "gs_device.cuh"
#include "gs_internal.cuh"

namespace gs {
namespace {

constexpr int kTile = 16;
constexpr int kBlock = kTile * kTile;

// Pixel of thread `tid` in the tile: warp w covers the 8x4 block at
// ((w & 1) * 8, (w >> 1) * 4).
__device__ __forceinline__ void tile_pixel(int tid, int& du, int& dv) {
  const int w = tid >> 5, l = tid & 31;
  du = (w & 1) * 8 + (l & 7);
  dv = (w >> 1) * 4 + (l >> 3);
}

struct FwdArgs {
  const float4* xyzo;
  const float4* conic;
  const float4* rgb;
  const uint32_t* vals;
  const uint2* ranges;
  int W, H, TW;
  float bg0, bg1, bg2;
  float* image;
  float* final_T;
  int32_t* n_contrib;
  int32_t* last;
};

__global__ void __launch_bounds__(kBlock) raster_fwd_kernel(FwdArgs a) {
  __shared__ float4 s_geo[kBlock];  // px, py, a2, b2
  __shared__ float2 s_co[kBlock];   // c2, opacity
  __shared__ float4 s_rgb[kBlock];
  const int tile = blockIdx.x;
  const int tid = threadIdx.x;
  int du, dv;
  tile_pixel(tid, du, dv);
  const int u = (tile % a.TW) * kTile + du, v = (tile / a.TW) * kTile + dv;
  const bool inside = u < a.W && v < a.H;
  const float xc = __fadd_rn((float)u, 0.5f), yc = __fadd_rn((float)v, 0.5f);
  const uint2 range = a.ranges[tile];
  const int n = (int)(range.y - range.x);
  float T = 1.0f, C0 = 0.0f, C1 = 0.0f, C2 = 0.0f;
  int cnt = 0, lst = 0;
  bool done = !inside;
  for (int base = 0; base < n; base += kBlock) {
    if (__syncthreads_count(done) == kBlock) break;
    if (base + tid < n) {
      const uint32_t i = a.vals[range.x + base + tid];
      const float4 g = a.xyzo[i];
      const float4 q = a.conic[i];
      s_geo[tid] = make_float4(g.x, g.y, __fmul_rn(q.x, kHalfNegLog2e), __fmul_rn(q.y, kNegLog2e));
      s_co[tid] = make_float2(__fmul_rn(q.z, kHalfNegLog2e), g.w);
      s_rgb[tid] = a.rgb[i];
    }
    __syncthreads();
    if (!done) {
      const int m = min(kBlock, n - base);
      for (int k = 0; k < m; ++k) {
        const float4 g = s_geo[k];
        const float2 co = s_co[k];
        const float dx = __fsub_rn(g.x, xc), dy = __fsub_rn(g.y, yc);
        float qv = __fmul_rn(g.z, dx);
        qv = __fmaf_rn(g.w, dy, qv);
        float p2 = __fmul_rn(dx, qv);
        const float wv = __fmul_rn(co.x, dy);
        p2 = __fmaf_rn(wv, dy, p2);
        const float e = exp2_raster(p2);
        const float alpha = fminf(__fmul_rn(co.y, e), kAlphaMax);
        if (alpha < kAlphaMin) continue;
        const float4 c = s_rgb[k];
        const float wgt = __fmul_rn(alpha, T);
        C0 = __fmaf_rn(wgt, c.x, C0);
        C1 = __fmaf_rn(wgt, c.y, C1);
        C2 = __fmaf_rn(wgt, c.z, C2);
        T = __fmul_rn(T, __fsub_rn(1.0f, alpha));
        ++cnt;
        lst = base + k + 1;
        if (T < kTMin) {
          done = true;
          break;
        }
      }
    }
  }
  if (inside) {
    const size_t P = (size_t)a.W * a.H, pix = (size_t)v * a.W + u;
    a.image[pix] = __fmaf_rn(T, a.bg0, C0);
    a.image[P + pix] = __fmaf_rn(T, a.bg1, C1);
    a.image[2 * P + pix] = __fmaf_rn(T, a.bg2, C2);
    a.final_T[pix] = T;
    a.n_contrib[pix] = cnt;
    a.last[pix] = lst;
  }
}

struct BwdArgs {
  const float4* xyzo;
  const float4* conic;
  const float4* rgb;
  const uint32_t* vals;
  const uint2* ranges;
  int W, H, TW;
  float bg0, bg1, bg2;
  const float* final_T;
  const int32_t* last;
  const float* dL_dimage;
  float4* grad2d;  // [n][3]
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(kBlock) raster_bwd_kernel(BwdArgs a) {
  __shared__ float4 s_geo[kBlock];  // px, py, a2, b2
  __shared__ float4 s_co[kBlock];   // c2, opacity, A, B
  __shared__ float4 s_rgb[kBlock];  // r, g, b, C
  __shared__ uint32_t s_idx[kBlock];
  __shared__ int s_maxlast;
  const int tile = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  int du, dv;
  tile_pixel(tid, du, dv);
  const int u = (tile % a.TW) * kTile + du, v = (tile / a.TW) * kTile + dv;
  const bool inside = u < a.W && v < a.H;
  const float xc = __fadd_rn((float)u, 0.5f), yc = __fadd_rn((float)v, 0.5f);
  const uint2 range = a.ranges[tile];
  const size_t P = (size_t)a.W * a.H, pix = (size_t)v * a.W + u;
  float T = 1.0f, g0 = 0.f, g1 = 0.f, g2 = 0.f;
  int my_last = 0;
  if (inside) {
    T = a.final_T[pix];
    my_last = a.last[pix];
    g0 = a.dL_dimage[pix];
    g1 = a.dL_dimage[P + pix];
    g2 = a.dL_dimage[2 * P + pix];
  }
  float R0 = a.bg0, R1 = a.bg1, R2 = a.bg2;
  if (tid == 0) s_maxlast = 0;
  __syncthreads();
  if (my_last > 0) atomicMax(&s_maxlast, my_last);
  __syncthreads();
  const int n = s_maxlast;  // list offsets [0, n) can hold a blend
  for (int done = 0; done < n; done += kBlock) {
    // this batch covers list offsets n-1-done down to max(0, n-done-kBlock)
    __syncthreads();
    const int off = n - 1 - done - tid;
    if (off >= 0) {
      const uint32_t i = a.vals[range.x + off];
      const float4 g = a.xyzo[i];
      const float4 q = a.conic[i];
      const float4 c = a.rgb[i];
      s_geo[tid] = make_float4(g.x, g.y, __fmul_rn(q.x, kHalfNegLog2e), __fmul_rn(q.y, kNegLog2e));
      s_co[tid] = make_float4(__fmul_rn(q.z, kHalfNegLog2e), g.w, q.x, q.y);
      s_rgb[tid] = make_float4(c.x, c.y, c.z, q.z);
      s_idx[tid] = i;
    }
    __syncthreads();
    const int m = min(kBlock, n - done);
    for (int k = 0; k < m; ++k) {
      const int offk = n - 1 - done - k;
      bool contrib = offk < my_last;
      float dpx = 0.f, dpy = 0.f, dop = 0.f, dA = 0.f, dB = 0.f, dC = 0.f, dr = 0.f, dg = 0.f, db = 0.f;
      if (contrib) {
        const float4 g = s_geo[k];
        const float4 co = s_co[k];
        const float dx = __fsub_rn(g.x, xc), dy = __fsub_rn(g.y, yc);
        float qv = __fmul_rn(g.z, dx);
        qv = __fmaf_rn(g.w, dy, qv);
        float p2 = __fmul_rn(dx, qv);
        const float wv = __fmul_rn(co.x, dy);
        p2 = __fmaf_rn(wv, dy, p2);
        const float e = exp2_raster(p2);
        const float vv = __fmul_rn(co.y, e);
        const float alpha = fminf(vv, kAlphaMax);
        contrib = alpha >= kAlphaMin;
        if (contrib) {
          const float4 c = s_rgb[k];
          const float oma = 1.0f - alpha;
          T = T / oma;  // transmittance in front of this Gaussian
          const float wgt = alpha * T;
          dr = g0 * wgt;
          dg = g1 * wgt;
          db = g2 * wgt;
          const float Gk = T * (g0 * (c.x - R0) + g1 * (c.y - R1) + g2 * (c.z - R2));
          if (vv < kAlphaMax) {
            dop = Gk * e;
            const float dp = Gk * alpha;
            const float A = co.z, B = co.w, Cc = c.w;
            dpx = -dp * fmaf(A, dx, B * dy);
            dpy = -dp * fmaf(B, dx, Cc * dy);
            dA = -0.5f * dp * dx * dx;
            dB = -dp * dx * dy;
            dC = -0.5f * dp * dy * dy;
          }
          R0 = fmaf(c.x, alpha, oma * R0);
          R1 = fmaf(c.y, alpha, oma * R1);
          R2 = fmaf(c.z, alpha, oma * R2);
        }
      }
      if (__any_sync(0xffffffffu, contrib)) {
        dpx = warp_sum(dpx);
        dpy = warp_sum(dpy);
        dop = warp_sum(dop);
        dA = warp_sum(dA);
        dB = warp_sum(dB);
        dC = warp_sum(dC);
        dr = warp_sum(dr);
        dg = warp_sum(dg);
        db = warp_sum(db);
        if (lane == 0) {
          float4* dst = a.grad2d + 3 * (size_t)s_idx[k];
          atomicAdd(dst, make_float4(dpx, dpy, dop, 0.f));
          atomicAdd(dst + 1, make_float4(dA, dB, dC, 0.f));
          atomicAdd(dst + 2, make_float4(dr, dg, db, 0.f));
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_raster_fwd(const Records& rec, const uint32_t* vals, const uint32_t* ranges,
                              const DevCam& cam, const float bg[3], float* image, float* final_T,
                              int32_t* n_contrib, int32_t* last, cudaStream_t s) {
  FwdArgs a;
  a.xyzo = rec.xyzo; a.conic = rec.conic; a.rgb = rec.rgb;
  a.vals = vals; a.ranges = reinterpret_cast<const uint2*>(ranges);
  a.W = cam.width; a.H = cam.height; a.TW = cam.TW;
  a.bg0 = bg[0]; a.bg1 = bg[1]; a.bg2 = bg[2];
  a.image = image; a.final_T = final_T; a.n_contrib = n_contrib; a.last = last;
  raster_fwd_kernel<<<cam.TW * cam.TH, kBlock, 0, s>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_raster_bwd(const Records& rec, const uint32_t* vals, const uint32_t* ranges,
                              const DevCam& cam, const float bg[3], const float* final_T,
                              const int32_t* last, const float* dL_dimage, float4* grad2d,
                              int64_t n_records, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(grad2d, 0, (size_t)n_records * 3 * sizeof(float4), s);
  if (e != cudaSuccess) return e;
  BwdArgs a;
  a.xyzo = rec.xyzo; a.conic = rec.conic; a.rgb = rec.rgb;
  a.vals = vals; a.ranges = reinterpret_cast<const uint2*>(ranges);
  a.W = cam.width; a.H = cam.height; a.TW = cam.TW;
  a.bg0 = bg[0]; a.bg1 = bg[1]; a.bg2 = bg[2];
  a.final_T = final_T; a.last = last; a.dL_dimage = dL_dimage; a.grad2d = grad2d;
  raster_bwd_kernel<<<cam.TW * cam.TH, kBlock, 0, s>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace gs
