// Fused Adam step over block-quantised SH coefficients (the Spirula Studio
// quantised-training layout): 16-bit linear block codes of the values, 8-bit
// linear block codes of the logarithms of both Adam moments, one (lo, hi)
// pair per 256 consecutive Gaussians of a unit plane, fp32 gradients.
//
// One warp per block of 256 units; lane l takes units l, l + 32, ..., so
// every load and store of the warp is one contiguous run. The warp decodes,
// steps, finds the new bounds with shuffles and re-encodes, all in fp32 in
// the order fixed by the specification (no fused multiply-add except in the
// log2 polynomial, where it is part of the definition). HBM-bound: per unit
// 4 B of gradient + 4 B of codes read, 4 B of codes written.

#include "gs_device.cuh"
#include "gs_internal.cuh"

namespace gs {
namespace {

constexpr int kBlockUnits = 256;
constexpr int kUnitsPerLane = kBlockUnits / 32;
// RN(2 / ((2k + 1) ln 2)), k = 0..5: ln(m) = 2 atanh(s), s = (m - 1)/(m + 1)
constexpr float kL2c0 = 2.88539008177792681472f;
constexpr float kL2c1 = 0.96179669392597560491f;
constexpr float kL2c2 = 0.57707801635558536294f;
constexpr float kL2c3 = 0.41219858311113240210f;
constexpr float kL2c4 = 0.32059889797532520164f;
constexpr float kL2c5 = 0.26230818925253880134f;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kSqrt2 = 1.41421356237309504880f;
__device__ __forceinline__ float inf_f() { return __int_as_float(0x7f800000); }

// log2 of y >= 1: y = m 2^e with m in (sqrt(1/2), sqrt(2)] from the bits
// (exact), then e + s * P(s^2); log2(+inf) = +inf.
__device__ __forceinline__ float log2_spec(float y) {
  if (!(y < inf_f())) return y;
  const uint32_t bits = __float_as_uint(y);
  int e = (int)((bits >> 23) & 0xffu) - 127;
  float m = __uint_as_float((bits & 0x7fffffu) | 0x3f800000u);
  if (m > kSqrt2) {
    m = __fmul_rn(m, 0.5f);
    e += 1;
  }
  const float s = __fdiv_rn(__fsub_rn(m, 1.0f), __fadd_rn(m, 1.0f));
  const float s2 = __fmul_rn(s, s);
  float p = kL2c5;
  p = __fmaf_rn(p, s2, kL2c4);
  p = __fmaf_rn(p, s2, kL2c3);
  p = __fmaf_rn(p, s2, kL2c2);
  p = __fmaf_rn(p, s2, kL2c1);
  p = __fmaf_rn(p, s2, kL2c0);
  return __fadd_rn((float)e, __fmul_rn(s, p));
}
__device__ __forceinline__ float log1p_spec(float z) { return __fmul_rn(kLn2, log2_spec(__fadd_rn(1.0f, z))); }
__device__ __forceinline__ float expm1_spec(float y) { return __fsub_rn(exp2_spec(__fmul_rn(y, kLog2e)), 1.0f); }

// A block's code: lower bound, step = (hi - lo) / Q and inverse step
// Q / (hi - lo) (both 0 when hi == lo, so every code is 0). Decoding is one
// multiplication and one addition per unit, encoding one multiplication.
struct QBlock {
  float lo, step, inv;
};
__device__ __forceinline__ QBlock q_block(float2 b, float Q) {
  const float d = __fsub_rn(b.y, b.x);
  return d > 0.0f ? QBlock{b.x, __fdiv_rn(d, Q), __fdiv_rn(Q, d)} : QBlock{b.x, 0.0f, 0.0f};
}
__device__ __forceinline__ uint32_t q_encode(float x, const QBlock& b, float Q) {
  const float t = rintf(__fmul_rn(__fsub_rn(x, b.lo), b.inv));
  return t < 0.0f ? 0u : (t > Q ? (uint32_t)Q : (uint32_t)t);
}
__device__ __forceinline__ float q_decode(uint32_t q, const QBlock& b) {
  return __fadd_rn(b.lo, __fmul_rn(b.step, (float)q));
}
// r = 1 / e, the code scale's reciprocal
// (one log1p / expm1 per unit, the sign applied after: the same values as
// the two-branch form, -0 included)
__device__ __forceinline__ float m_to_log(float m, float r) {
  const float y = log1p_spec(__fmul_rn(fabsf(m), r));
  return m >= 0.0f ? y : -y;
}
__device__ __forceinline__ float m_from_log(float y, float e) {
  const float t = __fmul_rn(e, expm1_spec(fabsf(y)));
  return y >= 0.0f ? t : -t;
}
__device__ __forceinline__ float v_to_log(float v, float r) { return log1p_spec(__fmul_rn(__fsqrt_rn(v), r)); }
__device__ __forceinline__ float v_from_log(float y, float e) {
  const float s = __fmul_rn(e, expm1_spec(y));
  return __fmul_rn(s, s);
}

// Bounds of the valid values of a warp's block (lanes hold kUnitsPerLane each).
__device__ __forceinline__ float2 warp_bounds(const float (&x)[kUnitsPerLane], int lane, int n) {
  float lo = inf_f(), hi = -inf_f();
#pragma unroll
  for (int k = 0; k < kUnitsPerLane; ++k)
    if (lane + 32 * k < n) {
      lo = fminf(lo, x[k]);
      hi = fmaxf(hi, x[k]);
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  return make_float2(lo, hi);
}

template <class Code>
__global__ void __launch_bounds__(256) quant_encode_kernel(const float* x, int64_t U, int64_t N, int64_t nblk,
                                                           float Q, Code* codes, float2* bounds) {
  const int64_t wid = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (wid >= U * nblk) return;  // whole warps
  const int lane = threadIdx.x & 31;
  const int64_t u = wid / nblk, g0 = (wid % nblk) * kBlockUnits;
  const int n = (int)(N - g0 < kBlockUnits ? N - g0 : kBlockUnits);
  float v[kUnitsPerLane];
#pragma unroll
  for (int k = 0; k < kUnitsPerLane; ++k) v[k] = lane + 32 * k < n ? x[u * N + g0 + lane + 32 * k] : 0.0f;
  const float2 b = warp_bounds(v, lane, n);
  const QBlock qb = q_block(b, Q);
  Code* out = codes + u * nblk * kBlockUnits + g0;
#pragma unroll
  for (int k = 0; k < kUnitsPerLane; ++k)
    out[lane + 32 * k] = (Code)(lane + 32 * k < n ? q_encode(v[k], qb, Q) : 0u);
  if (lane == 0) bounds[wid] = b;
}

template <class Code>
__global__ void __launch_bounds__(256) quant_decode_kernel(const Code* codes, const float2* bounds, int64_t U,
                                                           int64_t N, int64_t nblk, float Q, float* x) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= U * N) return;
  const int64_t u = i / N, g = i % N;
  x[i] = q_decode(codes[u * nblk * kBlockUnits + g], q_block(bounds[u * nblk + g / kBlockUnits], Q));
}

struct AdamArgs {
  const float* grad;  // [U][N]
  int64_t U, N, nblk;
  uint16_t* pc;
  float2* pb;
  uint8_t* mc;
  float2* mb;
  uint8_t* vc;
  float2* vb;
  float lr, b1, ob1, b2, ob2, c1, c2, eps, ec, er;
};

__global__ void __launch_bounds__(256) adam_sh_quant_kernel(AdamArgs a) {
  const int64_t wid = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (wid >= a.U * a.nblk) return;  // whole warps
  const int lane = threadIdx.x & 31;
  const int64_t u = wid / a.nblk, g0 = (wid % a.nblk) * kBlockUnits;
  const int64_t row = u * a.nblk * kBlockUnits + g0;
  const int n = (int)(a.N - g0 < kBlockUnits ? a.N - g0 : kBlockUnits);
  const QBlock qp = q_block(a.pb[wid], 65535.0f), qm = q_block(a.mb[wid], 255.0f), qv = q_block(a.vb[wid], 255.0f);
  // every load of the lane first (independent, all in flight together)
  uint32_t cp[kUnitsPerLane], cm[kUnitsPerLane], cv[kUnitsPerLane];
  float gr[kUnitsPerLane];
#pragma unroll
  for (int k = 0; k < kUnitsPerLane; ++k) {
    const int i = lane + 32 * k;
    const bool ok = i < n;
    cp[k] = ok ? a.pc[row + i] : 0u;
    cm[k] = ok ? a.mc[row + i] : 0u;
    cv[k] = ok ? a.vc[row + i] : 0u;
    gr[k] = ok ? a.grad[u * a.N + g0 + i] : 0.0f;
  }
  float np[kUnitsPerLane], my[kUnitsPerLane], vy[kUnitsPerLane];
#pragma unroll
  for (int k = 0; k < kUnitsPerLane; ++k) {
    const int i = lane + 32 * k;
    np[k] = my[k] = vy[k] = 0.0f;
    if (i < n) {
      const float ph = q_decode(cp[k], qp);
      const float mh = m_from_log(q_decode(cm[k], qm), a.ec);
      const float vh = v_from_log(q_decode(cv[k], qv), a.ec);
      const float g = gr[k];
      const float m1 = __fadd_rn(__fmul_rn(a.b1, mh), __fmul_rn(a.ob1, g));
      const float v1 = __fadd_rn(__fmul_rn(a.b2, vh), __fmul_rn(a.ob2, __fmul_rn(g, g)));
      const float num = __fmul_rn(m1, a.c1);
      const float den = __fadd_rn(__fsqrt_rn(__fmul_rn(v1, a.c2)), a.eps);
      np[k] = __fsub_rn(ph, __fmul_rn(a.lr, __fdiv_rn(num, den)));
      my[k] = m_to_log(m1, a.er);
      vy[k] = v_to_log(v1, a.er);
    }
  }
  const float2 nb = warp_bounds(np, lane, n), nm = warp_bounds(my, lane, n), nv = warp_bounds(vy, lane, n);
  const QBlock q16 = q_block(nb, 65535.0f), qm8 = q_block(nm, 255.0f), qv8 = q_block(nv, 255.0f);
#pragma unroll
  for (int k = 0; k < kUnitsPerLane; ++k) {
    const int i = lane + 32 * k;
    const bool ok = i < n;
    a.pc[row + i] = (uint16_t)(ok ? q_encode(np[k], q16, 65535.0f) : 0u);
    a.mc[row + i] = (uint8_t)(ok ? q_encode(my[k], qm8, 255.0f) : 0u);
    a.vc[row + i] = (uint8_t)(ok ? q_encode(vy[k], qv8, 255.0f) : 0u);
  }
  if (lane == 0) {
    a.pb[wid] = nb;
    a.mb[wid] = nm;
    a.vb[wid] = nv;
  }
}

unsigned warps_grid(int64_t warps) { return (unsigned)((warps + 7) / 8); }

}  // namespace

int64_t quant_blocks(int64_t N) { return (N + kBlockUnits - 1) / kBlockUnits; }

cudaError_t launch_quant_encode(const float* x, int64_t U, int64_t N, int bits, void* codes, float* bounds,
                                cudaStream_t s) {
  const int64_t nblk = quant_blocks(N);
  if (U * nblk == 0) return cudaSuccess;
  float2* b = reinterpret_cast<float2*>(bounds);
  if (bits == 16)
    quant_encode_kernel<uint16_t><<<warps_grid(U * nblk), 256, 0, s>>>(x, U, N, nblk, 65535.0f,
                                                                      static_cast<uint16_t*>(codes), b);
  else
    quant_encode_kernel<uint8_t><<<warps_grid(U * nblk), 256, 0, s>>>(x, U, N, nblk, 255.0f,
                                                                     static_cast<uint8_t*>(codes), b);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_quant_decode(const void* codes, const float* bounds, int64_t U, int64_t N, int bits, float* x,
                                cudaStream_t s) {
  const int64_t nblk = quant_blocks(N);
  if (U * N == 0) return cudaSuccess;
  const float2* b = reinterpret_cast<const float2*>(bounds);
  if (bits == 16)
    quant_decode_kernel<uint16_t><<<grid_for(U * N, 256), 256, 0, s>>>(static_cast<const uint16_t*>(codes), b, U,
                                                                      N, nblk, 65535.0f, x);
  else
    quant_decode_kernel<uint8_t><<<grid_for(U * N, 256), 256, 0, s>>>(static_cast<const uint8_t*>(codes), b, U, N,
                                                                     nblk, 255.0f, x);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_adam_sh_quant(const float* grad, int64_t U, int64_t N, uint16_t* pc, float* pb, uint8_t* mc,
                                 float* mb, uint8_t* vc, float* vb, const float hp[10], cudaStream_t s) {
  AdamArgs a;
  a.grad = grad;
  a.U = U;
  a.N = N;
  a.nblk = quant_blocks(N);
  if (U * a.nblk == 0) return cudaSuccess;
  a.pc = pc;
  a.pb = reinterpret_cast<float2*>(pb);
  a.mc = mc;
  a.mb = reinterpret_cast<float2*>(mb);
  a.vc = vc;
  a.vb = reinterpret_cast<float2*>(vb);
  a.lr = hp[0];
  a.b1 = hp[1];
  a.ob1 = hp[2];
  a.b2 = hp[3];
  a.ob2 = hp[4];
  a.c1 = hp[5];
  a.c2 = hp[6];
  a.eps = hp[7];
  a.ec = hp[8];
  a.er = hp[9];
  adam_sh_quant_kernel<<<warps_grid(U * a.nblk), 256, 0, s>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace gs
