// Fused Adam step over block-quantised SH coefficients (the Spirula Studio
// quantised-training layout): 16-bit linear block codes of the values, 8-bit
// linear block codes of the logarithms of both Adam moments, one (lo, hi)
// pair per 256 consecutive Gaussians of a unit plane, fp32 gradients.
//
// One warp per block of 256 units; lane l takes the 8 consecutive units
// 8 l .. 8 l + 7, so its codes move as one 16-byte and two 8-byte words and
// every access of the warp is one contiguous run. The warp decodes,
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
__device__ __forceinline__ float q_decode_f(float q, const QBlock& b) { return __fadd_rn(b.lo, __fmul_rn(b.step, q)); }
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
  bool vec_codes;  // pc 16-byte, mc and vc 8-byte aligned
  bool vec_grad;   // grad 16-byte aligned and N % 4 == 0
};

// (float)q of a code q < 2^23, exactly: q placed in the mantissa of 2^23,
// minus 2^23 (the byte permute builds the bit pattern in one instruction).
__device__ __forceinline__ float code_u8(uint32_t w, int k) {
  return __fsub_rn(__uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u + (uint32_t)k)), 8388608.0f);
}
__device__ __forceinline__ float code_u16(uint32_t w, int hi) {
  return __fsub_rn(__uint_as_float(__byte_perm(w, 0x4B000000u, hi ? 0x7432u : 0x7410u)), 8388608.0f);
}
// q_encode with one conversion: round to nearest even and saturate to
// [0, 2^32 - 1] (NaN -> 0), then clamp to Q; the same code for every input.
__device__ __forceinline__ uint32_t q_encode_fast(float x, const QBlock& b, uint32_t Q) {
  return min(__float2uint_rn(__fmul_rn(__fsub_rn(x, b.lo), b.inv)), Q);
}

// Lane l of the warp takes the units 8 l .. 8 l + 7 of the block (so the
// codes of a lane are one 16-byte and two 8-byte words). kFull: all 256
// units of the block are valid.
template <bool kFull>
__device__ __forceinline__ void adam_block(const AdamArgs& a, int64_t wid, int lane) {
  const int64_t u = wid / a.nblk, g0 = (wid % a.nblk) * kBlockUnits;
  const int64_t row = u * a.nblk * kBlockUnits + g0 + 8 * lane;
  const int n = kFull ? kBlockUnits : (int)(a.N - g0);
  const int i0 = 8 * lane;
  const QBlock qp = q_block(a.pb[wid], 65535.0f), qm = q_block(a.mb[wid], 255.0f), qv = q_block(a.vb[wid], 255.0f);
  // codes: rows are padded to whole blocks, so the lane's 8 codes are in
  // bounds whether or not they are valid units
  uint32_t wp[4], wm[2], wv[2];
  if (a.vec_codes) {
    const uint4 p4 = *reinterpret_cast<const uint4*>(a.pc + row);
    const uint2 m2 = *reinterpret_cast<const uint2*>(a.mc + row);
    const uint2 v2 = *reinterpret_cast<const uint2*>(a.vc + row);
    wp[0] = p4.x; wp[1] = p4.y; wp[2] = p4.z; wp[3] = p4.w;
    wm[0] = m2.x; wm[1] = m2.y; wv[0] = v2.x; wv[1] = v2.y;
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) wp[k] = (uint32_t)a.pc[row + 2 * k] | ((uint32_t)a.pc[row + 2 * k + 1] << 16);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      wm[k] = (uint32_t)a.mc[row + 4 * k] | ((uint32_t)a.mc[row + 4 * k + 1] << 8) |
              ((uint32_t)a.mc[row + 4 * k + 2] << 16) | ((uint32_t)a.mc[row + 4 * k + 3] << 24);
      wv[k] = (uint32_t)a.vc[row + 4 * k] | ((uint32_t)a.vc[row + 4 * k + 1] << 8) |
              ((uint32_t)a.vc[row + 4 * k + 2] << 16) | ((uint32_t)a.vc[row + 4 * k + 3] << 24);
    }
  }
  const float* gsrc = a.grad + u * a.N + g0 + i0;
  float gr[8];
  if (a.vec_grad && (kFull || i0 + 8 <= n)) {
    const float4 g0v = *reinterpret_cast<const float4*>(gsrc), g1v = *reinterpret_cast<const float4*>(gsrc + 4);
    gr[0] = g0v.x; gr[1] = g0v.y; gr[2] = g0v.z; gr[3] = g0v.w;
    gr[4] = g1v.x; gr[5] = g1v.y; gr[6] = g1v.z; gr[7] = g1v.w;
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) gr[k] = (kFull || i0 + k < n) ? gsrc[k] : 0.0f;
  }
  float np[8], my[8], vy[8];
  float plo = inf_f(), phi = -inf_f(), mlo = inf_f(), mhi = -inf_f(), vlo = inf_f(), vhi = -inf_f();
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float ph = q_decode_f(code_u16(wp[k >> 1], k & 1), qp);
    const float mh = m_from_log(q_decode_f(code_u8(wm[k >> 2], k & 3), qm), a.ec);
    const float vh = v_from_log(q_decode_f(code_u8(wv[k >> 2], k & 3), qv), a.ec);
    const float g = gr[k];
    const float m1 = __fadd_rn(__fmul_rn(a.b1, mh), __fmul_rn(a.ob1, g));
    const float v1 = __fadd_rn(__fmul_rn(a.b2, vh), __fmul_rn(a.ob2, __fmul_rn(g, g)));
    const float num = __fmul_rn(m1, a.c1);
    const float den = __fadd_rn(__fsqrt_rn(__fmul_rn(v1, a.c2)), a.eps);
    np[k] = __fsub_rn(ph, __fmul_rn(a.lr, __fdiv_rn(num, den)));
    my[k] = m_to_log(m1, a.er);
    vy[k] = v_to_log(v1, a.er);
    if (kFull || i0 + k < n) {
      plo = fminf(plo, np[k]); phi = fmaxf(phi, np[k]);
      mlo = fminf(mlo, my[k]); mhi = fmaxf(mhi, my[k]);
      vlo = fminf(vlo, vy[k]); vhi = fmaxf(vhi, vy[k]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    plo = fminf(plo, __shfl_xor_sync(0xffffffffu, plo, o));
    phi = fmaxf(phi, __shfl_xor_sync(0xffffffffu, phi, o));
    mlo = fminf(mlo, __shfl_xor_sync(0xffffffffu, mlo, o));
    mhi = fmaxf(mhi, __shfl_xor_sync(0xffffffffu, mhi, o));
    vlo = fminf(vlo, __shfl_xor_sync(0xffffffffu, vlo, o));
    vhi = fmaxf(vhi, __shfl_xor_sync(0xffffffffu, vhi, o));
  }
  const float2 nb = make_float2(plo, phi), nm = make_float2(mlo, mhi), nv = make_float2(vlo, vhi);
  const QBlock q16 = q_block(nb, 65535.0f), qm8 = q_block(nm, 255.0f), qv8 = q_block(nv, 255.0f);
  uint32_t op[4] = {0u, 0u, 0u, 0u}, om[2] = {0u, 0u}, ov[2] = {0u, 0u};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    if (kFull || i0 + k < n) {  // invalid units keep code 0
      op[k >> 1] |= q_encode_fast(np[k], q16, 65535u) << (16 * (k & 1));
      om[k >> 2] |= q_encode_fast(my[k], qm8, 255u) << (8 * (k & 3));
      ov[k >> 2] |= q_encode_fast(vy[k], qv8, 255u) << (8 * (k & 3));
    }
  }
  if (a.vec_codes) {
    *reinterpret_cast<uint4*>(a.pc + row) = make_uint4(op[0], op[1], op[2], op[3]);
    *reinterpret_cast<uint2*>(a.mc + row) = make_uint2(om[0], om[1]);
    *reinterpret_cast<uint2*>(a.vc + row) = make_uint2(ov[0], ov[1]);
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      a.pc[row + k] = (uint16_t)(op[k >> 1] >> (16 * (k & 1)));
      a.mc[row + k] = (uint8_t)(om[k >> 2] >> (8 * (k & 3)));
      a.vc[row + k] = (uint8_t)(ov[k >> 2] >> (8 * (k & 3)));
    }
  }
  if (lane == 0) {
    a.pb[wid] = nb;
    a.mb[wid] = nm;
    a.vb[wid] = nv;
  }
}

__global__ void __launch_bounds__(256) adam_sh_quant_kernel(AdamArgs a) {
  const int64_t wid = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (wid >= a.U * a.nblk) return;  // whole warps
  const int lane = threadIdx.x & 31;
  if ((wid % a.nblk) * kBlockUnits + kBlockUnits <= a.N)
    adam_block<true>(a, wid, lane);
  else
    adam_block<false>(a, wid, lane);
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
  a.vec_codes = reinterpret_cast<uintptr_t>(pc) % 16 == 0 && reinterpret_cast<uintptr_t>(mc) % 8 == 0 &&
                reinterpret_cast<uintptr_t>(vc) % 8 == 0;
  a.vec_grad = reinterpret_cast<uintptr_t>(grad) % 16 == 0 && N % 4 == 0;
  adam_sh_quant_kernel<<<warps_grid(U * a.nblk), 256, 0, s>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace gs
