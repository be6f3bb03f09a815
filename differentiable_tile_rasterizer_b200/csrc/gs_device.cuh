// Device-side arithmetic of the rasterizer: constants, the software exp2 and
// the spherical-harmonic basis, in the fixed fp32 operation order that every
// kernel shares. The library is compiled with -fmad=false, so an expression
// is evaluated exactly as written; each fused multiply-add is an explicit
// __fmaf_rn.
#pragma once

#include <cstdint>

namespace gs {

// Taylor coefficients of 2^f = sum_k (ln 2)^k f^k / k!, rounded to fp32.
constexpr float kExp2C1 = 6.93147180559945309417e-1f;
constexpr float kExp2C2 = 2.40226506959100712334e-1f;
constexpr float kExp2C3 = 5.55041086648215799531e-2f;
constexpr float kExp2C4 = 9.61812910762847716198e-3f;
constexpr float kExp2C5 = 1.33335581464284434234e-3f;
constexpr float kExp2C6 = 1.54035303933816099544e-4f;
constexpr float kExp2C7 = 1.52527338040598402800e-5f;

constexpr float kLog2e = 1.44269504088896340736f;      // log2(e)
constexpr float kHalfNegLog2e = -0.72134752044448170368f; // -log2(e)/2
constexpr float kNegLog2e = -1.44269504088896340736f;   // -log2(e)

constexpr float kAlphaMin = 1.0f / 255.0f;
constexpr float kAlphaMax = 0.99f;
constexpr float kTMin = 1e-4f;
constexpr float kDilation = 0.3f;

// Real orthonormal SH normalisations with the Condon-Shortley sign, basis
// order l = 0..3, m = -l..l.
constexpr float kSH0 = 2.82094791773878143474e-1f;   // 1/(2 sqrt(pi))
constexpr float kSH1 = 4.88602511902919921586e-1f;   // sqrt(3/(4 pi))
constexpr float kSH2a = 1.09254843059207907054e+0f;  // sqrt(15/pi)/2
constexpr float kSH2b = 3.15391565252520006031e-1f;  // sqrt(5/pi)/4
constexpr float kSH2c = 5.46274215296039535272e-1f;  // sqrt(15/pi)/4
constexpr float kSH3a = 5.90043589926643510346e-1f;  // sqrt(35/(2 pi))/4
constexpr float kSH3b = 2.89061144264055405539e+0f;  // sqrt(105/pi)/2
constexpr float kSH3c = 4.57045799464465736158e-1f;  // sqrt(21/(2 pi))/4
constexpr float kSH3d = 3.73176332590115391414e-1f;  // sqrt(7/pi)/4
constexpr float kSH3e = 1.44530572132027702769e+0f;  // sqrt(105/pi)/4

// 1.5 * 2^23: adding it to |x| < 2^22 rounds x to the nearest integer (ties to
// even) in the low mantissa bits.
constexpr float kRoundMagic = 12582912.0f;

__device__ __forceinline__ float poly_exp2(float f) {
  float p = kExp2C7;
  p = __fmaf_rn(p, f, kExp2C6);
  p = __fmaf_rn(p, f, kExp2C5);
  p = __fmaf_rn(p, f, kExp2C4);
  p = __fmaf_rn(p, f, kExp2C3);
  p = __fmaf_rn(p, f, kExp2C2);
  p = __fmaf_rn(p, f, kExp2C1);
  p = __fmaf_rn(p, f, 1.0f);
  return p;
}

// Software exp2 of the specification: x in [-125, 127] -> p(x - n) * 2^n with
// n = rint(x); below -125 (or NaN) 0, above 127 +inf.
__device__ __forceinline__ float exp2_spec(float x) {
  if (!(x >= -125.0f)) return 0.0f;
  if (x > 127.0f) return __int_as_float(0x7f800000);
  const float t = __fadd_rn(x, kRoundMagic);       // kRoundMagic + rint(x)
  const float n = __fsub_rn(t, kRoundMagic);       // rint(x), exact
  const float f = __fsub_rn(x, n);                 // exact, |f| <= 1/2
  const float p = poly_exp2(f);
  // bits(t) = bits(kRoundMagic) + n and bits(kRoundMagic) << 23 == 0 (mod 2^32),
  // so (bits(t) << 23) adds n to the exponent field.
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Same value as exp2_spec for x in [-125, 127]; below -125 it returns 2^-125
// instead of 0. Used where the result only feeds alpha = o * e compared against
// 1/255 (both give a skip there) and x <= 127 holds.
__device__ __forceinline__ float exp2_raster(float x) {
  const float xc = fmaxf(x, -125.0f);
  const float t = __fadd_rn(xc, kRoundMagic);
  const float n = __fsub_rn(t, kRoundMagic);
  const float f = __fsub_rn(xc, n);
  const float p = poly_exp2(f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

__device__ __forceinline__ float exp_spec(float x) { return exp2_spec(__fmul_rn(x, kLog2e)); }

// ---- packed fp32 pairs (the f32x2 instructions of sm_100): each half is
// rounded exactly as the scalar round-to-nearest operation, so a pair of
// pixels can run one instruction stream with unchanged results.
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 r;
  asm("{.reg .b64 ra, rb, rd; mov.b64 ra, {%2, %3}; mov.b64 rb, {%4, %5}; add.rn.f32x2 rd, ra, rb;"
      " mov.b64 {%0, %1}, rd;}"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  float2 r;
  asm("{.reg .b64 ra, rb, rd; mov.b64 ra, {%2, %3}; mov.b64 rb, {%4, %5}; sub.rn.f32x2 rd, ra, rb;"
      " mov.b64 {%0, %1}, rd;}"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 r;
  asm("{.reg .b64 ra, rb, rd; mov.b64 ra, {%2, %3}; mov.b64 rb, {%4, %5}; mul.rn.f32x2 rd, ra, rb;"
      " mov.b64 {%0, %1}, rd;}"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 r;
  asm("{.reg .b64 ra, rb, rc, rd; mov.b64 ra, {%2, %3}; mov.b64 rb, {%4, %5}; mov.b64 rc, {%6, %7};"
      " fma.rn.f32x2 rd, ra, rb, rc; mov.b64 {%0, %1}, rd;}"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}
__device__ __forceinline__ float2 splat2(float v) { return make_float2(v, v); }

// exp2_raster on a pair (the same two results).
__device__ __forceinline__ float2 exp2_raster2(float2 x) {
  const float2 xc = make_float2(fmaxf(x.x, -125.0f), fmaxf(x.y, -125.0f));
  const float2 t = add2(xc, splat2(kRoundMagic));
  const float2 n = sub2(t, splat2(kRoundMagic));
  const float2 f = sub2(xc, n);
  float2 p = splat2(kExp2C7);
  p = fma2(p, f, splat2(kExp2C6));
  p = fma2(p, f, splat2(kExp2C5));
  p = fma2(p, f, splat2(kExp2C4));
  p = fma2(p, f, splat2(kExp2C3));
  p = fma2(p, f, splat2(kExp2C2));
  p = fma2(p, f, splat2(kExp2C1));
  p = fma2(p, f, splat2(1.0f));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// SH basis at a unit direction, Y[0..K-1], in the specification's order.
template <int K>
__device__ __forceinline__ void sh_basis(float x, float y, float z, float* Y) {
  Y[0] = kSH0;
  if (K <= 1) return;
  Y[1] = __fmul_rn(-kSH1, y);
  Y[2] = __fmul_rn(kSH1, z);
  Y[3] = __fmul_rn(-kSH1, x);
  if (K <= 4) return;
  const float xx = __fmul_rn(x, x), yy = __fmul_rn(y, y), zz = __fmul_rn(z, z);
  const float xy = __fmul_rn(x, y), yz = __fmul_rn(y, z), xz = __fmul_rn(x, z);
  Y[4] = __fmul_rn(kSH2a, xy);
  Y[5] = __fmul_rn(-kSH2a, yz);
  const float t6 = __fsub_rn(__fsub_rn(__fmul_rn(2.0f, zz), xx), yy);
  Y[6] = __fmul_rn(kSH2b, t6);
  Y[7] = __fmul_rn(-kSH2a, xz);
  const float t8 = __fsub_rn(xx, yy);
  Y[8] = __fmul_rn(kSH2c, t8);
  if (K <= 9) return;
  const float t9 = __fsub_rn(__fmul_rn(3.0f, xx), yy);
  Y[9] = __fmul_rn(__fmul_rn(-kSH3a, y), t9);
  Y[10] = __fmul_rn(__fmul_rn(kSH3b, xy), z);
  const float t11 = __fsub_rn(__fsub_rn(__fmul_rn(4.0f, zz), xx), yy);
  Y[11] = __fmul_rn(__fmul_rn(-kSH3c, y), t11);
  const float t12 = __fsub_rn(__fsub_rn(__fmul_rn(2.0f, zz), __fmul_rn(3.0f, xx)), __fmul_rn(3.0f, yy));
  Y[12] = __fmul_rn(__fmul_rn(kSH3d, z), t12);
  Y[13] = __fmul_rn(__fmul_rn(-kSH3c, x), t11);
  Y[14] = __fmul_rn(__fmul_rn(kSH3e, z), t8);
  const float t15 = __fsub_rn(xx, __fmul_rn(3.0f, yy));
  Y[15] = __fmul_rn(__fmul_rn(-kSH3a, x), t15);
}

__device__ __forceinline__ bool finitef(float v) { return fabsf(v) <= 3.402823466e38f; }

}  // namespace gs
