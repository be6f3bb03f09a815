/*
 * CPU oracle for differentiable tile rasterization of 3D Gaussian splats.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library. It shares no code,
 * header, table or constant generator with the CUDA library; the only thing
 * both consume is the seeded input generator.
 *
 * What it computes (the method, stage by stage):
 *   cull        per-view active set: distance-LOD gate plus importance mask
 *               (BlitzGS write-up, section 2.3 "视图层级精细化修剪": a distance
 *               threshold drops far Gaussians, an importance mask drops
 *               low-weight ones). The mask keeps weights at or above the
 *               value of rank floor(q*N) among all N weights.
 *   preprocess  projection of each Gaussian: camera-space mean t = W mu + t0,
 *               covariance Sigma = R S S^T R^T, screen covariance
 *               Sigma' = J W Sigma W^T J^T + 0.3 I, conic = Sigma'^-1,
 *               3-sigma radius ceil(3 sqrt(lambda_max)), 16x16 tile rect,
 *               opacity sigmoid, degree<=3 spherical-harmonic colour.
 *               The split into per-Gaussian stages follows the Gsplat
 *               description (像素扩散与CUDA内核优化, section 三.2); SH3 colour
 *               sizing follows the Spirula Studio page, section "先算一笔账".
 *   bin/sort    64-bit keys (tile_id << 32 | depth bits), stable sort, per-tile
 *               [start, end) ranges.
 *   raster      per-pixel front-to-back alpha compositing over the tile's list
 *               (the 4D-GS page, section "技术架构与关键机制": tiled
 *               rasterization with per-pixel alpha blending):
 *               alpha = min(0.99, o exp(-1/2 d^T conic d)), skip alpha < 1/255,
 *               stop once T < 1e-4 (the Gaussian that crosses is blended).
 *   backward    exact derivatives of the above with every discrete decision
 *               (visibility, tile lists, skips, clamps, stop) held fixed.
 *
 * Two arithmetic modes.
 *   fp32 spec mode: single precision, each operation in the order of the
 *     arithmetic specification, every fused multiply-add explicit (fmaf), no
 *     contraction (built with -ffp-contract=off), and exp computed by the
 *     software exp2 below. Integer results (radius, rect, tiles, keys, order,
 *     ranges, contributor counts) and the decisions behind them come from here.
 *   fp64 mode: the same formulas in double precision with libm exp; used for
 *     closed-form pins, finite differences and the reference gradients.
 *
 * Software exp2 (spec): for x in [-125, 127], n = rint(x), f = x - n (exact,
 * |f| <= 1/2), p = Horner evaluation of the degree-7 Taylor polynomial of 2^f
 * = sum (ln 2)^k f^k / k! with coefficients rounded to fp32, result p * 2^n
 * (exact scaling). x < -125 (or NaN) gives 0, x > 127 gives +inf. This is
 * Cody-Waite style range reduction with a single-constant split (log2 domain,
 * so the reduction is exact) followed by a Taylor polynomial.
 */

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <limits>
#include <type_traits>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_API extern "C" __attribute__((visibility("default")))

namespace {

// ---------------------------------------------------------------- constants
struct Constants {
  float e2c[8];      // RN((ln 2)^k / k!)
  float l2e;         // RN(log2 e)
  float kh, kf;      // RN(-log2(e)/2), RN(-log2 e)
  float alpha_min, alpha_max, t_min, dilation;
  float shf[16];     // SH normalisation constants (with sign), fp32
  double shd[16];    // same, fp64
  Constants() {
    const double ln2 = std::log(2.0);
    const double pi = std::acos(-1.0);
    double term = 1.0;
    e2c[0] = 1.0f;
    for (int k = 1; k < 8; ++k) {
      term = term * ln2 / (double)k;
      e2c[k] = (float)term;
    }
    l2e = (float)(1.0 / ln2);
    kh = (float)(-0.5 / ln2);
    kf = (float)(-1.0 / ln2);
    alpha_min = (float)(1.0 / 255.0);
    alpha_max = (float)0.99;
    t_min = (float)1e-4;
    dilation = (float)0.3;
    // Real orthonormal spherical harmonics, l <= 3, ordered m = -l..l, with
    // the Condon-Shortley sign folded into the constants.
    shd[0] = 1.0 / (2.0 * std::sqrt(pi));
    const double c1 = std::sqrt(3.0 / (4.0 * pi));
    shd[1] = -c1;
    shd[2] = c1;
    shd[3] = -c1;
    const double a15 = std::sqrt(15.0 / pi);
    shd[4] = a15 / 2.0;
    shd[5] = -a15 / 2.0;
    shd[6] = std::sqrt(5.0 / pi) / 4.0;
    shd[7] = -a15 / 2.0;
    shd[8] = a15 / 4.0;
    const double a35 = std::sqrt(35.0 / (2.0 * pi)) / 4.0;
    const double a105 = std::sqrt(105.0 / pi);
    const double a21 = std::sqrt(21.0 / (2.0 * pi)) / 4.0;
    shd[9] = -a35;
    shd[10] = a105 / 2.0;
    shd[11] = -a21;
    shd[12] = std::sqrt(7.0 / pi) / 4.0;
    shd[13] = -a21;
    shd[14] = a105 / 4.0;
    shd[15] = -a35;
    for (int k = 0; k < 16; ++k) shf[k] = (float)shd[k];
  }
};
const Constants KC;

// ------------------------------------------------------ software exp2 (fp32)
float exp2_spec(float x) {
  if (!(x >= -125.0f)) return 0.0f;
  if (x > 127.0f) return std::numeric_limits<float>::infinity();
  const float n = std::rint(x);
  const float f = x - n;
  float p = KC.e2c[7];
  for (int k = 6; k >= 0; --k) p = std::fmaf(p, f, KC.e2c[k]);
  return std::ldexp(p, (int)n);
}
inline float exp_spec(float x) { return exp2_spec(x * KC.l2e); }

// --------------------------------------------------------- arithmetic modes
template <class R> struct Ar;
template <> struct Ar<float> {
  static float fma(float a, float b, float c) { return std::fmaf(a, b, c); }
  static float exp(float x) { return exp_spec(x); }
  static float sqrt(float x) { return std::sqrt(x); }
  static float dil() { return KC.dilation; }
  static float sh(int k) { return KC.shf[k]; }
};
template <> struct Ar<double> {
  static double fma(double a, double b, double c) { return std::fma(a, b, c); }
  static double exp(double x) { return std::exp(x); }
  static double sqrt(double x) { return std::sqrt(x); }
  static double dil() { return 0.3; }
  static double sh(int k) { return KC.shd[k]; }
};

struct Cam {
  float W[9], t[3], campos[3], fx, fy, cx, cy, near_z;
  int width, height, TW, TH;
};
Cam make_cam(const float* c, int width, int height) {
  Cam k;
  for (int i = 0; i < 9; ++i) k.W[i] = c[i];
  for (int i = 0; i < 3; ++i) k.t[i] = c[9 + i];
  for (int i = 0; i < 3; ++i) k.campos[i] = c[12 + i];
  k.fx = c[15]; k.fy = c[16]; k.cx = c[17]; k.cy = c[18]; k.near_z = c[19];
  k.width = width; k.height = height;
  k.TW = (width + 15) / 16; k.TH = (height + 15) / 16;
  return k;
}

// ----------------------------------------------------------- SH basis (spec)
template <class R>
void sh_basis(R x, R y, R z, int K, R Y[16]) {
  typedef Ar<R> A;
  Y[0] = A::sh(0);
  if (K <= 1) return;
  Y[1] = A::sh(1) * y;
  Y[2] = A::sh(2) * z;
  Y[3] = A::sh(3) * x;
  if (K <= 4) return;
  const R xx = x * x, yy = y * y, zz = z * z;
  const R xy = x * y, yz = y * z, xz = x * z;
  Y[4] = A::sh(4) * xy;
  Y[5] = A::sh(5) * yz;
  const R t6 = ((R(2) * zz) - xx) - yy;
  Y[6] = A::sh(6) * t6;
  Y[7] = A::sh(7) * xz;
  const R t8 = xx - yy;
  Y[8] = A::sh(8) * t8;
  if (K <= 9) return;
  const R t9 = (R(3) * xx) - yy;
  Y[9] = (A::sh(9) * y) * t9;
  Y[10] = (A::sh(10) * xy) * z;
  const R t11 = ((R(4) * zz) - xx) - yy;
  Y[11] = (A::sh(11) * y) * t11;
  const R t12 = ((R(2) * zz) - (R(3) * xx)) - (R(3) * yy);
  Y[12] = (A::sh(12) * z) * t12;
  Y[13] = (A::sh(13) * x) * t11;
  Y[14] = (A::sh(14) * z) * t8;
  const R t15 = xx - (R(3) * yy);
  Y[15] = (A::sh(15) * x) * t15;
}

// Gradient of each basis polynomial with respect to (x, y, z), fp64.
void sh_basis_grad(double x, double y, double z, int K, double G[16][3]) {
  const double* c = KC.shd;
  for (int k = 0; k < 16; ++k) G[k][0] = G[k][1] = G[k][2] = 0.0;
  if (K <= 1) return;
  G[1][1] = c[1];
  G[2][2] = c[2];
  G[3][0] = c[3];
  if (K <= 4) return;
  G[4][0] = c[4] * y; G[4][1] = c[4] * x;
  G[5][1] = c[5] * z; G[5][2] = c[5] * y;
  G[6][0] = -2.0 * c[6] * x; G[6][1] = -2.0 * c[6] * y; G[6][2] = 4.0 * c[6] * z;
  G[7][0] = c[7] * z; G[7][2] = c[7] * x;
  G[8][0] = 2.0 * c[8] * x; G[8][1] = -2.0 * c[8] * y;
  if (K <= 9) return;
  const double xx = x * x, yy = y * y, zz = z * z;
  G[9][0] = c[9] * 6.0 * x * y; G[9][1] = c[9] * (3.0 * xx - 3.0 * yy);
  G[10][0] = c[10] * y * z; G[10][1] = c[10] * x * z; G[10][2] = c[10] * x * y;
  G[11][0] = c[11] * (-2.0 * x * y);
  G[11][1] = c[11] * (4.0 * zz - xx - 3.0 * yy);
  G[11][2] = c[11] * 8.0 * y * z;
  G[12][0] = c[12] * (-6.0 * x * z);
  G[12][1] = c[12] * (-6.0 * y * z);
  G[12][2] = c[12] * (6.0 * zz - 3.0 * xx - 3.0 * yy);
  G[13][0] = c[13] * (4.0 * zz - 3.0 * xx - yy);
  G[13][1] = c[13] * (-2.0 * x * y);
  G[13][2] = c[13] * 8.0 * x * z;
  G[14][0] = c[14] * 2.0 * x * z; G[14][1] = c[14] * (-2.0 * y * z);
  G[14][2] = c[14] * (xx - yy);
  G[15][0] = c[15] * (3.0 * xx - 3.0 * yy); G[15][1] = c[15] * (-6.0 * x * y);
}

// Magnitude versions of the basis and its gradient: every polynomial
// evaluated on |x|, |y|, |z| with its subtractions turned into additions and
// |constant|. They bound the size of the terms an fp32 evaluation sums, which
// sets its rounding error where a polynomial nearly cancels.
void sh_basis_abs(double x, double y, double z, int K, double Y[16]) {
  x = std::fabs(x); y = std::fabs(y); z = std::fabs(z);
  const double* c = KC.shd;
  double a[16];
  for (int k = 0; k < 16; ++k) a[k] = std::fabs(c[k]);
  const double xx = x * x, yy = y * y, zz = z * z;
  Y[0] = a[0];
  Y[1] = a[1] * y; Y[2] = a[2] * z; Y[3] = a[3] * x;
  Y[4] = a[4] * x * y; Y[5] = a[5] * y * z; Y[6] = a[6] * (2 * zz + xx + yy);
  Y[7] = a[7] * x * z; Y[8] = a[8] * (xx + yy);
  Y[9] = a[9] * y * (3 * xx + yy); Y[10] = a[10] * x * y * z;
  Y[11] = a[11] * y * (4 * zz + xx + yy); Y[12] = a[12] * z * (2 * zz + 3 * xx + 3 * yy);
  Y[13] = a[13] * x * (4 * zz + xx + yy); Y[14] = a[14] * z * (xx + yy);
  Y[15] = a[15] * x * (xx + 3 * yy);
  for (int k = K; k < 16; ++k) Y[k] = 0.0;
}

void sh_basis_grad_abs(double x, double y, double z, int K, double G[16][3]) {
  sh_basis_grad(std::fabs(x), std::fabs(y), std::fabs(z), K, G);
  for (int k = 0; k < 16; ++k)
    for (int m = 0; m < 3; ++m) G[k][m] = std::fabs(G[k][m]);
  if (K <= 9) return;
  x = std::fabs(x); y = std::fabs(y); z = std::fabs(z);
  const double xx = x * x, yy = y * y, zz = z * z;
  const double* c = KC.shd;
  G[9][1] = std::fabs(c[9]) * (3 * xx + 3 * yy);
  G[11][1] = std::fabs(c[11]) * (4 * zz + xx + 3 * yy);
  G[12][2] = std::fabs(c[12]) * (6 * zz + 3 * xx + 3 * yy);
  G[13][0] = std::fabs(c[13]) * (4 * zz + 3 * xx + yy);
  G[14][2] = std::fabs(c[14]) * (xx + yy);
  G[15][0] = std::fabs(c[15]) * (3 * xx + 3 * yy);
  G[6][2] = std::fabs(c[6]) * 4 * z;
  G[8][0] = std::fabs(c[8]) * 2 * x;
}

// ------------------------------------------------------------- projection
template <class R>
struct Proj {
  bool visible;
  R px, py, depth, opacity, A, B, C;
  R rgb[3], pre[3];
  int radius, rect[4], tiles;
};

template <class R>
bool finite3(R a, R b, R c) { return std::isfinite(a) && std::isfinite(b) && std::isfinite(c); }

// Project one Gaussian. `coef` points at the K*3 SH coefficients (k-major,
// channel-minor) already gathered for this Gaussian. `clamp_fixed` (optional,
// fp64 mode) imposes the colour-clamp decisions of an fp32 run.
template <class R>
void project_one(const Cam& cam, const R mu[3], const R ls[3], const R q[4], R logit,
                 const R* coef, int K, Proj<R>& o, const bool* clamp_fixed) {
  typedef Ar<R> A;
  std::memset(&o, 0, sizeof(o));
  o.visible = false;
  if (!finite3(mu[0], mu[1], mu[2]) || !finite3(ls[0], ls[1], ls[2]) ||
      !finite3(q[0], q[1], q[2]) || !std::isfinite(q[3]) || !std::isfinite(logit))
    return;
  const R W[9] = {R(cam.W[0]), R(cam.W[1]), R(cam.W[2]), R(cam.W[3]), R(cam.W[4]),
                  R(cam.W[5]), R(cam.W[6]), R(cam.W[7]), R(cam.W[8])};
  // 1. camera space
  R t[3];
  for (int r = 0; r < 3; ++r) {
    R v = W[3 * r + 0] * mu[0];
    v = A::fma(W[3 * r + 1], mu[1], v);
    v = A::fma(W[3 * r + 2], mu[2], v);
    t[r] = v + R(cam.t[r]);
  }
  if (!(t[2] > R(cam.near_z))) return;
  // 2. scales
  const R s[3] = {A::exp(ls[0]), A::exp(ls[1]), A::exp(ls[2])};
  // 3. quaternion (w, x, y, z), normalised
  R n2 = q[0] * q[0];
  n2 = A::fma(q[1], q[1], n2);
  n2 = A::fma(q[2], q[2], n2);
  n2 = A::fma(q[3], q[3], n2);
  if (!(n2 > R(0))) return;
  const R nq = A::sqrt(n2);
  const R w = q[0] / nq, x = q[1] / nq, y = q[2] / nq, z = q[3] / nq;
  // 4. rotation matrix
  const R xx = x * x, yy = y * y, zz = z * z, xy = x * y, xz = x * z, yz = y * z;
  const R wx = w * x, wy = w * y, wz = w * z;
  R Rq[9];
  Rq[0] = R(1) - R(2) * (yy + zz);
  Rq[1] = R(2) * (xy - wz);
  Rq[2] = R(2) * (xz + wy);
  Rq[3] = R(2) * (xy + wz);
  Rq[4] = R(1) - R(2) * (xx + zz);
  Rq[5] = R(2) * (yz - wx);
  Rq[6] = R(2) * (xz - wy);
  Rq[7] = R(2) * (yz + wx);
  Rq[8] = R(1) - R(2) * (xx + yy);
  // 5. M = Rq diag(s)
  R M[9];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) M[3 * i + j] = Rq[3 * i + j] * s[j];
  // 6. Sigma = M M^T
  R S[9];
  for (int i = 0; i < 3; ++i)
    for (int j = i; j < 3; ++j) {
      R v = M[3 * i + 0] * M[3 * j + 0];
      v = A::fma(M[3 * i + 1], M[3 * j + 1], v);
      v = A::fma(M[3 * i + 2], M[3 * j + 2], v);
      S[3 * i + j] = v;
      S[3 * j + i] = v;
    }
  // 7. Jacobian of the perspective map at t
  const R fx = R(cam.fx), fy = R(cam.fy);
  const R tz2 = t[2] * t[2];
  const R j00 = fx / t[2], j11 = fy / t[2];
  const R j02 = -((fx * t[0]) / tz2), j12 = -((fy * t[1]) / tz2);
  // 8. T = J W (2x3)
  R T[6];
  for (int j = 0; j < 3; ++j) {
    T[j] = A::fma(j02, W[6 + j], j00 * W[j]);
    T[3 + j] = A::fma(j12, W[6 + j], j11 * W[3 + j]);
  }
  // 9. U = T Sigma (2x3)
  R U[6];
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < 3; ++j) {
      R v = T[3 * i + 0] * S[j];
      v = A::fma(T[3 * i + 1], S[3 + j], v);
      v = A::fma(T[3 * i + 2], S[6 + j], v);
      U[3 * i + j] = v;
    }
  // 10. Sigma' = U T^T + 0.3 I
  R c00 = U[0] * T[0];
  c00 = A::fma(U[1], T[1], c00);
  c00 = A::fma(U[2], T[2], c00);
  R c01 = U[0] * T[3];
  c01 = A::fma(U[1], T[4], c01);
  c01 = A::fma(U[2], T[5], c01);
  R c11 = U[3] * T[3];
  c11 = A::fma(U[4], T[4], c11);
  c11 = A::fma(U[5], T[5], c11);
  const R a = c00 + A::dil(), b = c01, c = c11 + A::dil();
  // 11. conic = Sigma'^-1
  const R bb = b * b;
  const R det = A::fma(a, c, -bb);
  if (!(det > R(0))) return;
  const R cA = c / det, cB = (-b) / det, cC = a / det;
  // 12. 3-sigma radius from the larger eigenvalue
  const R mid = R(0.5) * (a + c);
  R d = A::fma(mid, mid, -det);
  if (!(d > R(0))) d = R(0);
  const R lam = mid + A::sqrt(d);
  const R rf = std::ceil(R(3) * A::sqrt(lam));
  // 13. projected centre
  const R xn = t[0] / t[2], yn = t[1] / t[2];
  const R px = A::fma(fx, xn, R(cam.cx));
  const R py = A::fma(fy, yn, R(cam.cy));
  if (!finite3(px, py, rf) || !finite3(cA, cB, cC)) return;
  // 14. tile rect, end-exclusive, clamped to the grid
  auto clampg = [](R v, R hi) { return v < R(0) ? R(0) : (v > hi ? hi : v); };
  const R TWf = R(cam.TW), THf = R(cam.TH), inv16 = R(0.0625);
  const int x0 = (int)clampg(std::floor((px - rf) * inv16), TWf);
  const int x1 = (int)clampg(std::floor((px + rf) * inv16) + R(1), TWf);
  const int y0 = (int)clampg(std::floor((py - rf) * inv16), THf);
  const int y1 = (int)clampg(std::floor((py + rf) * inv16) + R(1), THf);
  const int tiles = (x1 - x0) * (y1 - y0);
  if (tiles <= 0) return;
  // 15. opacity
  const R op = R(1) / (R(1) + A::exp(-logit));
  // 16. colour from SH at the viewing direction
  const R dx = mu[0] - R(cam.campos[0]), dy = mu[1] - R(cam.campos[1]),
          dz = mu[2] - R(cam.campos[2]);
  R nn = dx * dx;
  nn = A::fma(dy, dy, nn);
  nn = A::fma(dz, dz, nn);
  const R nd = A::sqrt(nn);
  R Y[16];
  sh_basis<R>(dx / nd, dy / nd, dz / nd, K, Y);
  for (int ch = 0; ch < 3; ++ch) {
    R acc = Y[0] * coef[ch];
    for (int k = 1; k < K; ++k) acc = A::fma(Y[k], coef[3 * k + ch], acc);
    const R v = acc + R(0.5);
    o.pre[ch] = v;
    bool pass = v > R(0);
    if (clamp_fixed) pass = !clamp_fixed[ch];
    o.rgb[ch] = pass ? v : R(0);
  }
  // an infinite colour (from infinite SH coefficients) culls, like a non-finite parameter
  if (!finite3(o.rgb[0], o.rgb[1], o.rgb[2])) return;
  o.visible = true;
  o.px = px; o.py = py; o.depth = t[2]; o.opacity = op;
  o.A = cA; o.B = cB; o.C = cC;
  o.radius = rf < R(1073741824.0) ? (int)rf : 1073741824;
  o.rect[0] = x0; o.rect[1] = y0; o.rect[2] = x1; o.rect[3] = y1;
  o.tiles = tiles;
}

// Gather one Gaussian's parameters from the SoA planes.
template <class R, class Src>
void gather(const Src* means, const Src* ls, const Src* quats, const Src* logits,
            const Src* sh, int K, int64_t N, int64_t g, R mu[3], R l[3], R q[4], R& lg,
            R* coef) {
  for (int j = 0; j < 3; ++j) mu[j] = R(means[j * N + g]);
  for (int j = 0; j < 3; ++j) l[j] = R(ls[j * N + g]);
  for (int j = 0; j < 4; ++j) q[j] = R(quats[j * N + g]);
  lg = R(logits[g]);
  for (int k = 0; k < 3 * K; ++k) coef[k] = R(sh[(int64_t)k * N + g]);
}

// ------------------------------------------------------------- pixel walk
// Front-to-back walk of one pixel over its tile's list in fp32 spec mode.
// Calls blend(j, i, alpha, clamped, e) for every blended entry, in order
// (e = exp2 of the pair's exponent, alpha = min(0.99, o e), both fp32).
struct Rec32 {
  const float* xyzo;
  const float* conic;
  const float* rgb;
};
template <class F>
void walk_pixel(const Rec32& r, const uint32_t* vals, uint32_t start, uint32_t end,
                float xc, float yc, float& T, int& n, int& last, F blend) {
  T = 1.0f;
  n = 0;
  last = 0;
  for (uint32_t j = start; j < end; ++j) {
    const uint32_t i = vals[j];
    const float px = r.xyzo[4 * (size_t)i + 0], py = r.xyzo[4 * (size_t)i + 1];
    const float op = r.xyzo[4 * (size_t)i + 3];
    const float a2 = r.conic[4 * (size_t)i + 0] * KC.kh;
    const float b2 = r.conic[4 * (size_t)i + 1] * KC.kf;
    const float c2 = r.conic[4 * (size_t)i + 2] * KC.kh;
    const float dx = px - xc, dy = py - yc;
    float qv = a2 * dx;
    qv = std::fmaf(b2, dy, qv);
    float p2 = dx * qv;
    const float wv = c2 * dy;
    p2 = std::fmaf(wv, dy, p2);
    const float e = exp2_spec(p2);
    const float v = op * e;
    const bool clamped = !(v < KC.alpha_max);
    const float alpha = clamped ? KC.alpha_max : v;
    if (alpha < KC.alpha_min) continue;
    blend(j, i, alpha, clamped, e);
    T = T * (1.0f - alpha);
    n += 1;
    last = (int)(j - start + 1);
    if (T < KC.t_min) break;
  }
}

int64_t tile_count(int W, int H) { return (int64_t)((W + 15) / 16) * ((H + 15) / 16); }

}  // namespace

// =================================================================== API

// Library self-description and constants used by the pins.
OR_API int or_version(void) { return 1; }

OR_API int or_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

OR_API void or_constants(float* out /* 32 */) {
  for (int k = 0; k < 8; ++k) out[k] = KC.e2c[k];
  out[8] = KC.l2e; out[9] = KC.kh; out[10] = KC.kf;
  out[11] = KC.alpha_min; out[12] = KC.alpha_max; out[13] = KC.t_min; out[14] = KC.dilation;
  for (int k = 0; k < 16; ++k) out[16 + k] = KC.shf[k];
}

OR_API void or_exp2_array(const float* x, float* y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = exp2_spec(x[i]);
}

OR_API void or_sh_basis_f64(const double* dirs, int64_t n, double* Y) {
  for (int64_t i = 0; i < n; ++i) sh_basis<double>(dirs[3 * i], dirs[3 * i + 1], dirs[3 * i + 2], 16, Y + 16 * i);
}
OR_API void or_sh_basis_f32(const float* dirs, int64_t n, float* Y) {
  for (int64_t i = 0; i < n; ++i) sh_basis<float>(dirs[3 * i], dirs[3 * i + 1], dirs[3 * i + 2], 16, Y + 16 * i);
}
OR_API void or_sh_basis_grad_f64(const double* dirs, int64_t n, double* G /* n x 16 x 3 */) {
  for (int64_t i = 0; i < n; ++i) {
    double g[16][3];
    sh_basis_grad(dirs[3 * i], dirs[3 * i + 1], dirs[3 * i + 2], 16, g);
    std::memcpy(G + 48 * i, g, sizeof(g));
  }
}

// ---- cull (LOD gate + importance quantile mask + order-preserving compaction)
static uint32_t order_key(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
static float from_order_key(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

OR_API int or_cull(const float* means, const float* importance, int64_t N, const float* campos,
                   float lod_dist, float q, uint8_t* mask, int32_t* active_idx,
                   int64_t* n_active, float* tau_out) {
  if (N < 0 || !(q >= 0.0f) || q >= 1.0f) return 1;
  const bool use_lod = lod_dist > 0.0f;
  const bool use_imp = q > 0.0f && importance != nullptr && N > 0;
  const float dd = lod_dist * lod_dist;
  float tau = 0.0f;
  if (use_imp) {
    const int64_t rank = (int64_t)std::floor((double)q * (double)N);
    std::vector<uint32_t> keys(N);
    for (int64_t g = 0; g < N; ++g) keys[g] = order_key(importance[g]);
    std::nth_element(keys.begin(), keys.begin() + rank, keys.end());
    tau = from_order_key(keys[rank]);
  }
  if (tau_out) *tau_out = tau;
  int64_t na = 0;
  for (int64_t g = 0; g < N; ++g) {
    bool keep = true;
    if (use_lod) {
      const float dx = means[g] - campos[0];
      const float dy = means[N + g] - campos[1];
      const float dz = means[2 * N + g] - campos[2];
      const float s2 = ((dx * dx) + (dy * dy)) + (dz * dz);
      keep = keep && (s2 <= dd);
    }
    if (use_imp) keep = keep && (importance[g] >= tau);
    mask[g] = keep ? 1 : 0;
    if (keep) active_idx[na++] = (int32_t)g;
  }
  *n_active = na;
  return 0;
}

// ---- preprocess (fp32 spec)
OR_API int or_preprocess(const float* means, const float* log_scales, const float* quats,
                         const float* logits, const float* sh, int sh_degree, int64_t N,
                         const int32_t* active_idx, int64_t n_active, const float* camv,
                         int width, int height, float* xyzo, float* conic, float* rgb,
                         int32_t* radius, uint16_t* rect, int32_t* tiles) {
  if (sh_degree < 0 || sh_degree > 3 || N < 0 || n_active < 0 || n_active > N) return 1;
  const int K = (sh_degree + 1) * (sh_degree + 1);
  const Cam cam = make_cam(camv, width, height);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < N; ++i) {
    Proj<float> p;
    std::memset(&p, 0, sizeof(p));
    if (i < n_active) {
      const int64_t g = active_idx ? active_idx[i] : i;
      float mu[3], l[3], qq[4], lg, coef[48];
      gather<float, float>(means, log_scales, quats, logits, sh, K, N, g, mu, l, qq, lg, coef);
      project_one<float>(cam, mu, l, qq, lg, coef, K, p, nullptr);
    }
    float* X = xyzo + 4 * i;
    float* Cn = conic + 4 * i;
    float* Cl = rgb + 4 * i;
    if (p.visible) {
      X[0] = p.px; X[1] = p.py; X[2] = p.depth; X[3] = p.opacity;
      Cn[0] = p.A; Cn[1] = p.B; Cn[2] = p.C; Cn[3] = 0.0f;
      Cl[0] = p.rgb[0]; Cl[1] = p.rgb[1]; Cl[2] = p.rgb[2]; Cl[3] = 0.0f;
      radius[i] = p.radius;
      for (int k = 0; k < 4; ++k) rect[4 * i + k] = (uint16_t)p.rect[k];
      tiles[i] = p.tiles;
    } else {
      for (int k = 0; k < 4; ++k) { X[k] = 0.0f; Cn[k] = 0.0f; Cl[k] = 0.0f; rect[4 * i + k] = 0; }
      radius[i] = 0;
      tiles[i] = 0;
    }
  }
  return 0;
}

// ---- scan, key emission, stable sort, tile ranges
OR_API int or_bin_sort(const float* xyzo, const uint16_t* rect, const int32_t* tiles, int64_t n,
                       int width, int height, int32_t* offsets, uint64_t* keys, uint32_t* vals,
                       int64_t capacity, uint32_t* ranges, int64_t* n_instances) {
  const int TW = (width + 15) / 16;
  const int64_t TT = tile_count(width, height);
  int64_t total = 0;
  for (int64_t i = 0; i < n; ++i) {  // exclusive prefix sum
    offsets[i] = (int32_t)total;
    total += tiles[i];
  }
  *n_instances = total;
  if (total > capacity) return 2;
  std::vector<std::pair<uint64_t, uint32_t>> items((size_t)total);
  for (int64_t i = 0; i < n; ++i) {  // emission: Gaussian order, tiles row-major
    if (tiles[i] <= 0) continue;
    uint32_t dbits;
    std::memcpy(&dbits, &xyzo[4 * i + 2], 4);
    int64_t o = offsets[i];
    for (int ty = rect[4 * i + 1]; ty < rect[4 * i + 3]; ++ty)
      for (int tx = rect[4 * i + 0]; tx < rect[4 * i + 2]; ++tx) {
        const uint64_t tile = (uint64_t)ty * TW + tx;
        items[o++] = std::make_pair((tile << 32) | dbits, (uint32_t)i);
      }
  }
  std::stable_sort(items.begin(), items.end(),
                   [](const std::pair<uint64_t, uint32_t>& a, const std::pair<uint64_t, uint32_t>& b) {
                     return a.first < b.first;
                   });
  for (int64_t k = 0; k < total; ++k) {
    keys[k] = items[k].first;
    vals[k] = items[k].second;
  }
  for (int64_t t = 0; t < 2 * TT; ++t) ranges[t] = 0;
  for (int64_t k = 0; k < total; ++k) {
    const uint64_t tile = keys[k] >> 32;
    if (k == 0 || (keys[k - 1] >> 32) != tile) ranges[2 * tile] = (uint32_t)k;
    if (k == total - 1 || (keys[k + 1] >> 32) != tile) ranges[2 * tile + 1] = (uint32_t)(k + 1);
  }
  return 0;
}

// ---- raster forward (fp32 spec). tile_subset (optional) restricts the tiles.
OR_API int or_raster_fwd(const float* xyzo, const float* conic, const float* rgb,
                         const uint32_t* vals, const uint32_t* ranges, int width, int height,
                         const float* bg, float* image, float* final_T, int32_t* n_contrib,
                         int32_t* last, const int32_t* tile_subset, int64_t n_subset) {
  const int TW = (width + 15) / 16;
  const int64_t TT = tile_count(width, height);
  const int64_t nt = tile_subset ? n_subset : TT;
  const Rec32 r{xyzo, conic, rgb};
  const size_t P = (size_t)width * height;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t s = 0; s < nt; ++s) {
    const int64_t tile = tile_subset ? tile_subset[s] : s;
    const int tx = (int)(tile % TW), ty = (int)(tile / TW);
    const uint32_t start = ranges[2 * tile], end = ranges[2 * tile + 1];
    for (int v = ty * 16; v < std::min(height, ty * 16 + 16); ++v)
      for (int u = tx * 16; u < std::min(width, tx * 16 + 16); ++u) {
        float C[3] = {0.0f, 0.0f, 0.0f}, T;
        int n, lst;
        const float xc = (float)u + 0.5f, yc = (float)v + 0.5f;
        walk_pixel(r, vals, start, end, xc, yc, T, n, lst,
                   [&](uint32_t, uint32_t i, float alpha, bool, float) {
                     // T here is the transmittance before this blend.
                     const float wgt = alpha * T;
                     for (int ch = 0; ch < 3; ++ch) C[ch] = std::fmaf(wgt, rgb[4 * (size_t)i + ch], C[ch]);
                   });
        const size_t pix = (size_t)v * width + u;
        for (int ch = 0; ch < 3; ++ch) image[ch * P + pix] = std::fmaf(T, bg[ch], C[ch]);
        final_T[pix] = T;
        n_contrib[pix] = n;
        last[pix] = lst;
      }
  }
  return 0;
}

// ---- importance weights (BlitzGS write-up, section 2.2 "模型层级重要性评分传递":
// a cross-view visibility weight per Gaussian, its total contribution to the
// rendered views). Read as the sum over the view's pixels of the blend weight
// alpha T of each of its blends, with the fp32 spec values of the forward walk;
// accumulated (+=) in double into importance[gaussian], where the Gaussian of
// record i is active_idx[i] (or i when active_idx is null). Calling it once per
// view sums over views.
OR_API int or_importance(const float* xyzo, const float* conic, const float* rgb, const uint32_t* vals,
                         const uint32_t* ranges, int width, int height, const int32_t* active_idx,
                         double* importance) {
  const int TW = (width + 15) / 16;
  const int64_t TT = tile_count(width, height);
  const Rec32 r{xyzo, conic, rgb};
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t tile = 0; tile < TT; ++tile) {
    const int tx = (int)(tile % TW), ty = (int)(tile / TW);
    const uint32_t start = ranges[2 * tile], end = ranges[2 * tile + 1];
    for (int v = ty * 16; v < std::min(height, ty * 16 + 16); ++v)
      for (int u = tx * 16; u < std::min(width, tx * 16 + 16); ++u) {
        float T;
        int n, lst;
        walk_pixel(r, vals, start, end, (float)u + 0.5f, (float)v + 0.5f, T, n, lst,
                   [&](uint32_t, uint32_t i, float alpha, bool, float) {
                     const float wgt = alpha * T;  // T before this blend
                     const int64_t g = active_idx ? active_idx[i] : (int64_t)i;
#pragma omp atomic
                     importance[g] += (double)wgt;
                   });
      }
  }
  return 0;
}

// ---- brute force forward: no tile lists. Per pixel, every visible Gaussian
// whose rect contains the pixel's tile, in ascending (depth, index) order.
OR_API int or_raster_fwd_bruteforce(const float* xyzo, const float* conic, const float* rgb,
                                    const uint16_t* rect, const int32_t* tiles, int64_t n,
                                    int width, int height, const float* bg, float* image,
                                    float* final_T, int32_t* n_contrib, int32_t* last) {
  std::vector<uint32_t> order;
  for (int64_t i = 0; i < n; ++i)
    if (tiles[i] > 0) order.push_back((uint32_t)i);
  std::sort(order.begin(), order.end(), [&](uint32_t a, uint32_t b) {
    const float da = xyzo[4 * (size_t)a + 2], db = xyzo[4 * (size_t)b + 2];
    return da < db || (da == db && a < b);
  });
  const Rec32 r{xyzo, conic, rgb};
  const size_t P = (size_t)width * height;
  std::vector<uint32_t> list;
  for (int v = 0; v < height; ++v)
    for (int u = 0; u < width; ++u) {
      const int tx = u / 16, ty = v / 16;
      list.clear();
      for (uint32_t i : order)
        if (rect[4 * i] <= tx && tx < rect[4 * i + 2] && rect[4 * i + 1] <= ty && ty < rect[4 * i + 3])
          list.push_back(i);
      std::vector<uint32_t> idx(list.size());
      for (size_t k = 0; k < list.size(); ++k) idx[k] = list[k];
      float C[3] = {0.0f, 0.0f, 0.0f}, T;
      int nc, lst;
      walk_pixel(r, idx.data(), 0, (uint32_t)idx.size(), (float)u + 0.5f, (float)v + 0.5f, T, nc, lst,
                 [&](uint32_t, uint32_t i, float alpha, bool, float) {
                   const float wgt = alpha * T;
                   for (int ch = 0; ch < 3; ++ch) C[ch] = std::fmaf(wgt, rgb[4 * (size_t)i + ch], C[ch]);
                 });
      const size_t pix = (size_t)v * width + u;
      for (int ch = 0; ch < 3; ++ch) image[ch * P + pix] = std::fmaf(T, bg[ch], C[ch]);
      final_T[pix] = T;
      n_contrib[pix] = nc;
      last[pix] = lst;
    }
  return 0;
}

// ================================================== fp64 frozen-decision path

namespace {

// Per-active-Gaussian 2-D quantities in fp64, with the colour-clamp decisions
// of the fp32 records imposed.
struct P64 {
  double px, py, A, B, C, o, rgb[3];
  bool visible;
};

void project_all_f64(const double* means, const double* ls, const double* quats, const double* logits,
                     const double* sh, int K, int64_t N, const int32_t* active_idx, int64_t n_active,
                     const Cam& cam, const float* rgb32, const int32_t* tiles32, std::vector<P64>& out) {
  out.assign((size_t)n_active, P64());
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n_active; ++i) {
    P64& o = out[(size_t)i];
    o.visible = false;
    if (tiles32[i] <= 0) continue;
    const int64_t g = active_idx ? active_idx[i] : i;
    double mu[3], l[3], qq[4], lg, coef[48];
    gather<double, double>(means, ls, quats, logits, sh, K, N, g, mu, l, qq, lg, coef);
    bool cl[3];
    for (int ch = 0; ch < 3; ++ch) cl[ch] = !(rgb32[4 * i + ch] > 0.0f);
    Proj<double> p;
    project_one<double>(cam, mu, l, qq, lg, coef, K, p, cl);
    o.px = p.px; o.py = p.py; o.A = p.A; o.B = p.B; o.C = p.C; o.o = p.opacity;
    for (int ch = 0; ch < 3; ++ch) o.rgb[ch] = p.rgb[ch];
    o.visible = p.visible;
  }
}

struct Blend {
  uint32_t i;
  bool clamped;
  float alpha, e;  // fp32 values of the forward
};

// Gradient-flow number types for the preprocess backward: plain values, or
// magnitudes (every term replaced by its absolute value), which bound the
// rounding sensitivity of the same sums.
struct Mag {
  double v;
  Mag() : v(0) {}
  explicit Mag(double x) : v(std::fabs(x)) {}
};
inline Mag operator+(Mag a, Mag b) { Mag r; r.v = a.v + b.v; return r; }
inline Mag operator-(Mag a, Mag b) { Mag r; r.v = a.v + b.v; return r; }
inline Mag operator-(Mag a) { return a; }
inline Mag operator*(Mag a, double d) { Mag r; r.v = a.v * std::fabs(d); return r; }
inline Mag operator*(double d, Mag a) { return a * d; }
inline Mag& operator+=(Mag& a, Mag b) { a.v += b.v; return a; }
inline double val(double x) { return x; }
inline double val(Mag x) { return x.v; }
template <class G> G gz();
template <> double gz<double>() { return 0.0; }
template <> Mag gz<Mag>() { return Mag(); }
template <class G> G from2d(double x);
template <> double from2d<double>(double x) { return x; }
template <> Mag from2d<Mag>(double x) { return Mag(x); }

// Backward of the projection for one Gaussian: 2-D gradients (g2: px, py, A, B,
// C, opacity, r, g, b) -> parameter gradients. Forward quantities in fp64.
template <class G>
void preprocess_bwd_one(const Cam& cam, const double mu[3], const double ls[3], const double q[4],
                        double logit, const double* coef, int K, const bool clamped[3],
                        const G g2[9], G g_mu[3], G g_ls[3], G g_q[4], G& g_logit, G* g_sh) {
  const double* W = nullptr;
  double Wd[9];
  for (int k = 0; k < 9; ++k) Wd[k] = cam.W[k];
  W = Wd;
  double t[3];
  for (int r = 0; r < 3; ++r) t[r] = W[3 * r] * mu[0] + W[3 * r + 1] * mu[1] + W[3 * r + 2] * mu[2] + cam.t[r];
  const double s[3] = {std::exp(ls[0]), std::exp(ls[1]), std::exp(ls[2])};
  const double nq = std::sqrt(q[0] * q[0] + q[1] * q[1] + q[2] * q[2] + q[3] * q[3]);
  const double w = q[0] / nq, x = q[1] / nq, y = q[2] / nq, z = q[3] / nq;
  double Rq[9] = {1 - 2 * (y * y + z * z), 2 * (x * y - w * z), 2 * (x * z + w * y),
                  2 * (x * y + w * z), 1 - 2 * (x * x + z * z), 2 * (y * z - w * x),
                  2 * (x * z - w * y), 2 * (y * z + w * x), 1 - 2 * (x * x + y * y)};
  double M[9], S[9];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) M[3 * i + j] = Rq[3 * i + j] * s[j];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j)
      S[3 * i + j] = M[3 * i] * M[3 * j] + M[3 * i + 1] * M[3 * j + 1] + M[3 * i + 2] * M[3 * j + 2];
  const double fx = cam.fx, fy = cam.fy, tz = t[2], tz2 = tz * tz, tz3 = tz2 * tz;
  const double J00 = fx / tz, J11 = fy / tz, J02 = -fx * t[0] / tz2, J12 = -fy * t[1] / tz2;
  double T[6];
  for (int j = 0; j < 3; ++j) {
    T[j] = J00 * W[j] + J02 * W[6 + j];
    T[3 + j] = J11 * W[3 + j] + J12 * W[6 + j];
  }
  double TS[6];  // T Sigma
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < 3; ++j)
      TS[3 * i + j] = T[3 * i] * S[j] + T[3 * i + 1] * S[3 + j] + T[3 * i + 2] * S[6 + j];
  const double a = TS[0] * T[0] + TS[1] * T[1] + TS[2] * T[2] + 0.3;
  const double b = TS[0] * T[3] + TS[1] * T[4] + TS[2] * T[5];
  const double c = TS[3] * T[3] + TS[4] * T[4] + TS[5] * T[5] + 0.3;
  const double det = a * c - b * b, id2 = 1.0 / (det * det);
  const double op = 1.0 / (1.0 + std::exp(-logit));

  const G gpx = g2[0], gpy = g2[1], gA = g2[2], gB = g2[3], gC = g2[4], go = g2[5];
  // opacity
  g_logit = go * (op * (1.0 - op));
  // colour
  const double dv[3] = {mu[0] - cam.campos[0], mu[1] - cam.campos[1], mu[2] - cam.campos[2]};
  const double nd = std::sqrt(dv[0] * dv[0] + dv[1] * dv[1] + dv[2] * dv[2]);
  const double dir[3] = {dv[0] / nd, dv[1] / nd, dv[2] / nd};
  double Y[16], DY[16][3];
  if (std::is_same<G, Mag>::value) {
    sh_basis_abs(dir[0], dir[1], dir[2], K, Y);
    sh_basis_grad_abs(dir[0], dir[1], dir[2], K, DY);
  } else {
    sh_basis<double>(dir[0], dir[1], dir[2], K, Y);
    sh_basis_grad(dir[0], dir[1], dir[2], K, DY);
  }
  G gv[3];
  for (int ch = 0; ch < 3; ++ch) gv[ch] = clamped[ch] ? gz<G>() : g2[6 + ch];
  G gdir[3] = {gz<G>(), gz<G>(), gz<G>()};
  for (int k = 0; k < K; ++k) {
    G gY = gz<G>();
    for (int ch = 0; ch < 3; ++ch) {
      g_sh[3 * k + ch] = gv[ch] * Y[k];
      gY += gv[ch] * coef[3 * k + ch];
    }
    for (int m = 0; m < 3; ++m) gdir[m] += gY * DY[k][m];
  }
  const G ddot = gdir[0] * dir[0] + gdir[1] * dir[1] + gdir[2] * dir[2];
  for (int m = 0; m < 3; ++m) g_mu[m] = (gdir[m] - ddot * dir[m]) * (1.0 / nd);
  // projected centre
  G gt[3];
  gt[0] = gpx * (fx / tz);
  gt[1] = gpy * (fy / tz);
  gt[2] = gpx * (-fx * t[0] / tz2) + gpy * (-fy * t[1] / tz2);
  // conic -> Sigma' (a, b, c)
  const G ga = (gA * (-c * c) + gB * (b * c) + gC * (-b * b)) * id2;
  const G gb = (gA * (2 * b * c) + gB * (-(a * c + b * b)) + gC * (2 * a * b)) * id2;
  const G gc = (gA * (-b * b) + gB * (a * b) + gC * (-a * a)) * id2;
  // Sigma' = T Sigma T^T, gradient matrix Gm = [[ga, gb/2], [gb/2, gc]]
  const G Gm[4] = {ga, gb * 0.5, gb * 0.5, gc};
  // gSigma = T^T Gm T (3x3)
  G GT[6];  // Gm T (2x3)
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < 3; ++j) GT[3 * i + j] = Gm[2 * i] * T[j] + Gm[2 * i + 1] * T[3 + j];
  G gS[9];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) gS[3 * i + j] = GT[j] * T[i] + GT[3 + j] * T[3 + i];
  // gT = 2 Gm T Sigma = 2 Gm (T Sigma)
  G gT[6];
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < 3; ++j) gT[3 * i + j] = (Gm[2 * i] * TS[j] + Gm[2 * i + 1] * TS[3 + j]) * 2.0;
  // gM = 2 gSigma M
  G gM[9];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j)
      gM[3 * i + j] = (gS[3 * i] * M[j] + gS[3 * i + 1] * M[3 + j] + gS[3 * i + 2] * M[6 + j]) * 2.0;
  // M = Rq diag(s)
  G gR[9];
  for (int j = 0; j < 3; ++j) {
    G gs = gz<G>();
    for (int i = 0; i < 3; ++i) {
      gs += gM[3 * i + j] * Rq[3 * i + j];
      gR[3 * i + j] = gM[3 * i + j] * s[j];
    }
    g_ls[j] = gs * s[j];
  }
  // rotation matrix -> normalised quaternion
  G gw = (gR[1] * (-z) + gR[2] * y + gR[3] * z + gR[5] * (-x) + gR[6] * (-y) + gR[7] * x) * 2.0;
  G gx = (gR[1] * y + gR[2] * z + gR[3] * y + gR[4] * (-2 * x) + gR[5] * (-w) + gR[6] * z + gR[7] * w +
          gR[8] * (-2 * x)) * 2.0;
  G gy = (gR[0] * (-2 * y) + gR[1] * x + gR[2] * w + gR[3] * x + gR[5] * z + gR[6] * (-w) + gR[7] * z +
          gR[8] * (-2 * y)) * 2.0;
  G gzq = (gR[0] * (-2 * z) + gR[1] * (-w) + gR[2] * x + gR[3] * w + gR[4] * (-2 * z) + gR[5] * y +
           gR[6] * x + gR[7] * y) * 2.0;
  const double qn[4] = {w, x, y, z};
  const G gqn[4] = {gw, gx, gy, gzq};
  const G qdot = gqn[0] * qn[0] + gqn[1] * qn[1] + gqn[2] * qn[2] + gqn[3] * qn[3];
  for (int m = 0; m < 4; ++m) g_q[m] = (gqn[m] - qdot * qn[m]) * (1.0 / nq);
  // T = J W -> J -> t
  G gJ00 = gz<G>(), gJ02 = gz<G>(), gJ11 = gz<G>(), gJ12 = gz<G>();
  for (int j = 0; j < 3; ++j) {
    gJ00 += gT[j] * W[j];
    gJ02 += gT[j] * W[6 + j];
    gJ11 += gT[3 + j] * W[3 + j];
    gJ12 += gT[3 + j] * W[6 + j];
  }
  gt[0] += gJ02 * (-fx / tz2);
  gt[1] += gJ12 * (-fy / tz2);
  gt[2] += gJ00 * (-fx / tz2) + gJ11 * (-fy / tz2) + gJ02 * (2 * fx * t[0] / tz3) +
           gJ12 * (2 * fy * t[1] / tz3);
  // t = W mu + t0
  for (int m = 0; m < 3; ++m) g_mu[m] += gt[0] * W[m] + gt[1] * W[3 + m] + gt[2] * W[6 + m];
}

}  // namespace

// Loss sum(dL_dimage * image) of the fp64 forward with every decision of the
// fp32 records held fixed. Parameters in fp64 (perturbed copies for finite
// differences); the fp32 records, lists and ranges come from the unperturbed
// fp32 spec run.
OR_API double or_loss_frozen_f64(const double* means, const double* log_scales, const double* quats,
                                 const double* logits, const double* sh, int sh_degree, int64_t N,
                                 const int32_t* active_idx, int64_t n_active, const float* camv,
                                 int width, int height, const float* xyzo32, const float* conic32,
                                 const float* rgb32, const int32_t* tiles32, const uint32_t* vals,
                                 const uint32_t* ranges, const float* bg, const float* dL_dimage,
                                 double* image_out) {
  const int K = (sh_degree + 1) * (sh_degree + 1);
  const Cam cam = make_cam(camv, width, height);
  std::vector<P64> P;
  project_all_f64(means, log_scales, quats, logits, sh, K, N, active_idx, n_active, cam, rgb32, tiles32, P);
  const Rec32 r{xyzo32, conic32, rgb32};
  const int TW = cam.TW;
  const int64_t TT = tile_count(width, height);
  const size_t NP = (size_t)width * height;
  double loss = 0.0;
#pragma omp parallel for schedule(dynamic, 4) reduction(+ : loss)
  for (int64_t tile = 0; tile < TT; ++tile) {
    const int tx = (int)(tile % TW), ty = (int)(tile / TW);
    const uint32_t start = ranges[2 * tile], end = ranges[2 * tile + 1];
    for (int v = ty * 16; v < std::min(height, ty * 16 + 16); ++v)
      for (int u = tx * 16; u < std::min(width, tx * 16 + 16); ++u) {
        const double xc = u + 0.5, yc = v + 0.5;
        double C[3] = {0, 0, 0}, T64 = 1.0;
        float T32;
        int n, lst;
        walk_pixel(r, vals, start, end, (float)xc, (float)yc, T32, n, lst,
                   [&](uint32_t, uint32_t i, float, bool clamped, float) {
                     const P64& g = P[i];
                     const double dx = g.px - xc, dy = g.py - yc;
                     const double p = -0.5 * (g.A * dx * dx + g.C * dy * dy) - g.B * dx * dy;
                     const double al = clamped ? 0.99 : g.o * std::exp(p);
                     for (int ch = 0; ch < 3; ++ch) C[ch] += al * T64 * g.rgb[ch];
                     T64 *= (1.0 - al);
                   });
        const size_t pix = (size_t)v * width + u;
        for (int ch = 0; ch < 3; ++ch) {
          const double out = C[ch] + T64 * bg[ch];
          if (image_out) image_out[ch * NP + pix] = out;
          loss += (double)dL_dimage[ch * NP + pix] * out;
        }
      }
  }
  return loss;
}

// Backward in fp64 with the fp32 decisions. Outputs (any may be null):
//   g2d / s2d [n_active x 9]: 2-D gradients (px, py, A, B, C, opacity, r, g, b)
//     and the sums of absolute per-pixel contributions;
//   d_* / m_*: parameter gradients in the input SoA layout (zero for Gaussians
//     that are not active or not visible) and their magnitude bounds.
OR_API int or_backward_f64(const float* means, const float* log_scales, const float* quats,
                           const float* logits, const float* sh, int sh_degree, int64_t N,
                           const int32_t* active_idx, int64_t n_active, const float* camv, int width,
                           int height, const float* xyzo32, const float* conic32, const float* rgb32,
                           const int32_t* tiles32, const uint32_t* vals, const uint32_t* ranges,
                           const float* bg, const float* dL_dimage, double* g2d, double* s2d,
                           double* d_means, double* d_log_scales, double* d_quats, double* d_logits,
                           double* d_sh, double* m_means, double* m_log_scales, double* m_quats,
                           double* m_logits, double* m_sh, const int32_t* tile_subset,
                           int64_t n_subset, int records2d) {
  const int K = (sh_degree + 1) * (sh_degree + 1);
  const Cam cam = make_cam(camv, width, height);
  // fp64 copies of the parameters
  std::vector<double> mu64(3 * (size_t)N), ls64(3 * (size_t)N), q64(4 * (size_t)N), lg64((size_t)N),
      sh64((size_t)3 * K * N);
  for (size_t k = 0; k < mu64.size(); ++k) mu64[k] = means[k];
  for (size_t k = 0; k < ls64.size(); ++k) ls64[k] = log_scales[k];
  for (size_t k = 0; k < q64.size(); ++k) q64[k] = quats[k];
  for (size_t k = 0; k < lg64.size(); ++k) lg64[k] = logits[k];
  for (size_t k = 0; k < sh64.size(); ++k) sh64[k] = sh[k];
  std::vector<P64> P;
  project_all_f64(mu64.data(), ls64.data(), q64.data(), lg64.data(), sh64.data(), K, N, active_idx,
                  n_active, cam, rgb32, tiles32, P);
  if (records2d) {
    // The raster stage's backward takes the records as its inputs: differentiate
    // the compositing at the fp32 record values the forward used.
    for (int64_t i = 0; i < n_active; ++i) {
      P64& o = P[(size_t)i];
      if (!o.visible) continue;
      o.px = xyzo32[4 * i]; o.py = xyzo32[4 * i + 1]; o.o = xyzo32[4 * i + 3];
      o.A = conic32[4 * i]; o.B = conic32[4 * i + 1]; o.C = conic32[4 * i + 2];
      for (int ch = 0; ch < 3; ++ch) o.rgb[ch] = rgb32[4 * i + ch];
    }
  }
  std::vector<double> G2((size_t)n_active * 9, 0.0), S2((size_t)n_active * 9, 0.0);
  const Rec32 r{xyzo32, conic32, rgb32};
  const int TW = cam.TW;
  const int64_t TT = tile_count(width, height);
  const size_t NP = (size_t)width * height;
  const int64_t nt = tile_subset ? n_subset : TT;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t s = 0; s < nt; ++s) {
    const int64_t tile = tile_subset ? tile_subset[s] : s;
    const int tx = (int)(tile % TW), ty = (int)(tile / TW);
    const uint32_t start = ranges[2 * tile], end = ranges[2 * tile + 1];
    std::vector<Blend> bl;
    for (int v = ty * 16; v < std::min(height, ty * 16 + 16); ++v)
      for (int u = tx * 16; u < std::min(width, tx * 16 + 16); ++u) {
        const double xc = u + 0.5, yc = v + 0.5;
        bl.clear();
        float T32;
        int n, lst;
        walk_pixel(r, vals, start, end, (float)xc, (float)yc, T32, n, lst,
                   [&](uint32_t, uint32_t i, float alpha, bool clamped, float e) {
                     bl.push_back(Blend{i, clamped, alpha, e});
                   });
        const size_t pix = (size_t)v * width + u;
        const double gp[3] = {dL_dimage[pix], dL_dimage[NP + pix], dL_dimage[2 * NP + pix]};
        const size_t nb = bl.size();
        std::vector<double> al(nb), ex(nb), Tk(nb);
        double T = 1.0;
        for (size_t k = 0; k < nb; ++k) {
          const P64& g = P[bl[k].i];
          const double dx = g.px - xc, dy = g.py - yc;
          if (records2d) {
            // the forward's own alpha and exp values: the derivative of the
            // computation that produced the image
            ex[k] = bl[k].e;
            al[k] = bl[k].alpha;
          } else {
            const double p = -0.5 * (g.A * dx * dx + g.C * dy * dy) - g.B * dx * dy;
            ex[k] = std::exp(p);
            al[k] = bl[k].clamped ? 0.99 : g.o * ex[k];
          }
          Tk[k] = T;
          T *= (1.0 - al[k]);
        }
        double Rb[3] = {bg[0], bg[1], bg[2]};
        for (size_t kk = nb; kk-- > 0;) {
          const uint32_t i = bl[kk].i;
          const P64& g = P[i];
          // t9: the pair's terms; a9: the same terms with every operand replaced
          // by its magnitude (c - R becomes |c| + |R|), the scale of their
          // rounding error in a single-precision evaluation.
          double t9[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0}, a9[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
          double Gk = 0.0, Ga = 0.0;
          for (int ch = 0; ch < 3; ++ch) {
            t9[6 + ch] = gp[ch] * al[kk] * Tk[kk];
            a9[6 + ch] = std::fabs(t9[6 + ch]);
            Gk += gp[ch] * (g.rgb[ch] - Rb[ch]);
            Ga += std::fabs(gp[ch]) * (std::fabs(g.rgb[ch]) + std::fabs(Rb[ch]));
          }
          Gk *= Tk[kk];
          Ga *= Tk[kk];
          if (!bl[kk].clamped) {
            const double dx = g.px - xc, dy = g.py - yc;
            const double dp = Gk * al[kk], dpa = Ga * al[kk];
            t9[5] = Gk * ex[kk];
            t9[0] = dp * (-(g.A * dx + g.B * dy));
            t9[1] = dp * (-(g.B * dx + g.C * dy));
            t9[2] = dp * (-0.5 * dx * dx);
            t9[3] = dp * (-dx * dy);
            t9[4] = dp * (-0.5 * dy * dy);
            a9[5] = Ga * ex[kk];
            a9[0] = dpa * (std::fabs(g.A * dx) + std::fabs(g.B * dy));
            a9[1] = dpa * (std::fabs(g.B * dx) + std::fabs(g.C * dy));
            a9[2] = dpa * 0.5 * dx * dx;
            a9[3] = dpa * std::fabs(dx * dy);
            a9[4] = dpa * 0.5 * dy * dy;
          }
          for (int m = 0; m < 9; ++m) {
#pragma omp atomic
            G2[9 * (size_t)i + m] += t9[m];
#pragma omp atomic
            S2[9 * (size_t)i + m] += a9[m];
          }
          for (int ch = 0; ch < 3; ++ch) Rb[ch] = g.rgb[ch] * al[kk] + (1.0 - al[kk]) * Rb[ch];
        }
      }
  }
  if (g2d) std::memcpy(g2d, G2.data(), G2.size() * sizeof(double));
  if (s2d) std::memcpy(s2d, S2.data(), S2.size() * sizeof(double));
  const bool want_d = d_means != nullptr, want_m = m_means != nullptr;
  if (!want_d && !want_m) return 0;
  if (want_d) {
    std::fill(d_means, d_means + 3 * N, 0.0);
    std::fill(d_log_scales, d_log_scales + 3 * N, 0.0);
    std::fill(d_quats, d_quats + 4 * N, 0.0);
    std::fill(d_logits, d_logits + N, 0.0);
    std::fill(d_sh, d_sh + (size_t)3 * K * N, 0.0);
  }
  if (want_m) {
    std::fill(m_means, m_means + 3 * N, 0.0);
    std::fill(m_log_scales, m_log_scales + 3 * N, 0.0);
    std::fill(m_quats, m_quats + 4 * N, 0.0);
    std::fill(m_logits, m_logits + N, 0.0);
    std::fill(m_sh, m_sh + (size_t)3 * K * N, 0.0);
  }
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n_active; ++i) {
    if (!P[(size_t)i].visible) continue;
    const int64_t g = active_idx ? active_idx[i] : i;
    double mu[3], l[3], qq[4], lg, coef[48];
    gather<double, double>(mu64.data(), ls64.data(), q64.data(), lg64.data(), sh64.data(), K, N, g, mu,
                           l, qq, lg, coef);
    bool cl[3];
    for (int ch = 0; ch < 3; ++ch) cl[ch] = !(rgb32[4 * i + ch] > 0.0f);
    if (want_d) {
      double gm[3], gl[3], gq[4], glg, gs[48];
      preprocess_bwd_one<double>(cam, mu, l, qq, lg, coef, K, cl, &G2[9 * (size_t)i], gm, gl, gq, glg, gs);
      for (int m = 0; m < 3; ++m) d_means[m * N + g] = gm[m];
      for (int m = 0; m < 3; ++m) d_log_scales[m * N + g] = gl[m];
      for (int m = 0; m < 4; ++m) d_quats[m * N + g] = gq[m];
      d_logits[g] = glg;
      for (int k = 0; k < 3 * K; ++k) d_sh[(size_t)k * N + g] = gs[k];
    }
    if (want_m) {
      Mag s9[9], gm[3], gl[3], gq[4], glg, gs[48];
      for (int m = 0; m < 9; ++m) s9[m] = Mag(S2[9 * (size_t)i + m]);
      preprocess_bwd_one<Mag>(cam, mu, l, qq, lg, coef, K, cl, s9, gm, gl, gq, glg, gs);
      for (int m = 0; m < 3; ++m) m_means[m * N + g] = gm[m].v;
      for (int m = 0; m < 3; ++m) m_log_scales[m * N + g] = gl[m].v;
      for (int m = 0; m < 4; ++m) m_quats[m * N + g] = gq[m].v;
      m_logits[g] = glg.v;
      for (int k = 0; k < 3 * K; ++k) m_sh[(size_t)k * N + g] = gs[k].v;
    }
  }
  return 0;
}

// Preprocess backward alone: given 2-D gradients g2 [n_active x 9] (fp64),
// produce parameter gradients and magnitude bounds (magnitudes from |g2|).
OR_API int or_preprocess_bwd_f64(const float* means, const float* log_scales, const float* quats,
                                 const float* logits, const float* sh, int sh_degree, int64_t N,
                                 const int32_t* active_idx, int64_t n_active, const float* camv,
                                 int width, int height, const float* rgb32, const int32_t* tiles32,
                                 const double* g2, double* d_means, double* d_log_scales,
                                 double* d_quats, double* d_logits, double* d_sh, double* m_means,
                                 double* m_log_scales, double* m_quats, double* m_logits, double* m_sh) {
  const int K = (sh_degree + 1) * (sh_degree + 1);
  const Cam cam = make_cam(camv, width, height);
  std::fill(d_means, d_means + 3 * N, 0.0);
  std::fill(d_log_scales, d_log_scales + 3 * N, 0.0);
  std::fill(d_quats, d_quats + 4 * N, 0.0);
  std::fill(d_logits, d_logits + N, 0.0);
  std::fill(d_sh, d_sh + (size_t)3 * K * N, 0.0);
  std::fill(m_means, m_means + 3 * N, 0.0);
  std::fill(m_log_scales, m_log_scales + 3 * N, 0.0);
  std::fill(m_quats, m_quats + 4 * N, 0.0);
  std::fill(m_logits, m_logits + N, 0.0);
  std::fill(m_sh, m_sh + (size_t)3 * K * N, 0.0);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n_active; ++i) {
    if (tiles32[i] <= 0) continue;
    const int64_t g = active_idx ? active_idx[i] : i;
    double mu[3], l[3], qq[4], lg, coef[48];
    gather<double, float>(means, log_scales, quats, logits, sh, K, N, g, mu, l, qq, lg, coef);
    bool cl[3];
    for (int ch = 0; ch < 3; ++ch) cl[ch] = !(rgb32[4 * i + ch] > 0.0f);
    double gm[3], gl[3], gq[4], glg, gs[48];
    preprocess_bwd_one<double>(cam, mu, l, qq, lg, coef, K, cl, &g2[9 * (size_t)i], gm, gl, gq, glg, gs);
    Mag s9[9], mm[3], ml[3], mq[4], mlg, ms[48];
    for (int m = 0; m < 9; ++m) s9[m] = Mag(g2[9 * (size_t)i + m]);
    preprocess_bwd_one<Mag>(cam, mu, l, qq, lg, coef, K, cl, s9, mm, ml, mq, mlg, ms);
    for (int m = 0; m < 3; ++m) { d_means[m * N + g] = gm[m]; m_means[m * N + g] = mm[m].v; }
    for (int m = 0; m < 3; ++m) { d_log_scales[m * N + g] = gl[m]; m_log_scales[m * N + g] = ml[m].v; }
    for (int m = 0; m < 4; ++m) { d_quats[m * N + g] = gq[m]; m_quats[m * N + g] = mq[m].v; }
    d_logits[g] = glg;
    m_logits[g] = mlg.v;
    for (int k = 0; k < 3 * K; ++k) { d_sh[(size_t)k * N + g] = gs[k]; m_sh[(size_t)k * N + g] = ms[k].v; }
  }
  return 0;
}

// fp64 projection of every active Gaussian (for closed-form pins):
// out [n_active x 10] = px, py, depth, opacity, A, B, C, r, g, b; vis [n_active].
OR_API int or_project_f64(const double* means, const double* log_scales, const double* quats,
                          const double* logits, const double* sh, int sh_degree, int64_t N,
                          const float* camv, int width, int height, double* out, int32_t* vis,
                          int32_t* radius) {
  const int K = (sh_degree + 1) * (sh_degree + 1);
  const Cam cam = make_cam(camv, width, height);
  for (int64_t g = 0; g < N; ++g) {
    double mu[3], l[3], qq[4], lg, coef[48];
    gather<double, double>(means, log_scales, quats, logits, sh, K, N, g, mu, l, qq, lg, coef);
    Proj<double> p;
    project_one<double>(cam, mu, l, qq, lg, coef, K, p, nullptr);
    double* o = out + 10 * g;
    o[0] = p.px; o[1] = p.py; o[2] = p.depth; o[3] = p.opacity;
    o[4] = p.A; o[5] = p.B; o[6] = p.C;
    o[7] = p.rgb[0]; o[8] = p.rgb[1]; o[9] = p.rgb[2];
    vis[g] = p.visible ? 1 : 0;
    radius[g] = p.radius;
  }
  return 0;
}

// ===================================================== quantised SH Adam
// The fused optimizer step over block-quantised SH coefficients and Adam
// moments (Spirula Studio page, sections "先算一笔账", "一个开关" and
// "为什么 8-bit 量化 Adam 状态居然不掉精度"): the view-dependent SH units are
// stored as 16-bit linear block codes, each moment as an 8-bit linear block
// code of its logarithm, every 256 consecutive units of a plane sharing one
// (min, max) pair; gradients stay fp32. Readings fixed here (the page prints
// no formula beyond the log transform and the decode):
//   block      256 consecutive Gaussians of one unit plane (the transposed
//              layout); codes have row stride Npad = N rounded up to 256,
//              bounds are [U][N/256 rounded up][2] = (lo, hi)
//   code       per block step = (hi - lo) / Q and inv = Q / (hi - lo)
//              (0 when hi == lo, and then every code is 0), Q = 2^bits - 1;
//              q = rint((x - lo) * inv) clamped to [0, Q]; decode
//              lo + step * q (the page: one multiplication per unit); fp32,
//              no fused multiply-add
//   moments    first moment m: y = sign(m) log1p(|m| r); second moment v:
//              y = log1p(sqrt(v) r); e is the code scale (an input), r its
//              reciprocal rounded from double; decode e expm1(|y|) (signed)
//   log1p      ln 2 * log2(1 + z), log2 by the atanh series below; expm1 as
//              exp2(y log2 e) - 1 with the software exp2 of the raster
//   Adam       m' = b1 m + (1 - b1) g, v' = b2 v + (1 - b2) g^2,
//              p' = p - lr (m' c1) / (sqrt(v' c2) + eps), c1, c2 the bias
//              corrections of the step (inputs, like b1, 1 - b1, b2, 1 - b2)
//   bounds     of the new fp32 values of each block, every step.

namespace {

struct QuantConst {
  float l2c[6];  // RN(2 / ((2k + 1) ln 2)), k = 0..5
  float ln2, sqrt2;
  QuantConst() {
    const double ln2d = std::log(2.0);
    for (int k = 0; k < 6; ++k) l2c[k] = (float)(2.0 / ((2.0 * k + 1.0) * ln2d));
    ln2 = (float)ln2d;
    sqrt2 = (float)std::sqrt(2.0);
  }
};
const QuantConst QC;

}  // namespace

// log2 of y >= 1: y = m 2^e with m in (sqrt(1/2), sqrt(2)] (exact),
// s = (m - 1) / (m + 1), log2(m) = 2 atanh(s) / ln 2 as a Horner polynomial
// in s^2 with the coefficients above; log2(+inf) = +inf.
float log2_spec(float y) {
  if (!(y <= std::numeric_limits<float>::max())) return y;  // +inf (and NaN) pass through
  int e;
  float m = std::frexp(y, &e);  // y = m 2^e, m in [1/2, 1)
  m = m * 2.0f;
  e -= 1;                       // m in [1, 2)
  if (m > QC.sqrt2) {
    m = m * 0.5f;
    e += 1;
  }
  const float s = (m - 1.0f) / (m + 1.0f);
  const float s2 = s * s;
  float p = QC.l2c[5];
  for (int k = 4; k >= 0; --k) p = std::fmaf(p, s2, QC.l2c[k]);
  return (float)e + s * p;
}
inline float log1p_spec(float z) { return QC.ln2 * log2_spec(1.0f + z); }
inline float expm1_spec(float y) { return exp2_spec(y * KC.l2e) - 1.0f; }

// A block's code: its lower bound, step and inverse step.
struct QBlock {
  float lo, step, inv;
};
inline QBlock q_block(float lo, float hi, float Q) {
  const float d = hi - lo;
  return d > 0.0f ? QBlock{lo, d / Q, Q / d} : QBlock{lo, 0.0f, 0.0f};
}
inline uint32_t q_encode(float x, const QBlock& b, float Q) {
  const float t = std::rint((x - b.lo) * b.inv);
  return t < 0.0f ? 0u : (t > Q ? (uint32_t)Q : (uint32_t)t);
}
inline float q_decode(uint32_t q, const QBlock& b) { return b.lo + b.step * (float)q; }

inline float m_to_log(float m, float r) { return m >= 0.0f ? log1p_spec(m * r) : -log1p_spec(-m * r); }
inline float m_from_log(float y, float e) { return y >= 0.0f ? e * expm1_spec(y) : -(e * expm1_spec(-y)); }
inline float v_to_log(float v, float r) { return log1p_spec(std::sqrt(v) * r); }
inline float v_from_log(float y, float e) {
  const float s = e * expm1_spec(y);
  return s * s;
}

OR_API float or_log2_spec(float y) { return log2_spec(y); }
OR_API float or_log1p_spec(float z) { return log1p_spec(z); }
OR_API float or_expm1_spec(float y) { return expm1_spec(y); }

// Block codes of fp32 planes x [U][N] (row stride N): codes [U][Npad] (16 or
// 8 bit, stored as uint32 here), bounds [U][nblk][2].
OR_API int or_quant_encode(const float* x, int64_t U, int64_t N, int bits, uint32_t* codes, float* bounds) {
  const int64_t nblk = (N + 255) / 256, Npad = nblk * 256;
  const float Q = (float)((1u << bits) - 1u);
  for (int64_t u = 0; u < U; ++u)
    for (int64_t b = 0; b < nblk; ++b) {
      const int64_t g0 = b * 256, g1 = std::min(N, g0 + 256);
      float lo = x[u * N + g0], hi = lo;
      for (int64_t g = g0; g < g1; ++g) {
        lo = std::min(lo, x[u * N + g]);
        hi = std::max(hi, x[u * N + g]);
      }
      const QBlock qb = q_block(lo, hi, Q);
      for (int64_t g = g0; g < g0 + 256; ++g)
        codes[u * Npad + g] = g < g1 ? q_encode(x[u * N + g], qb, Q) : 0u;
      bounds[2 * (u * nblk + b)] = lo;
      bounds[2 * (u * nblk + b) + 1] = hi;
    }
  return 0;
}

// Decoded fp32 planes of block codes (inverse layout of or_quant_encode).
OR_API int or_quant_decode(const uint32_t* codes, const float* bounds, int64_t U, int64_t N, int bits, float* x) {
  const int64_t nblk = (N + 255) / 256, Npad = nblk * 256;
  const float Q = (float)((1u << bits) - 1u);
  for (int64_t u = 0; u < U; ++u)
    for (int64_t g = 0; g < N; ++g) {
      const int64_t b = g / 256;
      const QBlock qb = q_block(bounds[2 * (u * nblk + b)], bounds[2 * (u * nblk + b) + 1], Q);
      x[u * N + g] = q_decode(codes[u * Npad + g], qb);
    }
  return 0;
}

// One Adam step (number `step`, from 1) over U planes of N units, in place:
// 16-bit value codes, 8-bit log codes of m and v, fp32 gradients grad [U][N]
// (row stride N). The fp32 constants of the step are the roundings of
// lr, beta1, 1 - beta1, beta2, 1 - beta2, 1 / (1 - beta1^step),
// 1 / (1 - beta2^step), eps and the code scale, each computed in double.
OR_API int or_adam_sh_quant(const float* grad, int64_t U, int64_t N, uint32_t* pc, float* pb, uint32_t* mc,
                            float* mb, uint32_t* vc, float* vb, double lr_d, double beta1, double beta2,
                            double eps_d, double scale_d, int64_t step) {
  const float lr = (float)lr_d, b1 = (float)beta1, ob1 = (float)(1.0 - beta1), b2 = (float)beta2,
              ob2 = (float)(1.0 - beta2), c1 = (float)(1.0 / (1.0 - std::pow(beta1, (double)step))),
              c2 = (float)(1.0 / (1.0 - std::pow(beta2, (double)step))), eps = (float)eps_d,
              ec = (float)scale_d, er = (float)(1.0 / scale_d);
  const int64_t nblk = (N + 255) / 256, Npad = nblk * 256;
  const float Q16 = 65535.0f, Q8 = 255.0f;
  std::vector<float> np(256), ny(256), vy(256);
  for (int64_t u = 0; u < U; ++u)
    for (int64_t b = 0; b < nblk; ++b) {
      const int64_t g0 = b * 256, g1 = std::min(N, g0 + 256), n = g1 - g0;
      float* B[3] = {pb + 2 * (u * nblk + b), mb + 2 * (u * nblk + b), vb + 2 * (u * nblk + b)};
      const QBlock qp = q_block(B[0][0], B[0][1], Q16), qm = q_block(B[1][0], B[1][1], Q8),
                   qv = q_block(B[2][0], B[2][1], Q8);
      for (int64_t k = 0; k < n; ++k) {
        const int64_t c = u * Npad + g0 + k;
        const float ph = q_decode(pc[c], qp);
        const float mh = m_from_log(q_decode(mc[c], qm), ec);
        const float vh = v_from_log(q_decode(vc[c], qv), ec);
        const float g = grad[u * N + g0 + k];
        const float m1 = b1 * mh + ob1 * g;
        const float v1 = b2 * vh + ob2 * (g * g);
        const float a = m1 * c1;
        const float den = std::sqrt(v1 * c2) + eps;
        np[k] = ph - lr * (a / den);
        ny[k] = m_to_log(m1, er);
        vy[k] = v_to_log(v1, er);
      }
      const std::vector<float>* vals[3] = {&np, &ny, &vy};
      uint32_t* codes[3] = {pc, mc, vc};
      const float Qs[3] = {Q16, Q8, Q8};
      for (int t = 0; t < 3; ++t) {
        const std::vector<float>& y = *vals[t];
        float lo = y[0], hi = y[0];
        for (int64_t k = 1; k < n; ++k) {
          lo = std::min(lo, y[k]);
          hi = std::max(hi, y[k]);
        }
        const QBlock qb = q_block(lo, hi, Qs[t]);
        for (int64_t k = 0; k < 256; ++k) codes[t][u * Npad + g0 + k] = k < n ? q_encode(y[k], qb, Qs[t]) : 0u;
        B[t][0] = lo;
        B[t][1] = hi;
      }
    }
  return 0;
}
