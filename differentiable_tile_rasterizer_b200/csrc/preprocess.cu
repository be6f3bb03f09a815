// Per-Gaussian projection (EWA splatting with SH colour) and its backward.
//
// One thread per active position. Parameters are structure-of-arrays planes,
// so each of the 11 + 3K plane reads of a warp is one coalesced 128-byte
// line when the active list is the identity (and monotone gathers otherwise).
// Records are written as 16-byte vectors. The stage is HBM-bound: 236 bytes
// in and 64 bytes out per Gaussian at SH degree 3 against ~300 fp32 ops.
//
// Forward arithmetic follows the fixed fp32 specification step by step (the
// step numbers match the CPU oracle's comments); the backward is plain fp32.

#include "checked.cuh"
#include "gs_device.cuh"
#include "gs_internal.cuh"

namespace gs {
namespace {

struct Proj {
  bool visible;
  float px, py, depth, opacity, A, B, C, rf;
  float rgb[3];
  int x0, y0, x1, y1;
};

__device__ __forceinline__ float clamp_grid(float v, float hi) {
  return v < 0.0f ? 0.0f : (v > hi ? hi : v);
}

// Where project() reads a Gaussian's parameters: straight from the SoA
// planes (single view: the SH planes are read only for Gaussians that get
// that far) or from registers loaded once (several views).
struct PlaneSource {
  const Params& p;
  int64_t g;
  __device__ __forceinline__ float mean(int r) const { return p.means[r * p.N + g]; }
  __device__ __forceinline__ float log_scale(int r) const { return p.log_scales[r * p.N + g]; }
  __device__ __forceinline__ float quat(int r) const { return p.quats[r * p.N + g]; }
  __device__ __forceinline__ float logit() const { return p.logits[g]; }
  __device__ __forceinline__ float sh(int plane) const { return p.sh[(int64_t)plane * p.N + g]; }
};
template <int K>
struct RegisterSource {
  float m[3], l[3], q[4], lg, c[3 * K];
  __device__ __forceinline__ void load(const Params& p, int64_t g) {
#pragma unroll
    for (int r = 0; r < 3; ++r) m[r] = p.means[r * p.N + g];
#pragma unroll
    for (int r = 0; r < 3; ++r) l[r] = p.log_scales[r * p.N + g];
#pragma unroll
    for (int r = 0; r < 4; ++r) q[r] = p.quats[r * p.N + g];
    lg = p.logits[g];
#pragma unroll
    for (int k = 0; k < 3 * K; ++k) c[k] = p.sh[(int64_t)k * p.N + g];
  }
  __device__ __forceinline__ float mean(int r) const { return m[r]; }
  __device__ __forceinline__ float log_scale(int r) const { return l[r]; }
  __device__ __forceinline__ float quat(int r) const { return q[r]; }
  __device__ __forceinline__ float logit() const { return lg; }
  __device__ __forceinline__ float sh(int plane) const { return c[plane]; }
};

template <int K, class Src>
__device__ __forceinline__ void project(const Src& src, const DevCam& cam, Proj& o) {
  o.visible = false;
  const float mx = src.mean(0), my = src.mean(1), mz = src.mean(2);
  const float l0 = src.log_scale(0), l1 = src.log_scale(1), l2 = src.log_scale(2);
  const float qw = src.quat(0), qx = src.quat(1), qy = src.quat(2), qz = src.quat(3);
  const float logit = src.logit();
  if (!(finitef(mx) && finitef(my) && finitef(mz) && finitef(l0) && finitef(l1) && finitef(l2) &&
        finitef(qw) && finitef(qx) && finitef(qy) && finitef(qz) && finitef(logit)))
    return;
  const float* W = cam.W;
  // 1. camera space
  float tv[3];
#pragma unroll
  for (int r = 0; r < 3; ++r) {
    float v = __fmul_rn(W[3 * r], mx);
    v = __fmaf_rn(W[3 * r + 1], my, v);
    v = __fmaf_rn(W[3 * r + 2], mz, v);
    tv[r] = __fadd_rn(v, cam.t[r]);
  }
  const float tx = tv[0], ty = tv[1], tz = tv[2];
  if (!(tz > cam.near_z)) return;
  // 2. scales
  const float s[3] = {exp_spec(l0), exp_spec(l1), exp_spec(l2)};
  // 3. quaternion
  float n2 = __fmul_rn(qw, qw);
  n2 = __fmaf_rn(qx, qx, n2);
  n2 = __fmaf_rn(qy, qy, n2);
  n2 = __fmaf_rn(qz, qz, n2);
  if (!(n2 > 0.0f)) return;
  const float nq = __fsqrt_rn(n2);
  const float w = __fdiv_rn(qw, nq), x = __fdiv_rn(qx, nq), y = __fdiv_rn(qy, nq),
              z = __fdiv_rn(qz, nq);
  // 4. rotation matrix
  const float xx = __fmul_rn(x, x), yy = __fmul_rn(y, y), zz = __fmul_rn(z, z);
  const float xy = __fmul_rn(x, y), xz = __fmul_rn(x, z), yz = __fmul_rn(y, z);
  const float wx = __fmul_rn(w, x), wy = __fmul_rn(w, y), wz = __fmul_rn(w, z);
  float Rq[9];
  Rq[0] = __fsub_rn(1.0f, __fmul_rn(2.0f, __fadd_rn(yy, zz)));
  Rq[1] = __fmul_rn(2.0f, __fsub_rn(xy, wz));
  Rq[2] = __fmul_rn(2.0f, __fadd_rn(xz, wy));
  Rq[3] = __fmul_rn(2.0f, __fadd_rn(xy, wz));
  Rq[4] = __fsub_rn(1.0f, __fmul_rn(2.0f, __fadd_rn(xx, zz)));
  Rq[5] = __fmul_rn(2.0f, __fsub_rn(yz, wx));
  Rq[6] = __fmul_rn(2.0f, __fsub_rn(xz, wy));
  Rq[7] = __fmul_rn(2.0f, __fadd_rn(yz, wx));
  Rq[8] = __fsub_rn(1.0f, __fmul_rn(2.0f, __fadd_rn(xx, yy)));
  // 5. M = Rq diag(s)
  float M[9];
#pragma unroll
  for (int i = 0; i < 3; ++i)
#pragma unroll
    for (int j = 0; j < 3; ++j) M[3 * i + j] = __fmul_rn(Rq[3 * i + j], s[j]);
  // 6. Sigma = M M^T
  float S[9];
#pragma unroll
  for (int i = 0; i < 3; ++i)
#pragma unroll
    for (int j = i; j < 3; ++j) {
      float v = __fmul_rn(M[3 * i], M[3 * j]);
      v = __fmaf_rn(M[3 * i + 1], M[3 * j + 1], v);
      v = __fmaf_rn(M[3 * i + 2], M[3 * j + 2], v);
      S[3 * i + j] = v;
      S[3 * j + i] = v;
    }
  // 7. Jacobian of the pinhole map at t
  const float tz2 = __fmul_rn(tz, tz);
  const float j00 = __fdiv_rn(cam.fx, tz), j11 = __fdiv_rn(cam.fy, tz);
  const float j02 = -__fdiv_rn(__fmul_rn(cam.fx, tx), tz2);
  const float j12 = -__fdiv_rn(__fmul_rn(cam.fy, ty), tz2);
  // 8. T = J W
  float T[6];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    T[j] = __fmaf_rn(j02, W[6 + j], __fmul_rn(j00, W[j]));
    T[3 + j] = __fmaf_rn(j12, W[6 + j], __fmul_rn(j11, W[3 + j]));
  }
  // 9. U = T Sigma
  float U[6];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      float v = __fmul_rn(T[3 * i], S[j]);
      v = __fmaf_rn(T[3 * i + 1], S[3 + j], v);
      v = __fmaf_rn(T[3 * i + 2], S[6 + j], v);
      U[3 * i + j] = v;
    }
  // 10. Sigma' = U T^T + 0.3 I
  float c00 = __fmul_rn(U[0], T[0]);
  c00 = __fmaf_rn(U[1], T[1], c00);
  c00 = __fmaf_rn(U[2], T[2], c00);
  float c01 = __fmul_rn(U[0], T[3]);
  c01 = __fmaf_rn(U[1], T[4], c01);
  c01 = __fmaf_rn(U[2], T[5], c01);
  float c11 = __fmul_rn(U[3], T[3]);
  c11 = __fmaf_rn(U[4], T[4], c11);
  c11 = __fmaf_rn(U[5], T[5], c11);
  const float a = __fadd_rn(c00, kDilation), b = c01, c = __fadd_rn(c11, kDilation);
  // 11. conic
  const float bb = __fmul_rn(b, b);
  const float det = __fmaf_rn(a, c, -bb);
  if (!(det > 0.0f)) return;
  const float cA = __fdiv_rn(c, det), cB = __fdiv_rn(-b, det), cC = __fdiv_rn(a, det);
  // 12. radius
  const float mid = __fmul_rn(0.5f, __fadd_rn(a, c));
  float d = __fmaf_rn(mid, mid, -det);
  if (!(d > 0.0f)) d = 0.0f;
  const float lam = __fadd_rn(mid, __fsqrt_rn(d));
  const float rf = ceilf(__fmul_rn(3.0f, __fsqrt_rn(lam)));
  // 13. centre
  const float xn = __fdiv_rn(tx, tz), yn = __fdiv_rn(ty, tz);
  const float px = __fmaf_rn(cam.fx, xn, cam.cx);
  const float py = __fmaf_rn(cam.fy, yn, cam.cy);
  if (!(finitef(px) && finitef(py) && finitef(rf) && finitef(cA) && finitef(cB) && finitef(cC)))
    return;
  // 14. tile rect
  const float TWf = (float)cam.TW, THf = (float)cam.TH;
  const int x0 = (int)clamp_grid(floorf(__fmul_rn(__fsub_rn(px, rf), 0.0625f)), TWf);
  const int x1 = (int)clamp_grid(__fadd_rn(floorf(__fmul_rn(__fadd_rn(px, rf), 0.0625f)), 1.0f), TWf);
  const int y0 = (int)clamp_grid(floorf(__fmul_rn(__fsub_rn(py, rf), 0.0625f)), THf);
  const int y1 = (int)clamp_grid(__fadd_rn(floorf(__fmul_rn(__fadd_rn(py, rf), 0.0625f)), 1.0f), THf);
  if ((x1 - x0) * (y1 - y0) <= 0) return;
  // 15. opacity
  const float op = __fdiv_rn(1.0f, __fadd_rn(1.0f, exp_spec(-logit)));
  // 16. colour
  const float dx = __fsub_rn(mx, cam.campos[0]), dy = __fsub_rn(my, cam.campos[1]),
              dz = __fsub_rn(mz, cam.campos[2]);
  float nn = __fmul_rn(dx, dx);
  nn = __fmaf_rn(dy, dy, nn);
  nn = __fmaf_rn(dz, dz, nn);
  const float nd = __fsqrt_rn(nn);
  float Y[K];
  sh_basis<K>(__fdiv_rn(dx, nd), __fdiv_rn(dy, nd), __fdiv_rn(dz, nd), Y);
#pragma unroll
  for (int ch = 0; ch < 3; ++ch) {
    float acc = __fmul_rn(Y[0], src.sh(ch));
#pragma unroll
    for (int k = 1; k < K; ++k) acc = __fmaf_rn(Y[k], src.sh(3 * k + ch), acc);
    const float v = __fadd_rn(acc, 0.5f);
    o.rgb[ch] = v > 0.0f ? v : 0.0f;
  }
  // an infinite colour (from infinite SH coefficients) culls, like a non-finite parameter
  if (!(finitef(o.rgb[0]) && finitef(o.rgb[1]) && finitef(o.rgb[2]))) return;
  o.visible = true;
  o.px = px; o.py = py; o.depth = tz; o.opacity = op;
  o.A = cA; o.B = cB; o.C = cC; o.rf = rf;
  o.x0 = x0; o.y0 = y0; o.x1 = x1; o.y1 = y1;
}

// One record: the projection, or zeros for a Gaussian that is culled.
__device__ __forceinline__ void write_record(const Proj& o, const Records& out, int64_t i) {
  if (o.visible) {
    out.xyzo[i] = make_float4(o.px, o.py, o.depth, o.opacity);
    out.conic[i] = make_float4(o.A, o.B, o.C, 0.0f);
    out.rgb[i] = make_float4(o.rgb[0], o.rgb[1], o.rgb[2], 0.0f);
    out.radius[i] = o.rf < 1073741824.0f ? (int)o.rf : 1073741824;
    out.rect[i] = make_ushort4((unsigned short)o.x0, (unsigned short)o.y0, (unsigned short)o.x1,
                               (unsigned short)o.y1);
    out.tiles[i] = (o.x1 - o.x0) * (o.y1 - o.y0);
  } else {
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    out.xyzo[i] = z;
    out.conic[i] = z;
    out.rgb[i] = z;
    out.radius[i] = 0;
    out.rect[i] = make_ushort4(0, 0, 0, 0);
    out.tiles[i] = 0;
  }
}

template <int K>
__global__ void __launch_bounds__(256) preprocess_kernel(Params p, DevCam cam, Records out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= p.N) return;
  const int64_t na = p.n_active ? (int64_t)*p.n_active : p.N;
  Proj o;
  o.visible = false;
  if (i < na) {
    const int64_t g = p.active_idx ? (int64_t)p.active_idx[i] : i;
    if (check(g >= 0 && g < p.N, kCheckRecordIndex)) project<K>(PlaneSource{p, g}, cam, o);
  }
  write_record(o, out, i);
}

// Several views in one pass: each Gaussian's 11 + 3K parameters are read from
// HBM once and projected into every view. The 11 geometric parameters stay
// in registers, the 3K SH coefficients in shared memory (a column per
// thread, conflict-free), read through a volatile pointer where they are
// used so that the compiler does not hoist them into registers across the
// view loop: 64 registers, 4 CTAs per SM.
constexpr int kMvBlock = 256;
template <int K>
struct StagedSource {
  float m[3], l[3], q[4], lg;
  const volatile float* c;  // the thread's column: plane k at c[k * kMvBlock] (volatile: read where used)
  __device__ __forceinline__ void load(const Params& p, int64_t g, float* column) {
#pragma unroll
    for (int r = 0; r < 3; ++r) m[r] = p.means[r * p.N + g];
#pragma unroll
    for (int r = 0; r < 3; ++r) l[r] = p.log_scales[r * p.N + g];
#pragma unroll
    for (int r = 0; r < 4; ++r) q[r] = p.quats[r * p.N + g];
    lg = p.logits[g];
#pragma unroll
    for (int k = 0; k < 3 * K; ++k) column[k * kMvBlock] = p.sh[(int64_t)k * p.N + g];
    c = column;
  }
  __device__ __forceinline__ float mean(int r) const { return m[r]; }
  __device__ __forceinline__ float log_scale(int r) const { return l[r]; }
  __device__ __forceinline__ float quat(int r) const { return q[r]; }
  __device__ __forceinline__ float logit() const { return lg; }
  __device__ __forceinline__ float sh(int plane) const { return c[plane * kMvBlock]; }
};
template <int K>
__global__ void __launch_bounds__(kMvBlock, 4) preprocess_multiview_kernel(Params p, MultiViewArgs mv) {
  __shared__ float s_sh[3 * K][kMvBlock];
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= p.N) return;
  StagedSource<K> src;
  src.load(p, i, &s_sh[0][threadIdx.x]);
  for (int v = 0; v < mv.n_views; ++v) {
    Proj o;
    project<K>(src, mv.cam[v], o);
    write_record(o, mv.out[v], i);
  }
}


// ------------------------------------------------------------------ backward

// Gradients of the basis polynomials with respect to (x, y, z).
template <int K>
__device__ __forceinline__ void sh_basis_grad(float x, float y, float z, float G[][3]) {
#pragma unroll
  for (int k = 0; k < K; ++k) G[k][0] = G[k][1] = G[k][2] = 0.0f;
  if (K <= 1) return;
  G[1][1] = -kSH1;
  G[2][2] = kSH1;
  G[3][0] = -kSH1;
  if (K <= 4) return;
  G[4][0] = kSH2a * y; G[4][1] = kSH2a * x;
  G[5][1] = -kSH2a * z; G[5][2] = -kSH2a * y;
  G[6][0] = -2.0f * kSH2b * x; G[6][1] = -2.0f * kSH2b * y; G[6][2] = 4.0f * kSH2b * z;
  G[7][0] = -kSH2a * z; G[7][2] = -kSH2a * x;
  G[8][0] = 2.0f * kSH2c * x; G[8][1] = -2.0f * kSH2c * y;
  if (K <= 9) return;
  const float xx = x * x, yy = y * y, zz = z * z;
  G[9][0] = -kSH3a * 6.0f * x * y; G[9][1] = -kSH3a * 3.0f * (xx - yy);
  G[10][0] = kSH3b * y * z; G[10][1] = kSH3b * x * z; G[10][2] = kSH3b * x * y;
  G[11][0] = -kSH3c * (-2.0f * x * y);
  G[11][1] = -kSH3c * (4.0f * zz - xx - 3.0f * yy);
  G[11][2] = -kSH3c * 8.0f * y * z;
  G[12][0] = kSH3d * (-6.0f * x * z);
  G[12][1] = kSH3d * (-6.0f * y * z);
  G[12][2] = kSH3d * (6.0f * zz - 3.0f * xx - 3.0f * yy);
  G[13][0] = -kSH3c * (4.0f * zz - 3.0f * xx - yy);
  G[13][1] = -kSH3c * (-2.0f * x * y);
  G[13][2] = -kSH3c * 8.0f * x * z;
  G[14][0] = kSH3e * 2.0f * x * z; G[14][1] = kSH3e * (-2.0f * y * z); G[14][2] = kSH3e * (xx - yy);
  G[15][0] = -kSH3a * 3.0f * (xx - yy); G[15][1] = -kSH3a * (-6.0f * x * y);
}

__device__ __forceinline__ void zero_grads(const Grads& gr, int64_t N, int K, int64_t g) {
#pragma unroll
  for (int m = 0; m < 3; ++m) gr.d_means[m * N + g] = 0.0f;
#pragma unroll
  for (int m = 0; m < 3; ++m) gr.d_log_scales[m * N + g] = 0.0f;
#pragma unroll
  for (int m = 0; m < 4; ++m) gr.d_quats[m * N + g] = 0.0f;
  gr.d_logits[g] = 0.0f;
  for (int k = 0; k < 3 * K; ++k) gr.d_sh[(int64_t)k * N + g] = 0.0f;
}

// How the kernel writes the gradient rows.
enum GradMode {
  kWriteAll = 0,    // every row: the chain for visible records, zeros for culled and invisible ones
  kPreZeroed = 1,   // the rows were zeroed by a memset first (a cull mask is given, so most rows are
                    // zero and the memset writes them at copy bandwidth): visible records only
  kAccumulate = 2,  // visible records' chains added to the rows; nothing else touched
};

template <int kMode>
__device__ __forceinline__ void put_grad(float* p, float v) {
  if (kMode == kAccumulate)
    *p += v;
  else
    *p = v;
}

template <int K, int kMode>
__global__ void __launch_bounds__(256) preprocess_bwd_kernel(Params p, const uint8_t* mask, DevCam cam,
                                                             Records rec, const float4* grad2d,
                                                             Grads gr) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t N = p.N;
  if (i >= N) return;
  // Gaussian i culled by the active-set mask: its gradient is zero.
  if (kMode == kWriteAll && mask && mask[i] == 0) zero_grads(gr, N, K, i);
  const int64_t na = p.n_active ? (int64_t)*p.n_active : N;
  if (i >= na) return;
  const int64_t g = p.active_idx ? (int64_t)p.active_idx[i] : i;
  if (!check(g >= 0 && g < N, kCheckRecordIndex)) return;
  if (rec.tiles[i] <= 0) {
    if (kMode == kWriteAll) zero_grads(gr, N, K, g);
    return;
  }
  const float4 g0 = grad2d[3 * i], g1 = grad2d[3 * i + 1], g2 = grad2d[3 * i + 2];
  const float4 colour = rec.rgb[i];
  const float* W = cam.W;
  const float mu[3] = {p.means[g], p.means[N + g], p.means[2 * N + g]};
  const float ls[3] = {p.log_scales[g], p.log_scales[N + g], p.log_scales[2 * N + g]};
  const float q[4] = {p.quats[g], p.quats[N + g], p.quats[2 * N + g], p.quats[3 * N + g]};
  const float logit = p.logits[g];
  // forward quantities
  float t[3];
#pragma unroll
  for (int r = 0; r < 3; ++r) t[r] = fmaf(W[3 * r + 2], mu[2], fmaf(W[3 * r + 1], mu[1], W[3 * r] * mu[0])) + cam.t[r];
  const float s[3] = {exp_spec(ls[0]), exp_spec(ls[1]), exp_spec(ls[2])};
  const float nq = sqrtf(fmaf(q[3], q[3], fmaf(q[2], q[2], fmaf(q[1], q[1], q[0] * q[0]))));
  const float inq = 1.0f / nq;
  const float w = q[0] * inq, x = q[1] * inq, y = q[2] * inq, z = q[3] * inq;
  const float Rq[9] = {1.f - 2.f * (y * y + z * z), 2.f * (x * y - w * z), 2.f * (x * z + w * y),
                       2.f * (x * y + w * z), 1.f - 2.f * (x * x + z * z), 2.f * (y * z - w * x),
                       2.f * (x * z - w * y), 2.f * (y * z + w * x), 1.f - 2.f * (x * x + y * y)};
  float M[9], S[9];
#pragma unroll
  for (int a = 0; a < 3; ++a)
#pragma unroll
    for (int b = 0; b < 3; ++b) M[3 * a + b] = Rq[3 * a + b] * s[b];
#pragma unroll
  for (int a = 0; a < 3; ++a)
#pragma unroll
    for (int b = 0; b < 3; ++b)
      S[3 * a + b] = fmaf(M[3 * a + 2], M[3 * b + 2], fmaf(M[3 * a + 1], M[3 * b + 1], M[3 * a] * M[3 * b]));
  const float fx = cam.fx, fy = cam.fy, tz = t[2], itz = 1.0f / tz, itz2 = itz * itz;
  const float J00 = fx * itz, J11 = fy * itz, J02 = -fx * t[0] * itz2, J12 = -fy * t[1] * itz2;
  float T[6];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    T[j] = fmaf(J02, W[6 + j], J00 * W[j]);
    T[3 + j] = fmaf(J12, W[6 + j], J11 * W[3 + j]);
  }
  float TS[6];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int j = 0; j < 3; ++j)
      TS[3 * a + j] = fmaf(T[3 * a + 2], S[6 + j], fmaf(T[3 * a + 1], S[3 + j], T[3 * a] * S[j]));
  const float ca = fmaf(TS[2], T[2], fmaf(TS[1], T[1], TS[0] * T[0])) + kDilation;
  const float cb = fmaf(TS[2], T[5], fmaf(TS[1], T[4], TS[0] * T[3]));
  const float cc = fmaf(TS[5], T[5], fmaf(TS[4], T[4], TS[3] * T[3])) + kDilation;
  const float det = fmaf(ca, cc, -cb * cb);
  const float id = 1.0f / det, id2 = id * id;
  const float op = 1.0f / (1.0f + exp_spec(-logit));

  const float gpx = g0.x, gpy = g0.y, gop = g0.z, gA = g1.x, gB = g1.y, gC = g1.z;
  float g_mu[3], g_t[3];
  // opacity
  put_grad<kMode>(&gr.d_logits[g], gop * op * (1.0f - op));
  // colour
  const float dv[3] = {mu[0] - cam.campos[0], mu[1] - cam.campos[1], mu[2] - cam.campos[2]};
  const float nd = sqrtf(fmaf(dv[2], dv[2], fmaf(dv[1], dv[1], dv[0] * dv[0])));
  const float ind = 1.0f / nd;
  const float dir[3] = {dv[0] * ind, dv[1] * ind, dv[2] * ind};
  float Y[K];
  sh_basis<K>(dir[0], dir[1], dir[2], Y);
  const float gv[3] = {colour.x > 0.0f ? g2.x : 0.0f, colour.y > 0.0f ? g2.y : 0.0f,
                       colour.z > 0.0f ? g2.z : 0.0f};
  float gdir[3] = {0.f, 0.f, 0.f};
  {
    float DY[K][3];
    sh_basis_grad<K>(dir[0], dir[1], dir[2], DY);
#pragma unroll
    for (int k = 0; k < K; ++k) {
      float gY = 0.0f;
#pragma unroll
      for (int ch = 0; ch < 3; ++ch) {
        const int64_t plane = (int64_t)(3 * k + ch) * N + g;
        put_grad<kMode>(&gr.d_sh[plane], gv[ch] * Y[k]);
        gY = fmaf(gv[ch], p.sh[plane], gY);
      }
#pragma unroll
      for (int m = 0; m < 3; ++m) gdir[m] = fmaf(gY, DY[k][m], gdir[m]);
    }
  }
  const float ddot = gdir[0] * dir[0] + gdir[1] * dir[1] + gdir[2] * dir[2];
#pragma unroll
  for (int m = 0; m < 3; ++m) g_mu[m] = (gdir[m] - ddot * dir[m]) * ind;
  // projected centre
  g_t[0] = gpx * fx * itz;
  g_t[1] = gpy * fy * itz;
  g_t[2] = -(gpx * fx * t[0] + gpy * fy * t[1]) * itz2;
  // conic -> Sigma'
  const float ga = (-cc * cc * gA + cb * cc * gB - cb * cb * gC) * id2;
  const float gb = (2.f * cb * cc * gA - (ca * cc + cb * cb) * gB + 2.f * ca * cb * gC) * id2;
  const float gc = (-cb * cb * gA + ca * cb * gB - ca * ca * gC) * id2;
  const float Gm[4] = {ga, 0.5f * gb, 0.5f * gb, gc};
  float GT[6];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int j = 0; j < 3; ++j) GT[3 * a + j] = Gm[2 * a] * T[j] + Gm[2 * a + 1] * T[3 + j];
  float gS[9];
#pragma unroll
  for (int a = 0; a < 3; ++a)
#pragma unroll
    for (int b = 0; b < 3; ++b) gS[3 * a + b] = T[a] * GT[b] + T[3 + a] * GT[3 + b];
  float gT[6];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int j = 0; j < 3; ++j) gT[3 * a + j] = 2.f * (Gm[2 * a] * TS[j] + Gm[2 * a + 1] * TS[3 + j]);
  float gM[9];
#pragma unroll
  for (int a = 0; a < 3; ++a)
#pragma unroll
    for (int b = 0; b < 3; ++b)
      gM[3 * a + b] = 2.f * (gS[3 * a] * M[b] + gS[3 * a + 1] * M[3 + b] + gS[3 * a + 2] * M[6 + b]);
  float gR[9];
#pragma unroll
  for (int b = 0; b < 3; ++b) {
    float gs = 0.0f;
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      gs = fmaf(gM[3 * a + b], Rq[3 * a + b], gs);
      gR[3 * a + b] = gM[3 * a + b] * s[b];
    }
    put_grad<kMode>(&gr.d_log_scales[b * N + g], gs * s[b]);
  }
  const float gw = 2.f * (-z * gR[1] + y * gR[2] + z * gR[3] - x * gR[5] - y * gR[6] + x * gR[7]);
  const float gx = 2.f * (y * gR[1] + z * gR[2] + y * gR[3] - 2.f * x * gR[4] - w * gR[5] + z * gR[6] +
                          w * gR[7] - 2.f * x * gR[8]);
  const float gy = 2.f * (-2.f * y * gR[0] + x * gR[1] + w * gR[2] + x * gR[3] + z * gR[5] - w * gR[6] +
                          z * gR[7] - 2.f * y * gR[8]);
  const float gz = 2.f * (-2.f * z * gR[0] - w * gR[1] + x * gR[2] + w * gR[3] - 2.f * z * gR[4] + y * gR[5] +
                          x * gR[6] + y * gR[7]);
  const float qdot = gw * w + gx * x + gy * y + gz * z;
  put_grad<kMode>(&gr.d_quats[g], (gw - qdot * w) * inq);
  put_grad<kMode>(&gr.d_quats[N + g], (gx - qdot * x) * inq);
  put_grad<kMode>(&gr.d_quats[2 * N + g], (gy - qdot * y) * inq);
  put_grad<kMode>(&gr.d_quats[3 * N + g], (gz - qdot * z) * inq);
  float gJ00 = 0.f, gJ02 = 0.f, gJ11 = 0.f, gJ12 = 0.f;
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    gJ00 = fmaf(gT[j], W[j], gJ00);
    gJ02 = fmaf(gT[j], W[6 + j], gJ02);
    gJ11 = fmaf(gT[3 + j], W[3 + j], gJ11);
    gJ12 = fmaf(gT[3 + j], W[6 + j], gJ12);
  }
  g_t[0] += -fx * itz2 * gJ02;
  g_t[1] += -fy * itz2 * gJ12;
  g_t[2] += -(fx * gJ00 + fy * gJ11) * itz2 + 2.f * (fx * t[0] * gJ02 + fy * t[1] * gJ12) * itz2 * itz;
#pragma unroll
  for (int m = 0; m < 3; ++m)
    put_grad<kMode>(&gr.d_means[m * N + g], g_mu[m] + g_t[0] * W[m] + g_t[1] * W[3 + m] + g_t[2] * W[6 + m]);
}


// Backward of several views of one model in one pass: the parameter
// gradients of a loss summed over the views (record i of every view is
// Gaussian i, no cull, as gs_preprocess_multiview writes them). Each
// Gaussian's parameters are read once; its view-independent quantities
// (scales, rotation, Sigma, opacity) are computed once; per view that sees
// it, the chain to (Sigma, t, colour) runs as in preprocess_bwd_kernel and
// its gradients with respect to Sigma, the opacity, the mean and the SH
// coefficients are summed in registers; the chain from Sigma to the scales
// and the rotation, which is linear in dL/dSigma, then runs once on the sum.
// Every gradient row is written once (zeros for a Gaussian no view sees).
// The Gaussian's 3K SH coefficients and their 3K gradient sums live in
// shared memory ([coefficient][thread]: each thread its own column,
// conflict-free), the rest in registers: 96 registers and 24 KB per CTA of
// 64 threads, 9 CTAs (18 warps) per SM.
constexpr int kMvBwdBlock = 64;
template <int K>
__global__ void __launch_bounds__(kMvBwdBlock, 9) preprocess_bwd_multiview_kernel(Params p, MultiViewBwdArgs a,
                                                                             Grads gr) {
  __shared__ float s_gsh[3 * K][kMvBwdBlock];
  __shared__ float s_sh[3 * K][kMvBwdBlock];
  // coefficient k at [k * kMvBwdBlock]; volatile: each use reads shared memory
  // instead of a register copy hoisted out of the view loop
  volatile float* sum_gsh = &s_gsh[0][threadIdx.x];
  volatile float* shc = &s_sh[0][threadIdx.x];
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t N = p.N;
  if (g >= N) return;
  bool seen = false;
  for (int v = 0; v < a.n_views; ++v) seen |= a.rec[v].tiles[g] > 0;
  if (!seen) {
    zero_grads(gr, N, K, g);
    return;
  }
  const float mu[3] = {p.means[g], p.means[N + g], p.means[2 * N + g]};
  const float ls[3] = {p.log_scales[g], p.log_scales[N + g], p.log_scales[2 * N + g]};
  const float q[4] = {p.quats[g], p.quats[N + g], p.quats[2 * N + g], p.quats[3 * N + g]};
  const float logit = p.logits[g];
  // view-independent forward quantities
  const float s[3] = {exp_spec(ls[0]), exp_spec(ls[1]), exp_spec(ls[2])};
  const float nq = sqrtf(fmaf(q[3], q[3], fmaf(q[2], q[2], fmaf(q[1], q[1], q[0] * q[0]))));
  const float inq = 1.0f / nq;
  const float w = q[0] * inq, x = q[1] * inq, y = q[2] * inq, z = q[3] * inq;
  float S6[6];  // Sigma = M M^T, upper triangle
  {
    const float Rq[9] = {1.f - 2.f * (y * y + z * z), 2.f * (x * y - w * z), 2.f * (x * z + w * y),
                         2.f * (x * y + w * z), 1.f - 2.f * (x * x + z * z), 2.f * (y * z - w * x),
                         2.f * (x * z - w * y), 2.f * (y * z + w * x), 1.f - 2.f * (x * x + y * y)};
    float M[9];
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
      for (int j = 0; j < 3; ++j) M[3 * i + j] = Rq[3 * i + j] * s[j];
    int u = 0;
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
      for (int j = i; j < 3; ++j)
        S6[u++] = fmaf(M[3 * i + 2], M[3 * j + 2], fmaf(M[3 * i + 1], M[3 * j + 1], M[3 * i] * M[3 * j]));
  }
  // sums over the views
  // sums over the views; dL/dSigma as its upper triangle (Sigma is symmetric)
  float sum_gS[6] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, sum_gmu[3] = {0.f, 0.f, 0.f}, sum_gop = 0.0f;
#pragma unroll
  for (int k = 0; k < 3 * K; ++k) {
    sum_gsh[k * kMvBwdBlock] = 0.0f;
    shc[k * kMvBwdBlock] = p.sh[(int64_t)k * N + g];
  }
#pragma unroll 1
  for (int v = 0; v < a.n_views; ++v) {
    if (a.rec[v].tiles[g] <= 0) continue;
    const DevCam& cam = a.cam[v];
    const float4* g2d = a.grad2d[v];
    // colour first (its temporaries die before the geometry's are born)
    float gmu_dir[3];
    {
      const float4 g2 = g2d[3 * g + 2];
      const float4 colour = a.rec[v].rgb[g];
      const float dv[3] = {mu[0] - cam.campos[0], mu[1] - cam.campos[1], mu[2] - cam.campos[2]};
      const float nd = sqrtf(fmaf(dv[2], dv[2], fmaf(dv[1], dv[1], dv[0] * dv[0])));
      const float ind = 1.0f / nd;
      const float dir[3] = {dv[0] * ind, dv[1] * ind, dv[2] * ind};
      float Y[K];
      sh_basis<K>(dir[0], dir[1], dir[2], Y);
      const float gv[3] = {colour.x > 0.0f ? g2.x : 0.0f, colour.y > 0.0f ? g2.y : 0.0f,
                           colour.z > 0.0f ? g2.z : 0.0f};
      float gdir[3] = {0.f, 0.f, 0.f};
      float DY[K][3];
      sh_basis_grad<K>(dir[0], dir[1], dir[2], DY);
#pragma unroll
      for (int k = 0; k < K; ++k) {
        float gY = 0.0f;
#pragma unroll
        for (int ch = 0; ch < 3; ++ch) {
          sum_gsh[(3 * k + ch) * kMvBwdBlock] += gv[ch] * Y[k];
          gY = fmaf(gv[ch], shc[(3 * k + ch) * kMvBwdBlock], gY);
        }
#pragma unroll
        for (int m = 0; m < 3; ++m) gdir[m] = fmaf(gY, DY[k][m], gdir[m]);
      }
      const float ddot = gdir[0] * dir[0] + gdir[1] * dir[1] + gdir[2] * dir[2];
#pragma unroll
      for (int m = 0; m < 3; ++m) gmu_dir[m] = (gdir[m] - ddot * dir[m]) * ind;
    }
    // geometry
    const float4 g0 = g2d[3 * g], g1 = g2d[3 * g + 1];
    sum_gop += g0.z;
    const float* W = cam.W;
    float t[3];
#pragma unroll
    for (int r = 0; r < 3; ++r)
      t[r] = fmaf(W[3 * r + 2], mu[2], fmaf(W[3 * r + 1], mu[1], W[3 * r] * mu[0])) + cam.t[r];
    const float fx = cam.fx, fy = cam.fy, tz = t[2], itz = 1.0f / tz, itz2 = itz * itz;
    const float J00 = fx * itz, J11 = fy * itz, J02 = -fx * t[0] * itz2, J12 = -fy * t[1] * itz2;
    float T[6];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      T[j] = fmaf(J02, W[6 + j], J00 * W[j]);
      T[3 + j] = fmaf(J12, W[6 + j], J11 * W[3 + j]);
    }
    // TS = T Sigma, Sigma from its upper triangle S6 = (00, 01, 02, 11, 12, 22)
    const float Sf[9] = {S6[0], S6[1], S6[2], S6[1], S6[3], S6[4], S6[2], S6[4], S6[5]};
    float TS[6];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 3; ++j)
        TS[3 * i + j] = fmaf(T[3 * i + 2], Sf[6 + j], fmaf(T[3 * i + 1], Sf[3 + j], T[3 * i] * Sf[j]));
    const float ca = fmaf(TS[2], T[2], fmaf(TS[1], T[1], TS[0] * T[0])) + kDilation;
    const float cb = fmaf(TS[2], T[5], fmaf(TS[1], T[4], TS[0] * T[3]));
    const float cc = fmaf(TS[5], T[5], fmaf(TS[4], T[4], TS[3] * T[3])) + kDilation;
    const float det = fmaf(ca, cc, -cb * cb);
    const float id = 1.0f / det, id2 = id * id;
    const float gpx = g0.x, gpy = g0.y, gA = g1.x, gB = g1.y, gC = g1.z;
    float g_t[3];
    g_t[0] = gpx * fx * itz;
    g_t[1] = gpy * fy * itz;
    g_t[2] = -(gpx * fx * t[0] + gpy * fy * t[1]) * itz2;
    // conic -> Sigma'
    const float ga = (-cc * cc * gA + cb * cc * gB - cb * cb * gC) * id2;
    const float gb = (2.f * cb * cc * gA - (ca * cc + cb * cb) * gB + 2.f * ca * cb * gC) * id2;
    const float gc = (-cb * cb * gA + ca * cb * gB - ca * ca * gC) * id2;
    const float Gm[4] = {ga, 0.5f * gb, 0.5f * gb, gc};
    float GT[6];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 3; ++j) GT[3 * i + j] = Gm[2 * i] * T[j] + Gm[2 * i + 1] * T[3 + j];
    // dL/dSigma = T^T Gm T (upper triangle)
    {
      int u = 0;
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int j = i; j < 3; ++j) sum_gS[u++] += T[i] * GT[j] + T[3 + i] * GT[3 + j];
    }
    float gJ00 = 0.f, gJ02 = 0.f, gJ11 = 0.f, gJ12 = 0.f;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const float gT0 = 2.f * (Gm[0] * TS[j] + Gm[1] * TS[3 + j]);
      const float gT1 = 2.f * (Gm[2] * TS[j] + Gm[3] * TS[3 + j]);
      gJ00 = fmaf(gT0, W[j], gJ00);
      gJ02 = fmaf(gT0, W[6 + j], gJ02);
      gJ11 = fmaf(gT1, W[3 + j], gJ11);
      gJ12 = fmaf(gT1, W[6 + j], gJ12);
    }
    g_t[0] += -fx * itz2 * gJ02;
    g_t[1] += -fy * itz2 * gJ12;
    g_t[2] += -(fx * gJ00 + fy * gJ11) * itz2 + 2.f * (fx * t[0] * gJ02 + fy * t[1] * gJ12) * itz2 * itz;
#pragma unroll
    for (int m = 0; m < 3; ++m) sum_gmu[m] += gmu_dir[m] + g_t[0] * W[m] + g_t[1] * W[3 + m] + g_t[2] * W[6 + m];
  }
  // the view-independent chain, once, on the sums
  const float op = 1.0f / (1.0f + exp_spec(-logit));
  gr.d_logits[g] = sum_gop * op * (1.0f - op);
#pragma unroll
  for (int k = 0; k < 3 * K; ++k) gr.d_sh[(int64_t)k * N + g] = sum_gsh[k * kMvBwdBlock];
#pragma unroll
  for (int m = 0; m < 3; ++m) gr.d_means[m * N + g] = sum_gmu[m];
  const float Rq[9] = {1.f - 2.f * (y * y + z * z), 2.f * (x * y - w * z), 2.f * (x * z + w * y),
                       2.f * (x * y + w * z), 1.f - 2.f * (x * x + z * z), 2.f * (y * z - w * x),
                       2.f * (x * z - w * y), 2.f * (y * z + w * x), 1.f - 2.f * (x * x + y * y)};
  float M[9];
#pragma unroll
  for (int i = 0; i < 3; ++i)
#pragma unroll
    for (int j = 0; j < 3; ++j) M[3 * i + j] = Rq[3 * i + j] * s[j];
  const float gS[9] = {sum_gS[0], sum_gS[1], sum_gS[2], sum_gS[1], sum_gS[3], sum_gS[4],
                       sum_gS[2], sum_gS[4], sum_gS[5]};
  float gM[9];
#pragma unroll
  for (int i = 0; i < 3; ++i)
#pragma unroll
    for (int j = 0; j < 3; ++j)
      gM[3 * i + j] = 2.f * (gS[3 * i] * M[j] + gS[3 * i + 1] * M[3 + j] + gS[3 * i + 2] * M[6 + j]);
  float gR[9];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    float gs = 0.0f;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      gs = fmaf(gM[3 * i + j], Rq[3 * i + j], gs);
      gR[3 * i + j] = gM[3 * i + j] * s[j];
    }
    gr.d_log_scales[j * N + g] = gs * s[j];
  }
  const float gw = 2.f * (-z * gR[1] + y * gR[2] + z * gR[3] - x * gR[5] - y * gR[6] + x * gR[7]);
  const float gx = 2.f * (y * gR[1] + z * gR[2] + y * gR[3] - 2.f * x * gR[4] - w * gR[5] + z * gR[6] +
                          w * gR[7] - 2.f * x * gR[8]);
  const float gy = 2.f * (-2.f * y * gR[0] + x * gR[1] + w * gR[2] + x * gR[3] + z * gR[5] - w * gR[6] +
                          z * gR[7] - 2.f * y * gR[8]);
  const float gz = 2.f * (-2.f * z * gR[0] - w * gR[1] + x * gR[2] + w * gR[3] - 2.f * z * gR[4] + y * gR[5] +
                          x * gR[6] + y * gR[7]);
  const float qdot = gw * w + gx * x + gy * y + gz * z;
  gr.d_quats[g] = (gw - qdot * w) * inq;
  gr.d_quats[N + g] = (gx - qdot * x) * inq;
  gr.d_quats[2 * N + g] = (gy - qdot * y) * inq;
  gr.d_quats[3 * N + g] = (gz - qdot * z) * inq;
}

}  // namespace

cudaError_t launch_preprocess(const Params& p, const DevCam& cam, const Records& out, cudaStream_t s) {
  if (p.N == 0) return cudaSuccess;
  const unsigned grid = grid_for(p.N, 256);
  switch (p.sh_degree) {
    case 0: preprocess_kernel<1><<<grid, 256, 0, s>>>(p, cam, out); break;
    case 1: preprocess_kernel<4><<<grid, 256, 0, s>>>(p, cam, out); break;
    case 2: preprocess_kernel<9><<<grid, 256, 0, s>>>(p, cam, out); break;
    default: preprocess_kernel<16><<<grid, 256, 0, s>>>(p, cam, out); break;
  }
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_preprocess_multiview(const Params& p, const MultiViewArgs& mv, cudaStream_t s) {
  if (p.N == 0 || mv.n_views == 0) return cudaSuccess;
  const unsigned grid = grid_for(p.N, kMvBlock);
  switch (p.sh_degree) {
    case 0: preprocess_multiview_kernel<1><<<grid, kMvBlock, 0, s>>>(p, mv); break;
    case 1: preprocess_multiview_kernel<4><<<grid, kMvBlock, 0, s>>>(p, mv); break;
    case 2: preprocess_multiview_kernel<9><<<grid, kMvBlock, 0, s>>>(p, mv); break;
    default: preprocess_multiview_kernel<16><<<grid, kMvBlock, 0, s>>>(p, mv); break;
  }
  count_launches(1);
  return cudaGetLastError();
}

namespace {
template <int kMode>
void launch_chain(const Params& p, const uint8_t* mask, const DevCam& cam, const Records& in,
                  const float4* grad2d, const Grads& g, cudaStream_t s) {
  const unsigned grid = grid_for(p.N, 256);
  switch (p.sh_degree) {
    case 0: preprocess_bwd_kernel<1, kMode><<<grid, 256, 0, s>>>(p, mask, cam, in, grad2d, g); break;
    case 1: preprocess_bwd_kernel<4, kMode><<<grid, 256, 0, s>>>(p, mask, cam, in, grad2d, g); break;
    case 2: preprocess_bwd_kernel<9, kMode><<<grid, 256, 0, s>>>(p, mask, cam, in, grad2d, g); break;
    default: preprocess_bwd_kernel<16, kMode><<<grid, 256, 0, s>>>(p, mask, cam, in, grad2d, g); break;
  }
}

}  // namespace

cudaError_t launch_preprocess_bwd(const Params& p, const uint8_t* mask, const DevCam& cam,
                                  const Records& in, const float4* grad2d, const Grads& g,
                                  bool accumulate, cudaStream_t s) {
  if (p.N == 0) return cudaSuccess;
  const int K = (p.sh_degree + 1) * (p.sh_degree + 1);
  if (accumulate) {
    launch_chain<kAccumulate>(p, mask, cam, in, grad2d, g, s);
  } else if (mask) {  // most rows are culled: zero everything at copy bandwidth first
    const size_t row = (size_t)p.N * sizeof(float);
    const size_t planes[5] = {3, 3, 4, 1, (size_t)3 * K};
    float* dst[5] = {g.d_means, g.d_log_scales, g.d_quats, g.d_logits, g.d_sh};
    for (int k = 0; k < 5; ++k) {
      const cudaError_t e = cudaMemsetAsync(dst[k], 0, planes[k] * row, s);
      if (e != cudaSuccess) return e;
    }
    launch_chain<kPreZeroed>(p, mask, cam, in, grad2d, g, s);
  } else {
    launch_chain<kWriteAll>(p, mask, cam, in, grad2d, g, s);
  }
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_preprocess_bwd_multiview(const Params& p, const MultiViewBwdArgs& mv, const Grads& g,
                                            cudaStream_t s) {
  if (p.N == 0) return cudaSuccess;
  const unsigned grid = grid_for(p.N, kMvBwdBlock);
  switch (p.sh_degree) {
    case 0: preprocess_bwd_multiview_kernel<1><<<grid, kMvBwdBlock, 0, s>>>(p, mv, g); break;
    case 1: preprocess_bwd_multiview_kernel<4><<<grid, kMvBwdBlock, 0, s>>>(p, mv, g); break;
    case 2: preprocess_bwd_multiview_kernel<9><<<grid, kMvBwdBlock, 0, s>>>(p, mv, g); break;
    default: preprocess_bwd_multiview_kernel<16><<<grid, kMvBwdBlock, 0, s>>>(p, mv, g); break;
  }
  count_launches(1);
  return cudaGetLastError();
}

uint32_t checked_status_preprocess() { return take_checked_status(); }

}  // namespace gs
