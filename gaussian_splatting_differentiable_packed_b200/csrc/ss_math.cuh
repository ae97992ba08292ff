// Forward math of the packed projection and the rasterizer in the canonical
// fp32 operation order: every product, sum, quotient and square root is an
// explicitly rounded intrinsic (never contracted into an fma by the compiler),
// fma appears only where the operation order prescribes one.  The integer
// outputs (visibility, AABB16, keys, last_id) are decided by these values.
//
// EWA splatting as named on the "Spirula Studio backward pass" page, section 5
// (projection through intrinsics/extrinsics), with the method's constants: 0.3
// dilation, 3-sigma radius, alpha clamp 0.99, skip below 1/255, stop below
// T = 1e-4.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ss {

__device__ __forceinline__ float mul(float a, float b) { return __fmul_rn(a, b); }
__device__ __forceinline__ float add(float a, float b) { return __fadd_rn(a, b); }
__device__ __forceinline__ float sub(float a, float b) { return __fsub_rn(a, b); }
__device__ __forceinline__ float div_(float a, float b) { return __fdiv_rn(a, b); }
// 1/b correctly rounded: the same value as div_(1.0f, b) (both are the exact
// quotient rounded to nearest even), through the reciprocal intrinsic.
__device__ __forceinline__ float rcp_(float b) { return __frcp_rn(b); }
__device__ __forceinline__ float sqrt_(float a) { return __fsqrt_rn(a); }
__device__ __forceinline__ float fma_(float a, float b, float c) { return __fmaf_rn(a, b, c); }

// Camera constants, computed per camera (identical wherever computed).
// 16-byte aligned and padded to six 16-byte words, so that a warp's read of
// a camera from shared memory can use 16-byte loads.
struct __align__(16) Cam {
  float R[9], t[3], fx, fy, cx, cy, limx, limy, cpos[3], pad[3];
};

__device__ __forceinline__ Cam load_cam(const float* c20, int W, int H) {
  Cam k;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
#pragma unroll
    for (int j = 0; j < 3; ++j) k.R[3 * i + j] = c20[4 * i + j];
    k.t[i] = c20[4 * i + 3];
  }
  k.fx = c20[16]; k.fy = c20[17]; k.cx = c20[18]; k.cy = c20[19];
  k.limx = mul(1.3f, div_(mul(0.5f, (float)W), k.fx));
  k.limy = mul(1.3f, div_(mul(0.5f, (float)H), k.fy));
#pragma unroll
  for (int j = 0; j < 3; ++j)
    k.cpos[j] = -add(add(mul(k.R[j], k.t[0]), mul(k.R[3 + j], k.t[1])), mul(k.R[6 + j], k.t[2]));
  return k;
}

// Per-Gaussian covariance Sigma = M M^T, M = R(q/|q|) diag(s).
struct Cov3 {
  float s00, s01, s02, s11, s12, s22;
};

struct QuatRot {
  float w, x, y, z, inv;  // normalised quaternion and 1/|q|
  float R[9];
};

__device__ __forceinline__ QuatRot quat_rot(float qw, float qx, float qy, float qz) {
  QuatRot o;
  float n2 = add(add(add(mul(qw, qw), mul(qx, qx)), mul(qy, qy)), mul(qz, qz));
  o.inv = rcp_(sqrt_(n2));
  float w = mul(qw, o.inv), x = mul(qx, o.inv), y = mul(qy, o.inv), z = mul(qz, o.inv);
  o.w = w; o.x = x; o.y = y; o.z = z;
  float xx = mul(x, x), yy = mul(y, y), zz = mul(z, z);
  float xy = mul(x, y), xz = mul(x, z), yz = mul(y, z);
  float wx = mul(w, x), wy = mul(w, y), wz = mul(w, z);
  o.R[0] = sub(1.0f, mul(2.0f, add(yy, zz)));
  o.R[1] = mul(2.0f, sub(xy, wz));
  o.R[2] = mul(2.0f, add(xz, wy));
  o.R[3] = mul(2.0f, add(xy, wz));
  o.R[4] = sub(1.0f, mul(2.0f, add(xx, zz)));
  o.R[5] = mul(2.0f, sub(yz, wx));
  o.R[6] = mul(2.0f, sub(xz, wy));
  o.R[7] = mul(2.0f, add(yz, wx));
  o.R[8] = sub(1.0f, mul(2.0f, add(xx, yy)));
  return o;
}

__device__ __forceinline__ Cov3 cov3(const QuatRot& q, float sx, float sy, float sz) {
  float M[9];
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    M[3 * i + 0] = mul(q.R[3 * i + 0], sx);
    M[3 * i + 1] = mul(q.R[3 * i + 1], sy);
    M[3 * i + 2] = mul(q.R[3 * i + 2], sz);
  }
  auto d = [&](int i, int j) {
    return add(add(mul(M[3 * i], M[3 * j]), mul(M[3 * i + 1], M[3 * j + 1])), mul(M[3 * i + 2], M[3 * j + 2]));
  };
  Cov3 S;
  S.s00 = d(0, 0); S.s01 = d(0, 1); S.s02 = d(0, 2);
  S.s11 = d(1, 1); S.s12 = d(1, 2); S.s22 = d(2, 2);
  return S;
}

// Result of projecting one pair.
struct Proj {
  float px, py, pz;   // camera-space mean
  float u, v;         // unclamped x/z, y/z
  float ux, uy;       // clamped for the Jacobian
  float T[6];         // T = J R, rows 0 and 1
  float a, b, c;      // dilated 2D covariance
  float det, mx, my, r;
  bool vis;
};

// Camera-space position only (for the cheap depth rejection).
__device__ __forceinline__ void cam_point(const Cam& k, float mx, float my, float mz, float& x, float& y, float& z) {
  x = add(add(add(mul(k.R[0], mx), mul(k.R[1], my)), mul(k.R[2], mz)), k.t[0]);
  y = add(add(add(mul(k.R[3], mx), mul(k.R[4], my)), mul(k.R[5], mz)), k.t[1]);
  z = add(add(add(mul(k.R[6], mx), mul(k.R[7], my)), mul(k.R[8], mz)), k.t[2]);
}

// Full EWA projection after the depth test passed.  vis covers det > 0 and the
// image-overlap test; the caller has checked near < z < far.
__device__ __forceinline__ void project_rest(const Cam& k, const Cov3& S, int W, int H, Proj& o) {
  float iz = rcp_(o.pz);
  o.u = mul(o.px, iz);
  o.v = mul(o.py, iz);
  o.ux = fminf(fmaxf(o.u, -k.limx), k.limx);
  o.uy = fminf(fmaxf(o.v, -k.limy), k.limy);
  float j00 = mul(k.fx, iz);
  float j02 = -mul(j00, o.ux);
  float j11 = mul(k.fy, iz);
  float j12 = -mul(j11, o.uy);
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    o.T[m] = add(mul(j00, k.R[m]), mul(j02, k.R[6 + m]));
    o.T[3 + m] = add(mul(j11, k.R[3 + m]), mul(j12, k.R[6 + m]));
  }
  const float S0[3] = {S.s00, S.s01, S.s02};
  const float S1[3] = {S.s01, S.s11, S.s12};
  const float S2[3] = {S.s02, S.s12, S.s22};
  float U0[3], U1[3];
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    U0[m] = add(add(mul(o.T[0], S0[m]), mul(o.T[1], S1[m])), mul(o.T[2], S2[m]));
    U1[m] = add(add(mul(o.T[3], S0[m]), mul(o.T[4], S1[m])), mul(o.T[5], S2[m]));
  }
  o.a = add(add(add(mul(U0[0], o.T[0]), mul(U0[1], o.T[1])), mul(U0[2], o.T[2])), 0.3f);
  o.b = add(add(mul(U0[0], o.T[3]), mul(U0[1], o.T[4])), mul(U0[2], o.T[5]));
  o.c = add(add(add(mul(U1[0], o.T[3]), mul(U1[1], o.T[4])), mul(U1[2], o.T[5])), 0.3f);
  o.det = sub(mul(o.a, o.c), mul(o.b, o.b));
  o.mx = add(mul(k.fx, o.u), k.cx);
  o.my = add(mul(k.fy, o.v), k.cy);
  float mid = mul(0.5f, add(o.a, o.c));
  float disc = fmaxf(sub(mul(mid, mid), o.det), 0.0f);
  float lam = add(mid, sqrt_(disc));
  o.r = mul(3.0f, sqrt_(lam));
  const float Wf = (float)W, Hf = (float)H;
  o.vis = (o.det > 0.0f) && (add(o.mx, o.r) > 0.0f) && (sub(o.mx, o.r) < Wf) && (add(o.my, o.r) > 0.0f) &&
          (sub(o.my, o.r) < Hf);
}

// ---------------------------------------------------------------------------
// Real spherical harmonics, degree <= 3 (degree-major, m = -l..l; real form of
// the Condon-Shortley-phased complex harmonics).
#define SS_SH_C0 0.28209479177387814f
#define SS_SH_C1 0.4886025119029199f
#define SS_SH_C2A 1.0925484305920792f
#define SS_SH_C2C 0.31539156525252005f
#define SS_SH_C2E 0.5462742152960396f
#define SS_SH_C3A 0.5900435899266435f
#define SS_SH_C3B 2.890611442640554f
#define SS_SH_C3C 0.4570457994644658f
#define SS_SH_C3D 0.3731763325901154f
#define SS_SH_C3F 1.445305721320277f

__device__ __forceinline__ void sh_basis(int deg, float X, float Y, float Z, float* b) {
  b[0] = SS_SH_C0;
  if (deg < 1) return;
  b[1] = mul(-SS_SH_C1, Y);
  b[2] = mul(SS_SH_C1, Z);
  b[3] = mul(-SS_SH_C1, X);
  if (deg < 2) return;
  float XX = mul(X, X), YY = mul(Y, Y), ZZ = mul(Z, Z), XY = mul(X, Y), YZ = mul(Y, Z), XZ = mul(X, Z);
  b[4] = mul(SS_SH_C2A, XY);
  b[5] = mul(-SS_SH_C2A, YZ);
  b[6] = mul(SS_SH_C2C, sub(sub(mul(2.0f, ZZ), XX), YY));
  b[7] = mul(-SS_SH_C2A, XZ);
  b[8] = mul(SS_SH_C2E, sub(XX, YY));
  if (deg < 3) return;
  b[9] = mul(-SS_SH_C3A, mul(Y, sub(mul(3.0f, XX), YY)));
  b[10] = mul(SS_SH_C3B, mul(XY, Z));
  b[11] = mul(-SS_SH_C3C, mul(Y, sub(sub(mul(4.0f, ZZ), XX), YY)));
  b[12] = mul(SS_SH_C3D, mul(Z, sub(sub(mul(2.0f, ZZ), mul(3.0f, XX)), mul(3.0f, YY))));
  b[13] = mul(-SS_SH_C3C, mul(X, sub(sub(mul(4.0f, ZZ), XX), YY)));
  b[14] = mul(SS_SH_C3F, mul(Z, sub(XX, YY)));
  b[15] = mul(-SS_SH_C3A, mul(X, sub(XX, mul(3.0f, YY))));
}

// Unit view direction from the camera centre to the mean.
__device__ __forceinline__ void view_dir(const Cam& k, float mx, float my, float mz, float& X, float& Y, float& Z,
                                         float& il) {
  float d0 = sub(mx, k.cpos[0]), d1 = sub(my, k.cpos[1]), d2 = sub(mz, k.cpos[2]);
  float l2 = add(add(mul(d0, d0), mul(d1, d1)), mul(d2, d2));
  il = rcp_(sqrt_(l2));
  X = mul(d0, il); Y = mul(d1, il); Z = mul(d2, il);
}

// ---------------------------------------------------------------------------
// exp(x) for x <= 0: Cody-Waite reduction with ln2 split into a 16-bit head and
// a tail, degree-7 Taylor polynomial of e^r in Horner form, 2^k from exponent
// bits.  Below -87 the result is 0 (far under the 1/255 threshold).
__device__ __forceinline__ float exp_neg(float x) {
  if (x < -87.0f) return 0.0f;
  float kf = rintf(mul(x, 0x1.715476p+0f));
  float r = fma_(kf, -0x1.62e4p-1f, x);
  r = fma_(kf, -0x1.7f7d1cp-20f, r);
  float p = 0x1.a01a02p-13f;
  p = fma_(p, r, 0x1.6c16c2p-10f);
  p = fma_(p, r, 0x1.111112p-7f);
  p = fma_(p, r, 0x1.555556p-5f);
  p = fma_(p, r, 0x1.555556p-3f);
  p = fma_(p, r, 0.5f);
  p = fma_(p, r, 1.0f);
  p = fma_(p, r, 1.0f);
  int ki = (int)kf;
  return mul(p, __int_as_float((ki + 127) << 23));
}

// sigma = 1/2 d^T conic d, canonical order; ha = 0.5*ca, hc = 0.5*cc.
__device__ __forceinline__ float gauss_sigma(float ha, float cb, float hc, float dx, float dy) {
  float s = mul(mul(cb, dx), dy);
  s = fma_(mul(hc, dy), dy, s);
  return fma_(mul(ha, dx), dx, s);
}

// Rasterizer thresholds.
#define SS_ALPHA_MAX 0.99f
#define SS_T_STOP 1e-4f
// sigma beyond which o*exp(-sigma) < 1/255 for every o <= 1 (exp(-5.6) =
// 0.0037 < 1/255 = 0.0039): lets the kernels skip the exp, same decision.
#define SS_SIGMA_SKIP 5.6f

__device__ __forceinline__ float alpha_min() { return div_(1.0f, 255.0f); }

// 16-bit edges: floor/ceil of v*65535/extent in fp64 (exact decisions).
__device__ __forceinline__ uint32_t q16_floor(float v, int extent) {
  double t = floor(__ddiv_rn(__dmul_rn((double)v, 65535.0), (double)extent));
  t = fmin(65535.0, fmax(0.0, t));
  return (uint32_t)t;
}
__device__ __forceinline__ uint32_t q16_ceil(float v, int extent) {
  double t = ceil(__ddiv_rn(__dmul_rn((double)v, 65535.0), (double)extent));
  t = fmin(65535.0, fmax(0.0, t));
  return (uint32_t)t;
}

// Tile range [t0, t1) of a decoded 16-bit edge pair (integers only).
__device__ __forceinline__ void tile_span(uint32_t q0, uint32_t q1, int extent, int ntiles, int& t0, int& t1) {
  constexpr uint32_t kDen = 65535u * 16u;
  int64_t a, b;
  if (extent <= 65535) {
    // q * extent < 2^32: the same quotients in 32-bit arithmetic
    const uint32_t x0 = q0 * (uint32_t)extent, x1 = q1 * (uint32_t)extent;
    a = x0 / kDen;
    b = x1 / kDen + (x1 % kDen != 0u ? 1 : 0);
  } else {
    a = ((int64_t)q0 * extent) / kDen;
    b = ((int64_t)q1 * extent + kDen - 1) / kDen;
  }
  t0 = (int)min64(max64(a, 0), ntiles);
  t1 = (int)min64(max64(b, 0), ntiles);
}

}  // namespace ss
