// CPU oracle for the packed 3D Gaussian Splatting forward+backward step.
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and
// bench.py's cpu_baseline / reference legs load this library.  It shares no
// code, header, table or constant with the CUDA path: every formula below is
// written from the method's definition (the plainest standard EWA-splatting
// reading, see the "Canonical arithmetic" section of the design notes).
//
// Sources (all on the "Spirula Studio" pages):
//   * packed projection, bitmask compaction, 16-bit AABB, 64-bit counts:
//     "Spirula Studio VRAM deep-dive", sections "bitmask compaction",
//     "16-bit packed AABB", "4 GiB rule and 2^31 limit";
//   * rasterizer state kept for the backward pass, the backward chain
//     (raster bwd -> projection bwd, six attribute gradients):
//     "Spirula Studio backward pass", sections 4 and 5.
//
// Precision.  The forward is computed in fp32 following the canonical
// operation order (every +,-,*,/,sqrt rounded once, fma only where written,
// built with -ffp-contract=off), because the integer outputs (mask, AABB16,
// keys, last_id) are decided by float comparisons and must be decided in the
// kernel's precision.  Gradients are computed in fp64 on top of the fp32
// decisions.  Every routine is also instantiated in fp64 end to end so that
// the backward can be checked against central finite differences.
//
// Style: plain loops, one item at a time.  OpenMP only splits independent
// items (pairs, pixels, Gaussians); every reduction is serial.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {
typedef struct {
  int32_t C, W, H, sh_degree;
  int64_t N;
  float near_plane, far_plane;
} orc_dims;
}

namespace {

constexpr int64_t kPairsPerBlock = 128;  // pairs per workgroup popcount
constexpr int kTile = 16;                // tile edge in pixels
constexpr int kRow = 12;                 // floats per screen row (48 bytes, 16-byte vectors)

void set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// ---------------------------------------------------------------------------
// exp.  fp32: Cody-Waite reduction x = k*ln2 + r (ln2 split into a 16-bit head
// and a tail), degree-7 Taylor polynomial of e^r in Horner form with fma,
// scaling by 2^k built from exponent bits.  Used for x <= 0 only.
// fp64: the library exp (the finite-difference instantiation).
float exp_fp32(float x) {
  if (x < -87.0f) return 0.0f;
  const float log2e = 0x1.715476p+0f;
  const float ln2_hi = 0x1.62e4p-1f;
  const float ln2_lo = 0x1.7f7d1cp-20f;
  float kf = std::rint(x * log2e);
  float r = std::fma(kf, -ln2_hi, x);
  r = std::fma(kf, -ln2_lo, r);
  float p = 0x1.a01a02p-13f;        // 1/7!
  p = std::fma(p, r, 0x1.6c16c2p-10f);  // 1/6!
  p = std::fma(p, r, 0x1.111112p-7f);   // 1/5!
  p = std::fma(p, r, 0x1.555556p-5f);   // 1/4!
  p = std::fma(p, r, 0x1.555556p-3f);   // 1/3!
  p = std::fma(p, r, 0.5f);             // 1/2!
  p = std::fma(p, r, 1.0f);
  p = std::fma(p, r, 1.0f);
  int ki = (int)kf;
  uint32_t bits = (uint32_t)(ki + 127) << 23;
  float s;
  std::memcpy(&s, &bits, 4);
  return p * s;
}
inline float expR(float x) { return exp_fp32(x); }
inline double expR(double x) { return std::exp(x); }

// ---------------------------------------------------------------------------
// Real spherical harmonics up to degree 3, ordered by degree l then m=-l..l,
// with the Condon-Shortley phase kept in the real form (m<0: sqrt2*Im Y_l^|m|,
// m>0: sqrt2*Re Y_l^m).  Constants from their closed forms.
struct ShConst {
  double c0, c1, c2[5], c3[7];
  ShConst() {
    const double pi = 3.14159265358979323846;
    c0 = 0.5 * std::sqrt(1.0 / pi);
    c1 = std::sqrt(3.0 / (4.0 * pi));
    c2[0] = 0.5 * std::sqrt(15.0 / pi);
    c2[1] = -0.5 * std::sqrt(15.0 / pi);
    c2[2] = 0.25 * std::sqrt(5.0 / pi);
    c2[3] = -0.5 * std::sqrt(15.0 / pi);
    c2[4] = 0.25 * std::sqrt(15.0 / pi);
    c3[0] = -0.25 * std::sqrt(35.0 / (2.0 * pi));
    c3[1] = 0.5 * std::sqrt(105.0 / pi);
    c3[2] = -0.25 * std::sqrt(21.0 / (2.0 * pi));
    c3[3] = 0.25 * std::sqrt(7.0 / pi);
    c3[4] = -0.25 * std::sqrt(21.0 / (2.0 * pi));
    c3[5] = 0.25 * std::sqrt(105.0 / pi);
    c3[6] = -0.25 * std::sqrt(35.0 / (2.0 * pi));
  }
};
const ShConst kSh;

// Basis values Y[0..K) at unit direction (X,Y,Z).
template <typename R>
void sh_basis(int degree, R X, R Y, R Z, R* b) {
  b[0] = R(kSh.c0);
  if (degree < 1) return;
  b[1] = R(-kSh.c1) * Y;
  b[2] = R(kSh.c1) * Z;
  b[3] = R(-kSh.c1) * X;
  if (degree < 2) return;
  R XX = X * X, YY = Y * Y, ZZ = Z * Z, XY = X * Y, YZ = Y * Z, XZ = X * Z;
  b[4] = R(kSh.c2[0]) * XY;
  b[5] = R(kSh.c2[1]) * YZ;
  b[6] = R(kSh.c2[2]) * ((R(2) * ZZ - XX) - YY);
  b[7] = R(kSh.c2[3]) * XZ;
  b[8] = R(kSh.c2[4]) * (XX - YY);
  if (degree < 3) return;
  b[9] = R(kSh.c3[0]) * (Y * (R(3) * XX - YY));
  b[10] = R(kSh.c3[1]) * (XY * Z);
  b[11] = R(kSh.c3[2]) * (Y * ((R(4) * ZZ - XX) - YY));
  b[12] = R(kSh.c3[3]) * (Z * ((R(2) * ZZ - R(3) * XX) - R(3) * YY));
  b[13] = R(kSh.c3[4]) * (X * ((R(4) * ZZ - XX) - YY));
  b[14] = R(kSh.c3[5]) * (Z * (XX - YY));
  b[15] = R(kSh.c3[6]) * (X * (XX - R(3) * YY));
}

// d b_k / d(X,Y,Z) treating X, Y, Z as independent (fp64 only).
void sh_basis_grad(int degree, double X, double Y, double Z, double (*g)[3]) {
  for (int k = 0; k < 16; ++k) g[k][0] = g[k][1] = g[k][2] = 0.0;
  if (degree < 1) return;
  g[1][1] = -kSh.c1;
  g[2][2] = kSh.c1;
  g[3][0] = -kSh.c1;
  if (degree < 2) return;
  const double* c2 = kSh.c2;
  g[4][0] = c2[0] * Y; g[4][1] = c2[0] * X;
  g[5][1] = c2[1] * Z; g[5][2] = c2[1] * Y;
  g[6][0] = -2.0 * c2[2] * X; g[6][1] = -2.0 * c2[2] * Y; g[6][2] = 4.0 * c2[2] * Z;
  g[7][0] = c2[3] * Z; g[7][2] = c2[3] * X;
  g[8][0] = 2.0 * c2[4] * X; g[8][1] = -2.0 * c2[4] * Y;
  if (degree < 3) return;
  const double* c3 = kSh.c3;
  double XX = X * X, YY = Y * Y, ZZ = Z * Z;
  g[9][0] = c3[0] * 6.0 * X * Y; g[9][1] = c3[0] * (3.0 * XX - 3.0 * YY);
  g[10][0] = c3[1] * Y * Z; g[10][1] = c3[1] * X * Z; g[10][2] = c3[1] * X * Y;
  g[11][0] = -2.0 * c3[2] * X * Y; g[11][1] = c3[2] * (4.0 * ZZ - XX - 3.0 * YY); g[11][2] = 8.0 * c3[2] * Y * Z;
  g[12][0] = -6.0 * c3[3] * X * Z; g[12][1] = -6.0 * c3[3] * Y * Z; g[12][2] = c3[3] * (6.0 * ZZ - 3.0 * XX - 3.0 * YY);
  g[13][0] = c3[4] * (4.0 * ZZ - 3.0 * XX - YY); g[13][1] = -2.0 * c3[4] * X * Y; g[13][2] = 8.0 * c3[4] * X * Z;
  g[14][0] = 2.0 * c3[5] * X * Z; g[14][1] = -2.0 * c3[5] * Y * Z; g[14][2] = c3[5] * (XX - YY);
  g[15][0] = c3[6] * (3.0 * XX - 3.0 * YY); g[15][1] = -6.0 * c3[6] * X * Y;
}

// ---------------------------------------------------------------------------
// Camera: world-to-camera rotation R and translation t (OpenCV axes), pinhole
// intrinsics, the off-axis limits of the EWA Jacobian and the camera centre.
template <typename R>
struct Camera {
  R Rm[9], t[3], fx, fy, cx, cy, limx, limy, cpos[3];
};

template <typename R>
Camera<R> make_camera(const double* c20, int W, int H) {
  Camera<R> k;
  for (int i = 0; i < 3; ++i) {
    for (int j = 0; j < 3; ++j) k.Rm[3 * i + j] = R(c20[4 * i + j]);
    k.t[i] = R(c20[4 * i + 3]);
  }
  k.fx = R(c20[16]); k.fy = R(c20[17]); k.cx = R(c20[18]); k.cy = R(c20[19]);
  k.limx = R(1.3) * ((R(0.5) * R(W)) / k.fx);
  k.limy = R(1.3) * ((R(0.5) * R(H)) / k.fy);
  for (int j = 0; j < 3; ++j)
    k.cpos[j] = -((k.Rm[j] * k.t[0] + k.Rm[3 + j] * k.t[1]) + k.Rm[6 + j] * k.t[2]);
  return k;
}

// Gaussian: normalised quaternion, its rotation matrix, M = R_q diag(s) and
// the 3D covariance Sigma = M M^T (upper triangle S00 S01 S02 S11 S12 S22).
template <typename R>
struct Gauss {
  R mu[3], q[4], inv, Rq[9], s[3], M[9], S[6], o;
};

template <typename R>
Gauss<R> make_gauss(const double* mu, const double* q, const double* s, double o) {
  Gauss<R> g;
  for (int i = 0; i < 3; ++i) { g.mu[i] = R(mu[i]); g.s[i] = R(s[i]); }
  g.o = R(o);
  R qw = R(q[0]), qx = R(q[1]), qy = R(q[2]), qz = R(q[3]);
  R n2 = ((qw * qw + qx * qx) + qy * qy) + qz * qz;
  g.inv = R(1) / std::sqrt(n2);
  R w = qw * g.inv, x = qx * g.inv, y = qy * g.inv, z = qz * g.inv;
  g.q[0] = w; g.q[1] = x; g.q[2] = y; g.q[3] = z;
  R xx = x * x, yy = y * y, zz = z * z, xy = x * y, xz = x * z, yz = y * z;
  R wx = w * x, wy = w * y, wz = w * z;
  R* Q = g.Rq;
  Q[0] = R(1) - R(2) * (yy + zz); Q[1] = R(2) * (xy - wz);        Q[2] = R(2) * (xz + wy);
  Q[3] = R(2) * (xy + wz);        Q[4] = R(1) - R(2) * (xx + zz); Q[5] = R(2) * (yz - wx);
  Q[6] = R(2) * (xz - wy);        Q[7] = R(2) * (yz + wx);        Q[8] = R(1) - R(2) * (xx + yy);
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) g.M[3 * i + j] = Q[3 * i + j] * g.s[j];
  const R* M = g.M;
  auto dot = [&](int i, int j) { return (M[3 * i] * M[3 * j] + M[3 * i + 1] * M[3 * j + 1]) + M[3 * i + 2] * M[3 * j + 2]; };
  g.S[0] = dot(0, 0); g.S[1] = dot(0, 1); g.S[2] = dot(0, 2);
  g.S[3] = dot(1, 1); g.S[4] = dot(1, 2); g.S[5] = dot(2, 2);
  return g;
}

template <typename R>
inline R sym(const R* S, int i, int j) {
  static const int idx[3][3] = {{0, 1, 2}, {1, 3, 4}, {2, 4, 5}};
  return S[idx[i][j]];
}

// One (camera, Gaussian) pair through the EWA projection.
template <typename R>
struct Pair {
  bool vis;
  R p[3], iz, u, v, ux, uy;
  bool clx, cly;
  R j00, j02, j11, j12, T[6], a, b, c, det, mx, my, r, x0, x1, y0, y1;
};

template <typename R>
void project_pair(const Camera<R>& k, const Gauss<R>& g, int W, int H, R nearp, R farp, Pair<R>& o) {
  // Every intermediate is computed; visibility is the conjunction at the end
  // (each comparison is false for NaN, so NaN pairs are never visible).
  for (int i = 0; i < 3; ++i)
    o.p[i] = ((k.Rm[3 * i] * g.mu[0] + k.Rm[3 * i + 1] * g.mu[1]) + k.Rm[3 * i + 2] * g.mu[2]) + k.t[i];
  R z = o.p[2];
  bool in_depth = (nearp < z) && (z < farp);
  o.iz = R(1) / z;
  o.u = o.p[0] * o.iz;
  o.v = o.p[1] * o.iz;
  o.ux = std::fmin(std::fmax(o.u, -k.limx), k.limx);
  o.uy = std::fmin(std::fmax(o.v, -k.limy), k.limy);
  o.clx = (o.u < -k.limx) || (o.u > k.limx);
  o.cly = (o.v < -k.limy) || (o.v > k.limy);
  o.j00 = k.fx * o.iz;
  o.j02 = -(o.j00 * o.ux);
  o.j11 = k.fy * o.iz;
  o.j12 = -(o.j11 * o.uy);
  // T = J R (rows 0 and 1)
  for (int m = 0; m < 3; ++m) {
    o.T[m] = o.j00 * k.Rm[m] + o.j02 * k.Rm[6 + m];
    o.T[3 + m] = o.j11 * k.Rm[3 + m] + o.j12 * k.Rm[6 + m];
  }
  const R* T = o.T;
  R U0[3], U1[3];
  for (int m = 0; m < 3; ++m) {
    U0[m] = (T[0] * sym(g.S, 0, m) + T[1] * sym(g.S, 1, m)) + T[2] * sym(g.S, 2, m);
    U1[m] = (T[3] * sym(g.S, 0, m) + T[4] * sym(g.S, 1, m)) + T[5] * sym(g.S, 2, m);
  }
  o.a = ((U0[0] * T[0] + U0[1] * T[1]) + U0[2] * T[2]) + R(0.3);
  o.b = (U0[0] * T[3] + U0[1] * T[4]) + U0[2] * T[5];
  o.c = ((U1[0] * T[3] + U1[1] * T[4]) + U1[2] * T[5]) + R(0.3);
  o.det = o.a * o.c - o.b * o.b;
  o.mx = k.fx * o.u + k.cx;
  o.my = k.fy * o.v + k.cy;
  R mid = R(0.5) * (o.a + o.c);
  R disc = std::fmax(mid * mid - o.det, R(0));
  R lam = mid + std::sqrt(disc);
  o.r = R(3) * std::sqrt(lam);
  R Wf = R(W), Hf = R(H);
  o.x0 = std::fmax(o.mx - o.r, R(0));
  o.x1 = std::fmin(o.mx + o.r, Wf);
  o.y0 = std::fmax(o.my - o.r, R(0));
  o.y1 = std::fmin(o.my + o.r, Hf);
  o.vis = in_depth && (o.det > R(0)) && (o.mx + o.r > R(0)) && (o.mx - o.r < Wf) && (o.my + o.r > R(0)) &&
          (o.my - o.r < Hf);
}

// View-dependent colour; clamped[ch] records where max(.,0) cut the value.
template <typename R>
void sh_colour(const Camera<R>& k, const Gauss<R>& g, int degree, const double* sh, R* rgb, bool* clamped, R* dir_out) {
  int K = (degree + 1) * (degree + 1);
  R b[16];
  R X = R(0), Y = R(0), Z = R(0);
  if (degree > 0) {
    R d0 = g.mu[0] - k.cpos[0], d1 = g.mu[1] - k.cpos[1], d2 = g.mu[2] - k.cpos[2];
    R l2 = (d0 * d0 + d1 * d1) + d2 * d2;
    R il = R(1) / std::sqrt(l2);
    X = d0 * il; Y = d1 * il; Z = d2 * il;
  }
  if (dir_out) { dir_out[0] = X; dir_out[1] = Y; dir_out[2] = Z; }
  sh_basis<R>(degree, X, Y, Z, b);
  for (int ch = 0; ch < 3; ++ch) {
    R acc = R(sh[ch]) * b[0];
    for (int kk = 1; kk < K; ++kk) acc = acc + R(sh[3 * kk + ch]) * b[kk];
    R v = acc + R(0.5);
    clamped[ch] = !(v >= R(0));
    rgb[ch] = std::fmax(v, R(0));
  }
}

// 16-bit quantisation of a box edge on the uniform grid step = extent/65535,
// min edge floored and max edge ceiled, computed in fp64.
uint32_t q16_floor(double v, int extent) {
  double t = std::floor((double)v * 65535.0 / (double)extent);
  return (uint32_t)std::min(65535.0, std::max(0.0, t));
}
uint32_t q16_ceil(double v, int extent) {
  double t = std::ceil((double)v * 65535.0 / (double)extent);
  return (uint32_t)std::min(65535.0, std::max(0.0, t));
}

// Tile range [t0, t1) covered by the decoded edge pair (q0, q1), integers only.
void tile_range(uint32_t q0, uint32_t q1, int extent, int ntiles, int64_t* t0, int64_t* t1) {
  const int64_t den = 65535LL * kTile;
  int64_t a = ((int64_t)q0 * extent) / den;
  int64_t b = ((int64_t)q1 * extent + den - 1) / den;
  *t0 = std::min<int64_t>(std::max<int64_t>(a, 0), ntiles);
  *t1 = std::min<int64_t>(std::max<int64_t>(b, 0), ntiles);
}

// The definition the range form must agree with: tile t is hit iff it overlaps
// the decoded box, i.e. 16t < x1_dec and 16t+16 > x0_dec (exact integers).
bool tile_hit(int64_t t, uint32_t q0, uint32_t q1, int extent) {
  int64_t lo = (int64_t)kTile * t * 65535LL, hi = (int64_t)kTile * (t + 1) * 65535LL;
  return lo < (int64_t)q1 * extent && hi > (int64_t)q0 * extent;
}

struct Geo {
  int tiles_x, tiles_y;
  int64_t tiles_per_cam, n_pad, words_per_cam, blocks_per_cam;
};
Geo geometry(const orc_dims* d) {
  Geo g;
  g.tiles_x = (d->W + kTile - 1) / kTile;
  g.tiles_y = (d->H + kTile - 1) / kTile;
  g.tiles_per_cam = (int64_t)g.tiles_x * g.tiles_y;
  g.n_pad = round_up(d->N, kPairsPerBlock);
  g.words_per_cam = g.n_pad / 32;
  g.blocks_per_cam = g.n_pad / kPairsPerBlock;
  return g;
}

// Screen row: x, y, conic a, b, c, opacity, r, g, b, depth, 0, 0.
template <typename R>
struct Row {
  R x, y, ca, cb, cc, o, rgb[3], depth;
};
template <typename R>
Row<R> load_row(const double* s) {
  Row<R> r;
  r.x = R(s[0]); r.y = R(s[1]); r.ca = R(s[2]); r.cb = R(s[3]); r.cc = R(s[4]); r.o = R(s[5]);
  r.rgb[0] = R(s[6]); r.rgb[1] = R(s[7]); r.rgb[2] = R(s[8]);
  r.depth = R(s[9]);
  return r;
}

inline float fmaR(float a, float b, float c) { return std::fma(a, b, c); }
inline double fmaR(double a, double b, double c) { return std::fma(a, b, c); }

// sigma = 1/2 d^T conic d with d = mean - pixel centre, in the canonical order.
template <typename R>
inline R gauss_sigma(const Row<R>& g, R dx, R dy) {
  R ha = R(0.5) * g.ca, hc = R(0.5) * g.cc;
  R s = (g.cb * dx) * dy;
  s = fmaR(hc * dy, dy, s);
  return fmaR(ha * dx, dx, s);
}

struct Contrib {
  int64_t idx;
  bool clamped;
};

// Front-to-back compositing of one pixel over its tile list.  Records the
// composited entries when `list` is given.
//
// Optional extensions (the "depth and T outputs, background blend" row): with
// depth_out the pixel's expected depth D = sum_i w_i * depth_i is returned,
// accumulated with the same weights w_i = alpha_i * T_i as the colour; with
// bg (the camera's background colour) the returned colour is C + T * bg.
template <typename R>
void composite_pixel(const double* screen, const uint32_t* vals, int64_t beg, int64_t end, R px, R py,
                     R* rgb_out, R* T_out, int64_t* last_out, std::vector<Contrib>* list,
                     int64_t* n_eval = nullptr, int64_t* n_comp = nullptr, R* depth_out = nullptr,
                     const double* bg = nullptr) {
  R T = R(1), Cc[3] = {R(0), R(0), R(0)}, D = R(0);
  int64_t last = -1;
  const R alpha_min = R(1) / R(255);
  for (int64_t i = beg; i < end; ++i) {
    if (n_eval) ++*n_eval;
    Row<R> g = load_row<R>(screen + (int64_t)vals[i] * kRow);
    R dx = g.x - px, dy = g.y - py;
    R sig = gauss_sigma(g, dx, dy);
    if (sig < R(0)) continue;
    R e = expR(-sig);
    R oe = g.o * e;
    R alpha = std::fmin(R(0.99), oe);
    if (alpha < alpha_min) continue;
    R Tn = T * (R(1) - alpha);
    if (Tn < R(1e-4)) break;
    R w = alpha * T;
    for (int ch = 0; ch < 3; ++ch) Cc[ch] = fmaR(g.rgb[ch], w, Cc[ch]);
    D = fmaR(g.depth, w, D);
    T = Tn;
    last = i;
    if (n_comp) ++*n_comp;
    if (list) list->push_back({i, !(oe < R(0.99))});
  }
  for (int ch = 0; ch < 3; ++ch) rgb_out[ch] = bg ? fmaR(T, R(bg[ch]), Cc[ch]) : Cc[ch];
  *T_out = T;
  *last_out = last;
  if (depth_out) *depth_out = D;
}

// Gradient of one pixel (fp64) given the composited list decided in the
// forward precision.  Accumulates into v_screen rows (fp64, 12 per row).
// With the extensions: gD = dL/dD for the expected depth (the depth is a
// fourth "channel" composited with the same weights, so it enters dL/dalpha
// like a colour and adds w_i * gD to the row's depth gradient), and bg adds
// sum_ch g_ch * bg_ch to dL/dT_final (img = C + T_final * bg).
void pixel_backward(const double* screen, const uint32_t* vals, const std::vector<Contrib>& list, double px,
                    double py, const double* g, double vT, double* v_screen, double gD = 0.0,
                    const double* bg = nullptr) {
  if (bg) vT += g[0] * bg[0] + g[1] * bg[1] + g[2] * bg[2];
  size_t n = list.size();
  std::vector<double> alpha(n), e(n), T(n + 1);
  T[0] = 1.0;
  for (size_t j = 0; j < n; ++j) {
    Row<double> gr = load_row<double>(screen + (int64_t)vals[list[j].idx] * kRow);
    double dx = gr.x - px, dy = gr.y - py;
    double sig = 0.5 * (gr.ca * dx * dx + gr.cc * dy * dy) + gr.cb * dx * dy;
    e[j] = std::exp(-sig);
    alpha[j] = list[j].clamped ? 0.99 : gr.o * e[j];
    T[j + 1] = T[j] * (1.0 - alpha[j]);
  }
  double Tfin = T[n];
  double S[3] = {0.0, 0.0, 0.0}, Sd = 0.0;
  for (size_t jj = n; jj-- > 0;) {
    int64_t row = vals[list[jj].idx];
    Row<double> gr = load_row<double>(screen + row * kRow);
    double dx = gr.x - px, dy = gr.y - py;
    double a = alpha[jj], Ti = T[jj];
    double* vr = v_screen + row * kRow;
    double v_alpha = 0.0;
    for (int ch = 0; ch < 3; ++ch) {
      vr[6 + ch] += a * Ti * g[ch];
      v_alpha += g[ch] * (gr.rgb[ch] * Ti - S[ch] / (1.0 - a));
    }
    vr[9] += a * Ti * gD;
    v_alpha += gD * (gr.depth * Ti - Sd / (1.0 - a));
    v_alpha -= vT * Tfin / (1.0 - a);
    for (int ch = 0; ch < 3; ++ch) S[ch] += gr.rgb[ch] * a * Ti;
    Sd += gr.depth * a * Ti;
    if (list[jj].clamped) continue;
    double v_o = e[jj] * v_alpha;
    double v_sig = -gr.o * e[jj] * v_alpha;
    vr[5] += v_o;
    vr[2] += v_sig * 0.5 * dx * dx;
    vr[3] += v_sig * dx * dy;
    vr[4] += v_sig * 0.5 * dy * dy;
    vr[0] += v_sig * (gr.ca * dx + gr.cb * dy);
    vr[1] += v_sig * (gr.cb * dx + gr.cc * dy);
  }
}

// Decisions of the forward projection that gate gradients.
struct Gates {
  bool clx, cly, rgb_clamped[3];
};

// Chain rule of one visible pair (fp64): screen-row gradient -> Gaussian.
void pair_backward(const Camera<double>& k, const Gauss<double>& g, const Pair<double>& P, const Gates& gate,
                   int degree, const double* sh, const double* vrow, double* v_mu, double* v_q, double* v_s,
                   double* v_o, double* v_sh) {
  const double vmx = vrow[0], vmy = vrow[1], vca = vrow[2], vcb = vrow[3], vcc = vrow[4];
  const double a = P.a, b = P.b, c = P.c, det = P.det, det2 = det * det;
  // conic (ca, cb, cc) = (c, -b, a) / det  ->  dilated 2D covariance (a, b, c)
  double va = (-vca * c * c + vcb * b * c - vcc * b * b) / det2;
  double vb = (2.0 * vca * b * c - vcb * (a * c + b * b) + 2.0 * vcc * a * b) / det2;
  double vc = (-vca * b * b + vcb * a * b - vcc * a * a) / det2;
  // Sigma2 = T Sigma T^T: dL/dT = 2 V2 T Sigma, dL/dSigma = T^T V2 T
  double V2[2][2] = {{va, 0.5 * vb}, {0.5 * vb, vc}};
  const double* T = P.T;
  double TS[2][3];
  for (int i = 0; i < 2; ++i)
    for (int m = 0; m < 3; ++m) {
      double acc = 0.0;
      for (int l = 0; l < 3; ++l) acc += T[3 * i + l] * sym(g.S, l, m);
      TS[i][m] = acc;
    }
  double GT[2][3];
  for (int i = 0; i < 2; ++i)
    for (int m = 0; m < 3; ++m) GT[i][m] = 2.0 * (V2[i][0] * TS[0][m] + V2[i][1] * TS[1][m]);
  double GS[3][3];
  for (int l = 0; l < 3; ++l)
    for (int m = 0; m < 3; ++m) {
      double acc = 0.0;
      for (int i = 0; i < 2; ++i)
        for (int j = 0; j < 2; ++j) acc += T[3 * i + l] * V2[i][j] * T[3 * j + m];
      GS[l][m] = acc;
    }
  // T = J R: dL/dJ = dL/dT R^T
  auto GJ = [&](int i, int m) {
    double acc = 0.0;
    for (int l = 0; l < 3; ++l) acc += GT[i][l] * k.Rm[3 * m + l];
    return acc;
  };
  double gj00 = GJ(0, 0), gj02 = GJ(0, 2), gj11 = GJ(1, 1), gj12 = GJ(1, 2);
  const double z = P.p[2], iz = 1.0 / z, iz2 = iz * iz;
  double gx = 0.0, gy = 0.0, gz = 0.0;
  gz += -k.fx * iz2 * gj00 + k.fx * P.ux * iz2 * gj02 - k.fy * iz2 * gj11 + k.fy * P.uy * iz2 * gj12;
  double gux = -k.fx * iz * gj02, guy = -k.fy * iz * gj12;
  if (!gate.clx) { gx += gux * iz; gz += -gux * P.p[0] * iz2; }
  if (!gate.cly) { gy += guy * iz; gz += -guy * P.p[1] * iz2; }
  gx += vmx * k.fx * iz; gz += -vmx * k.fx * P.p[0] * iz2;
  gy += vmy * k.fy * iz; gz += -vmy * k.fy * P.p[1] * iz2;
  gz += vrow[9];
  for (int j = 0; j < 3; ++j) v_mu[j] += k.Rm[j] * gx + k.Rm[3 + j] * gy + k.Rm[6 + j] * gz;
  // Sigma = M M^T: dL/dM = 2 GS M;  M = R_q diag(s)
  double GRq[9];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) {
      double gm = 2.0 * (GS[i][0] * g.M[j] + GS[i][1] * g.M[3 + j] + GS[i][2] * g.M[6 + j]);
      v_s[j] += gm * g.Rq[3 * i + j];
      GRq[3 * i + j] = gm * g.s[j];
    }
  const double w = g.q[0], x = g.q[1], y = g.q[2], zq = g.q[3];
  double vw = 0, vx = 0, vy = 0, vz = 0;
  vy += -4.0 * y * GRq[0]; vz += -4.0 * zq * GRq[0];
  vw += -2.0 * zq * GRq[1]; vx += 2.0 * y * GRq[1]; vy += 2.0 * x * GRq[1]; vz += -2.0 * w * GRq[1];
  vw += 2.0 * y * GRq[2]; vx += 2.0 * zq * GRq[2]; vy += 2.0 * w * GRq[2]; vz += 2.0 * x * GRq[2];
  vw += 2.0 * zq * GRq[3]; vx += 2.0 * y * GRq[3]; vy += 2.0 * x * GRq[3]; vz += 2.0 * w * GRq[3];
  vx += -4.0 * x * GRq[4]; vz += -4.0 * zq * GRq[4];
  vw += -2.0 * x * GRq[5]; vx += -2.0 * w * GRq[5]; vy += 2.0 * zq * GRq[5]; vz += 2.0 * y * GRq[5];
  vw += -2.0 * y * GRq[6]; vx += 2.0 * zq * GRq[6]; vy += -2.0 * w * GRq[6]; vz += 2.0 * x * GRq[6];
  vw += 2.0 * x * GRq[7]; vx += 2.0 * w * GRq[7]; vy += 2.0 * zq * GRq[7]; vz += 2.0 * y * GRq[7];
  vx += -4.0 * x * GRq[8]; vy += -4.0 * y * GRq[8];
  double dotq = w * vw + x * vx + y * vy + zq * vz;
  v_q[0] += (vw - w * dotq) * g.inv;
  v_q[1] += (vx - x * dotq) * g.inv;
  v_q[2] += (vy - y * dotq) * g.inv;
  v_q[3] += (vz - zq * dotq) * g.inv;
  *v_o += vrow[5];
  // colour
  int K = (degree + 1) * (degree + 1);
  double rgb[3], dir[3];
  bool dummy[3];
  sh_colour<double>(k, g, degree, sh, rgb, dummy, dir);
  double bas[16], bg[16][3];
  sh_basis<double>(degree, dir[0], dir[1], dir[2], bas);
  sh_basis_grad(degree, dir[0], dir[1], dir[2], bg);
  double vdir[3] = {0, 0, 0};
  for (int ch = 0; ch < 3; ++ch) {
    if (gate.rgb_clamped[ch]) continue;
    double vr = vrow[6 + ch];
    for (int kk = 0; kk < K; ++kk) {
      v_sh[3 * kk + ch] += bas[kk] * vr;
      for (int l = 0; l < 3; ++l) vdir[l] += vr * sh[3 * kk + ch] * bg[kk][l];
    }
  }
  if (degree > 0) {
    double d[3] = {g.mu[0] - k.cpos[0], g.mu[1] - k.cpos[1], g.mu[2] - k.cpos[2]};
    double il = 1.0 / std::sqrt(d[0] * d[0] + d[1] * d[1] + d[2] * d[2]);
    double dd = dir[0] * vdir[0] + dir[1] * vdir[1] + dir[2] * vdir[2];
    for (int l = 0; l < 3; ++l) v_mu[l] += (vdir[l] - dir[l] * dd) * il;
  }
}

// Gradient gates as decided in precision F.
template <typename F>
Gates decide_gates(const double* cam20, const orc_dims* d, const double* mu, const double* q, const double* s,
                   double o, const double* sh) {
  Camera<F> k = make_camera<F>(cam20, d->W, d->H);
  Gauss<F> g = make_gauss<F>(mu, q, s, o);
  Pair<F> P;
  project_pair<F>(k, g, d->W, d->H, F(d->near_plane), F(d->far_plane), P);
  Gates gt;
  gt.clx = P.clx; gt.cly = P.cly;
  F rgb[3];
  sh_colour<F>(k, g, d->sh_degree, sh, rgb, gt.rgb_clamped, nullptr);
  return gt;
}

// Order of opacities for the visible cap: the IEEE total order of the fp32
// value (for the activated opacities in (0, 1) this is the numeric order).
uint32_t opacity_order_key(double o) {
  float f = (float)o;
  uint32_t b;
  std::memcpy(&b, &f, 4);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Per-image visible cap ("Spirula Studio VRAM deep-dive", practical guide:
// --cap-max, the per-image visible splat cap that holds down nnz).  The page
// gives no selection rule; reading: in each camera whose visible pairs
// exceed cap_max, keep the cap_max of highest opacity, ties going to the
// lower Gaussian index, and drop the others.  Written as a plain
// sort-and-truncate of each camera's visible list.
void apply_visible_cap(std::vector<uint8_t>& vis, const double* opac, int64_t C, int64_t N, int64_t cap_max) {
  if (cap_max < 0) return;
  std::vector<int64_t> list;
  for (int64_t c = 0; c < C; ++c) {
    list.clear();
    for (int64_t n = 0; n < N; ++n)
      if (vis[c * N + n]) list.push_back(n);
    if ((int64_t)list.size() <= cap_max) continue;
    std::stable_sort(list.begin(), list.end(), [&](int64_t a, int64_t b) {
      return opacity_order_key(opac[a]) > opacity_order_key(opac[b]);
    });
    for (size_t k = (size_t)cap_max; k < list.size(); ++k) vis[c * N + list[k]] = 0;
  }
}

}  // namespace

// ===========================================================================
extern "C" {

// Exposed for the pins: the fp32 exp and the SH basis.
float orc_exp_fp32(float x) { return exp_fp32(x); }
void orc_exp_fp32_vec(const float* x, float* y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = exp_fp32(x[i]);
}
void orc_sh_basis_f64(int degree, double X, double Y, double Z, double* out) {
  sh_basis<double>(degree, X, Y, Z, out);
}
void orc_sh_basis_grad_f64(int degree, double X, double Y, double Z, double* out48) {
  double g[16][3];
  sh_basis_grad(degree, X, Y, Z, g);
  std::memcpy(out48, g, sizeof(g));
}
void orc_geometry(const orc_dims* d, int64_t* out) {
  Geo g = geometry(d);
  out[0] = g.tiles_x; out[1] = g.tiles_y; out[2] = g.tiles_per_cam; out[3] = g.n_pad;
  out[4] = g.words_per_cam; out[5] = g.blocks_per_cam;
}

// Packed projection.  Visibility is decided per pair; rows are numbered in
// camera-major pair order.  Two independent compactions are computed and
// compared: (a) the plain one, a per-pair 0/1 flag and its running count; (b)
// the bitmask one, bit (c*n_pad + n) of mask, one popcount per 128-pair block,
// an exclusive scan of the block counts and the set bits before the pair.
// Returns 0, or -1 if (a) and (b) disagree, or -2 if cap_rows is too small
// (nnz_out is still exact).  precision: 0 = fp32 decisions and values (inputs
// must then be fp32-representable), 1 = fp64 throughout.  Screen rows are
// stored in fp64: x, y, conic a, b, c, opacity, r, g, b, depth, 0, 0.
// cap_max < 0: no visible cap.
int orc_project(const orc_dims* d, const double* cams, const double* means, const double* quats,
                const double* scales, const double* opac, const double* sh, int precision, uint32_t* mask,
                uint32_t* block_count, int64_t* block_off, int64_t* nnz_out, double* screen, uint32_t* aabb,
                int32_t* row_cam, int64_t* row_gauss, uint8_t* rgb_clamped, int64_t cap_rows, int nthreads,
                int64_t cap_max) {
  set_threads(nthreads);
  const int64_t N = d->N, C = d->C;
  const int K = (d->sh_degree + 1) * (d->sh_degree + 1);
  Geo geo = geometry(d);
  std::vector<uint8_t> vis((size_t)(C * N));
#pragma omp parallel for schedule(dynamic, 4096)
  for (int64_t i = 0; i < C * N; ++i) {
    int64_t c = i / N, n = i % N;
    bool v;
    if (precision == 0) {
      Camera<float> k = make_camera<float>(cams + 20 * c, d->W, d->H);
      Gauss<float> g = make_gauss<float>(means + 3 * n, quats + 4 * n, scales + 3 * n, opac[n]);
      Pair<float> P;
      project_pair<float>(k, g, d->W, d->H, d->near_plane, d->far_plane, P);
      v = P.vis;
    } else {
      Camera<double> k = make_camera<double>(cams + 20 * c, d->W, d->H);
      Gauss<double> g = make_gauss<double>(means + 3 * n, quats + 4 * n, scales + 3 * n, opac[n]);
      Pair<double> P;
      project_pair<double>(k, g, d->W, d->H, d->near_plane, d->far_plane, P);
      v = P.vis;
    }
    vis[i] = v ? 1 : 0;
  }
  apply_visible_cap(vis, opac, C, N, cap_max);
  // (a) plain compaction
  std::vector<int64_t> slot_a((size_t)(C * N));
  int64_t run = 0;
  for (int64_t i = 0; i < C * N; ++i) { slot_a[i] = run; run += vis[i]; }
  const int64_t nnz = run;
  // (b) bitmask compaction
  const int64_t words = C * geo.words_per_cam, blocks = C * geo.blocks_per_cam;
  for (int64_t w = 0; w < words; ++w) mask[w] = 0;
  for (int64_t c = 0; c < C; ++c)
    for (int64_t n = 0; n < N; ++n)
      if (vis[c * N + n]) {
        int64_t bit = c * geo.n_pad + n;
        mask[bit >> 5] |= 1u << (bit & 31);
      }
  for (int64_t b = 0; b < blocks; ++b) {
    uint32_t cnt = 0;
    for (int w = 0; w < 4; ++w) cnt += (uint32_t)__builtin_popcount(mask[4 * b + w]);
    block_count[b] = cnt;
  }
  block_off[0] = 0;
  for (int64_t b = 0; b < blocks; ++b) block_off[b + 1] = block_off[b] + block_count[b];
  if (block_off[blocks] != nnz) return -1;
  int bad = 0;
#pragma omp parallel for reduction(| : bad)
  for (int64_t c = 0; c < C; ++c)
    for (int64_t n = 0; n < N; ++n) {
      if (!vis[c * N + n]) continue;
      int64_t bit = c * geo.n_pad + n, b = bit / kPairsPerBlock, w = bit >> 5;
      int64_t slot = block_off[b];
      for (int64_t ww = 4 * b; ww < w; ++ww) slot += __builtin_popcount(mask[ww]);
      slot += __builtin_popcount(mask[w] & ((1u << (bit & 31)) - 1u));
      if (slot != slot_a[c * N + n]) bad = 1;
    }
  if (bad) return -1;
  *nnz_out = nnz;
  if (!screen) return 0;
  if (nnz > cap_rows) return -2;
#pragma omp parallel for schedule(dynamic, 4096)
  for (int64_t i = 0; i < C * N; ++i) {
    if (!vis[i]) continue;
    int64_t c = i / N, n = i % N, row = slot_a[i];
    double* out = screen + row * kRow;
    bool clamped[3];
    double x0, x1, y0, y1;
    float depth32;
    if (precision == 0) {
      Camera<float> k = make_camera<float>(cams + 20 * c, d->W, d->H);
      Gauss<float> g = make_gauss<float>(means + 3 * n, quats + 4 * n, scales + 3 * n, opac[n]);
      Pair<float> P;
      project_pair<float>(k, g, d->W, d->H, d->near_plane, d->far_plane, P);
      float idet = 1.0f / P.det;
      float rgb[3];
      sh_colour<float>(k, g, d->sh_degree, sh + (int64_t)K * 3 * n, rgb, clamped, nullptr);
      float v[10] = {P.mx, P.my, P.c * idet, -(P.b * idet), P.a * idet, g.o, rgb[0], rgb[1], rgb[2], P.p[2]};
      for (int q = 0; q < 10; ++q) out[q] = v[q];
      x0 = P.x0; x1 = P.x1; y0 = P.y0; y1 = P.y1;
      depth32 = P.p[2];
    } else {
      Camera<double> k = make_camera<double>(cams + 20 * c, d->W, d->H);
      Gauss<double> g = make_gauss<double>(means + 3 * n, quats + 4 * n, scales + 3 * n, opac[n]);
      Pair<double> P;
      project_pair<double>(k, g, d->W, d->H, d->near_plane, d->far_plane, P);
      double idet = 1.0 / P.det;
      double rgb[3];
      sh_colour<double>(k, g, d->sh_degree, sh + (int64_t)K * 3 * n, rgb, clamped, nullptr);
      double v[10] = {P.mx, P.my, P.c * idet, -(P.b * idet), P.a * idet, g.o, rgb[0], rgb[1], rgb[2], P.p[2]};
      for (int q = 0; q < 10; ++q) out[q] = v[q];
      x0 = P.x0; x1 = P.x1; y0 = P.y0; y1 = P.y1;
      depth32 = (float)P.p[2];
    }
    out[10] = 0.0;
    out[11] = 0.0;
    (void)depth32;
    if (aabb) {
      aabb[2 * row] = q16_floor(x0, d->W) | (q16_floor(y0, d->H) << 16);
      aabb[2 * row + 1] = q16_ceil(x1, d->W) | (q16_ceil(y1, d->H) << 16);
    }
    if (row_cam) row_cam[row] = (int32_t)c;
    if (row_gauss) row_gauss[row] = n;
    if (rgb_clamped)
      for (int ch = 0; ch < 3; ++ch) rgb_clamped[3 * row + ch] = clamped[ch];
  }
  return 0;
}

// Float box of each row in fp32 (for the AABB containment pin).
int orc_row_boxes(const orc_dims* d, const double* cams, const double* means, const double* quats,
                  const double* scales, const double* opac, const int32_t* row_cam, const int64_t* row_gauss,
                  int64_t nnz, float* box4) {
  for (int64_t r = 0; r < nnz; ++r) {
    int64_t c = row_cam[r], n = row_gauss[r];
    Camera<float> k = make_camera<float>(cams + 20 * c, d->W, d->H);
    Gauss<float> g = make_gauss<float>(means + 3 * n, quats + 4 * n, scales + 3 * n, opac[n]);
    Pair<float> P;
    project_pair<float>(k, g, d->W, d->H, d->near_plane, d->far_plane, P);
    if (!P.vis) return -1;
    box4[4 * r] = P.x0; box4[4 * r + 1] = P.x1; box4[4 * r + 2] = P.y0; box4[4 * r + 3] = P.y1;
  }
  return 0;
}

// Number of tiles each row covers (range form), and the exact 64-bit total.
int orc_count_tiles(const orc_dims* d, const uint32_t* aabb, int64_t nnz, int64_t* per_row, uint64_t* total) {
  Geo geo = geometry(d);
  uint64_t tot = 0;
  for (int64_t r = 0; r < nnz; ++r) {
    int64_t tx0, tx1, ty0, ty1;
    tile_range(aabb[2 * r] & 0xFFFFu, aabb[2 * r + 1] & 0xFFFFu, d->W, geo.tiles_x, &tx0, &tx1);
    tile_range(aabb[2 * r] >> 16, aabb[2 * r + 1] >> 16, d->H, geo.tiles_y, &ty0, &ty1);
    int64_t cnt = (tx1 - tx0) * (ty1 - ty0);
    if (per_row) per_row[r] = cnt;
    tot += (uint64_t)cnt;
  }
  *total = tot;
  return 0;
}

// Intersections: for each row and each candidate tile of its camera, the
// overlap test of the decoded box; the range form must give the same set.
// When all_pairs != 0 every tile of the camera is tested, otherwise every tile
// in the float-box window widened by one tile (the decoded box exceeds the
// float box by less than one quantisation step).  Writes (key, row) in
// row-major order over (row, ty, tx).  Returns 0, -1 on a disagreement, -2 if
// the capacity is short (the total is still exact).
// Intersection keys.  Rows are visited in order of their depth (the IEEE bits
// of the fp32 camera-space depth, ties by row index), each row's tiles
// row-major over (ty, tx); order_out (nullable) receives the visiting order.
// Write order is a layout choice (the keys themselves are the page's); with
// the rows in depth order, a stable sort by tile id alone yields the key order.
int orc_intersect(const orc_dims* d, const double* screen, const uint32_t* aabb, const int32_t* row_cam, int64_t nnz,
                  int all_pairs, uint64_t* keys, uint32_t* vals, int64_t cap, uint64_t* total_out, int64_t* order_out) {
  Geo geo = geometry(d);
  std::vector<int64_t> per_row((size_t)nnz);
  uint64_t total = 0;
  orc_count_tiles(d, aabb, nnz, per_row.data(), &total);
  *total_out = total;
  if ((int64_t)total > cap) return -2;
  std::vector<uint32_t> dbits_of((size_t)nnz);
  for (int64_t r = 0; r < nnz; ++r) {
    float depth32 = (float)screen[r * kRow + 9];
    std::memcpy(&dbits_of[r], &depth32, 4);
  }
  std::vector<int64_t> order((size_t)nnz);
  for (int64_t r = 0; r < nnz; ++r) order[r] = r;
  std::stable_sort(order.begin(), order.end(), [&](int64_t a, int64_t b) { return dbits_of[a] < dbits_of[b]; });
  if (order_out)
    for (int64_t p = 0; p < nnz; ++p) order_out[p] = order[p];
  std::vector<int64_t> off((size_t)nnz + 1);
  off[0] = 0;
  for (int64_t p = 0; p < nnz; ++p) off[p + 1] = off[p] + per_row[order[p]];
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 256) reduction(| : bad)
  for (int64_t p = 0; p < nnz; ++p) {
    const int64_t r = order[p];
    uint32_t qx0 = aabb[2 * r] & 0xFFFFu, qx1 = aabb[2 * r + 1] & 0xFFFFu;
    uint32_t qy0 = aabb[2 * r] >> 16, qy1 = aabb[2 * r + 1] >> 16;
    int64_t tx0, tx1, ty0, ty1;
    tile_range(qx0, qx1, d->W, geo.tiles_x, &tx0, &tx1);
    tile_range(qy0, qy1, d->H, geo.tiles_y, &ty0, &ty1);
    int64_t wx0 = 0, wx1 = geo.tiles_x, wy0 = 0, wy1 = geo.tiles_y;
    if (!all_pairs) {
      // window from the decoded box's float neighbourhood, one tile of slack
      double fx0 = qx0 * (double)d->W / 65535.0, fx1 = qx1 * (double)d->W / 65535.0;
      double fy0 = qy0 * (double)d->H / 65535.0, fy1 = qy1 * (double)d->H / 65535.0;
      wx0 = std::max<int64_t>(0, (int64_t)std::floor(fx0 / kTile) - 1);
      wx1 = std::min<int64_t>(geo.tiles_x, (int64_t)std::ceil(fx1 / kTile) + 1);
      wy0 = std::max<int64_t>(0, (int64_t)std::floor(fy0 / kTile) - 1);
      wy1 = std::min<int64_t>(geo.tiles_y, (int64_t)std::ceil(fy1 / kTile) + 1);
    }
    int64_t w = off[p];
    // key low word: IEEE bits of the fp32 camera-space depth
    const uint32_t dbits = dbits_of[r];
    const uint64_t cam_base = (uint64_t)row_cam[r] * (uint64_t)geo.tiles_per_cam;
    int64_t found = 0;
    for (int64_t ty = wy0; ty < wy1; ++ty) {
      bool hy = tile_hit(ty, qy0, qy1, d->H);
      for (int64_t tx = wx0; tx < wx1; ++tx) {
        bool hit = hy && tile_hit(tx, qx0, qx1, d->W);
        bool in_range = (tx >= tx0 && tx < tx1 && ty >= ty0 && ty < ty1);
        if (hit != in_range) bad = 1;
        if (!hit) continue;
        uint64_t tile = cam_base + (uint64_t)ty * geo.tiles_x + (uint64_t)tx;
        keys[w] = (tile << 32) | dbits;
        vals[w] = (uint32_t)r;
        ++w;
        ++found;
      }
    }
    if (found != per_row[r]) bad = 1;
  }
  return bad ? -1 : 0;
}

// Stable sort of (key, value) by key.
int orc_sort(uint64_t* keys, uint32_t* vals, int64_t n) {
  std::vector<int64_t> perm((size_t)n);
  for (int64_t i = 0; i < n; ++i) perm[i] = i;
  std::stable_sort(perm.begin(), perm.end(), [&](int64_t a, int64_t b) { return keys[a] < keys[b]; });
  std::vector<uint64_t> k2((size_t)n);
  std::vector<uint32_t> v2((size_t)n);
  for (int64_t i = 0; i < n; ++i) { k2[i] = keys[perm[i]]; v2[i] = vals[perm[i]]; }
  std::memcpy(keys, k2.data(), sizeof(uint64_t) * n);
  std::memcpy(vals, v2.data(), sizeof(uint32_t) * n);
  return 0;
}

// tile_off[t] = number of sorted entries whose tile id is below t.
int orc_tile_ranges(const uint64_t* keys, int64_t n, int64_t n_tiles, int64_t* tile_off) {
  std::vector<int64_t> cnt((size_t)n_tiles, 0);
  for (int64_t i = 0; i < n; ++i) {
    uint64_t t = keys[i] >> 32;
    if ((int64_t)t >= n_tiles) return -1;
    cnt[t]++;
  }
  tile_off[0] = 0;
  for (int64_t t = 0; t < n_tiles; ++t) tile_off[t + 1] = tile_off[t] + cnt[t];
  return 0;
}

// Forward rasterizer, one pixel at a time.  img [C][H][W][3], T_final and
// last_id [C][H][W].  precision 0: fp32 (canonical), 1: fp64.
// Optional evals[npix]: entries each pixel evaluated (up to and including the
// one that stopped it); comps[npix]: entries composited.
// depth (nullable): expected depth per pixel; bg (nullable): [C][3]
// background colours blended as img = C + T_final * bg.
int orc_rasterize_fwd(const orc_dims* d, const double* screen, const uint32_t* vals, const int64_t* tile_off,
                      int precision, double* img, double* T_final, int64_t* last_id, int64_t* evals,
                      int64_t* comps, int nthreads, double* depth, const double* bg) {
  set_threads(nthreads);
  Geo geo = geometry(d);
  const int64_t npix = (int64_t)d->C * d->H * d->W;
#pragma omp parallel for schedule(dynamic, 1024)
  for (int64_t p = 0; p < npix; ++p) {
    int64_t* ev = evals ? evals + p : nullptr;
    int64_t* cp = comps ? comps + p : nullptr;
    if (ev) *ev = 0;
    if (cp) *cp = 0;
    int64_t c = p / ((int64_t)d->H * d->W), rem = p % ((int64_t)d->H * d->W);
    int64_t j = rem / d->W, i = rem % d->W;
    int64_t t = c * geo.tiles_per_cam + (j / kTile) * geo.tiles_x + (i / kTile);
    int64_t last;
    const double* bgc = bg ? bg + 3 * c : nullptr;
    if (precision == 0) {
      float rgb[3], T, D;
      composite_pixel<float>(screen, vals, tile_off[t], tile_off[t + 1], (float)i + 0.5f, (float)j + 0.5f, rgb, &T,
                             &last, nullptr, ev, cp, &D, bgc);
      for (int ch = 0; ch < 3; ++ch) img[3 * p + ch] = rgb[ch];
      T_final[p] = T;
      if (depth) depth[p] = D;
    } else {
      double rgb[3], T, D;
      composite_pixel<double>(screen, vals, tile_off[t], tile_off[t + 1], (double)i + 0.5, (double)j + 0.5, rgb,
                              &T, &last, nullptr, ev, cp, &D, bgc);
      for (int ch = 0; ch < 3; ++ch) img[3 * p + ch] = rgb[ch];
      T_final[p] = T;
      if (depth) depth[p] = D;
    }
    last_id[p] = last;
  }
  return 0;
}

// Backward rasterizer: per pixel, the composited list decided in `precision`
// (0 fp32, 1 fp64), then fp64 gradients summed into v_screen[nnz][12].
// v_T may be NULL.  Pixels are visited serially (deterministic sums); with
// nthreads > 1 cameras/pixel blocks are split over per-thread fp64 buffers
// that are added in thread order.
// v_depth (nullable): dL/d(expected depth) per pixel; bg (nullable): [C][3].
int orc_rasterize_bwd(const orc_dims* d, const double* screen, const uint32_t* vals, const int64_t* tile_off,
                      const double* v_img, const double* v_T, int precision, int64_t nnz, double* v_screen,
                      int nthreads, const double* v_depth, const double* bg) {
  set_threads(nthreads);
  Geo geo = geometry(d);
  const int64_t npix = (int64_t)d->C * d->H * d->W;
  int nt = 1;
#ifdef _OPENMP
  nt = std::max(1, nthreads > 0 ? nthreads : omp_get_max_threads());
#endif
  std::vector<std::vector<double>> bufs((size_t)nt);
#pragma omp parallel num_threads(nt)
  {
    int tid = 0;
#ifdef _OPENMP
    tid = omp_get_thread_num();
#endif
    std::vector<double>& acc = bufs[tid];
    acc.assign((size_t)nnz * kRow, 0.0);
    std::vector<Contrib> list;
#pragma omp for schedule(static)
    for (int64_t p = 0; p < npix; ++p) {
      int64_t c = p / ((int64_t)d->H * d->W), rem = p % ((int64_t)d->H * d->W);
      int64_t j = rem / d->W, i = rem % d->W;
      int64_t t = c * geo.tiles_per_cam + (j / kTile) * geo.tiles_x + (i / kTile);
      list.clear();
      int64_t last;
      if (precision == 0) {
        float rgb[3], T;
        composite_pixel<float>(screen, vals, tile_off[t], tile_off[t + 1], (float)i + 0.5f, (float)j + 0.5f, rgb,
                               &T, &last, &list);
      } else {
        double rgb[3], T;
        composite_pixel<double>(screen, vals, tile_off[t], tile_off[t + 1], (double)i + 0.5, (double)j + 0.5, rgb,
                                &T, &last, &list);
      }
      double g[3] = {v_img[3 * p], v_img[3 * p + 1], v_img[3 * p + 2]};
      double vT = v_T ? v_T[p] : 0.0;
      pixel_backward(screen, vals, list, (double)i + 0.5, (double)j + 0.5, g, vT, acc.data(),
                     v_depth ? v_depth[p] : 0.0, bg ? bg + 3 * c : nullptr);
    }
  }
  for (int64_t q = 0; q < nnz * kRow; ++q) {
    double s = 0.0;
    for (int t = 0; t < nt; ++t) s += bufs[t][q];
    v_screen[q] = s;
  }
  return 0;
}

// Projection backward: v_screen rows (fp64) -> per-Gaussian gradients (fp64),
// summed over cameras.  Gates (J clamp, SH clamp) decided in `precision`.
int orc_project_bwd(const orc_dims* d, const double* cams, const double* means, const double* quats,
                    const double* scales, const double* opac, const double* sh, const int32_t* row_cam, const int64_t* row_gauss, int64_t nnz,
                    const double* v_screen, int precision, double* v_means, double* v_quats, double* v_scales,
                    double* v_opac, double* v_sh) {
  const int K = (d->sh_degree + 1) * (d->sh_degree + 1);
  for (int64_t i = 0; i < 3 * d->N; ++i) { v_means[i] = 0; v_scales[i] = 0; }
  for (int64_t i = 0; i < 4 * d->N; ++i) v_quats[i] = 0;
  for (int64_t i = 0; i < d->N; ++i) v_opac[i] = 0;
  for (int64_t i = 0; i < 3 * K * d->N; ++i) v_sh[i] = 0;
  for (int64_t r = 0; r < nnz; ++r) {
    int64_t c = row_cam[r], n = row_gauss[r];
    const double* cam = cams + 20 * c;
    const double *mu = means + 3 * n, *q = quats + 4 * n, *s = scales + 3 * n, *shn = sh + (int64_t)K * 3 * n;
    Gates gt = precision == 0 ? decide_gates<float>(cam, d, mu, q, s, opac[n], shn)
                              : decide_gates<double>(cam, d, mu, q, s, opac[n], shn);
    Camera<double> k = make_camera<double>(cam, d->W, d->H);
    Gauss<double> g = make_gauss<double>(mu, q, s, opac[n]);
    Pair<double> P;
    project_pair<double>(k, g, d->W, d->H, d->near_plane, d->far_plane, P);
    pair_backward(k, g, P, gt, d->sh_degree, shn, v_screen + r * kRow, v_means + 3 * n, v_quats + 4 * n,
                  v_scales + 3 * n, v_opac + n, v_sh + (int64_t)K * 3 * n);
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Sampled checks at full size.  These restate the same definitions for a
// chosen subset of tiles or rows, so that outputs can be compared one by one
// where the whole step is too large for the oracle.

// Exact number of entries per tile (row-major walk over every row's range).
int orc_tile_counts(const orc_dims* d, const uint32_t* aabb, const int32_t* row_cam, int64_t nnz, int64_t* counts) {
  Geo geo = geometry(d);
  const int64_t T = geo.tiles_per_cam * d->C;
  for (int64_t t = 0; t < T; ++t) counts[t] = 0;
  for (int64_t r = 0; r < nnz; ++r) {
    int64_t tx0, tx1, ty0, ty1;
    tile_range(aabb[2 * r] & 0xFFFFu, aabb[2 * r + 1] & 0xFFFFu, d->W, geo.tiles_x, &tx0, &tx1);
    tile_range(aabb[2 * r] >> 16, aabb[2 * r + 1] >> 16, d->H, geo.tiles_y, &ty0, &ty1);
    const int64_t base = (int64_t)row_cam[r] * geo.tiles_per_cam;
    for (int64_t ty = ty0; ty < ty1; ++ty)
      for (int64_t tx = tx0; tx < tx1; ++tx) counts[base + ty * geo.tiles_x + tx]++;
  }
  return 0;
}

// Sorted (key, row) lists of the selected tiles: every row whose decoded box
// overlaps the tile, ordered by key then row.  out_off[nsel+1] gives each
// selected tile's slice of out_keys/out_vals (capacity cap); returns -2 if cap
// is too small (out_off still complete).
int orc_tile_lists(const orc_dims* d, const double* screen, const uint32_t* aabb, const int32_t* row_cam,
                   int64_t nnz, const int64_t* sel, int64_t nsel, int64_t* out_off, uint64_t* out_keys,
                   uint32_t* out_vals, int64_t cap) {
  Geo geo = geometry(d);
  const int64_t T = geo.tiles_per_cam * d->C;
  std::vector<int64_t> slot((size_t)T, -1);
  for (int64_t i = 0; i < nsel; ++i) slot[sel[i]] = i;
  std::vector<std::vector<std::pair<uint64_t, uint32_t>>> lists((size_t)nsel);
  for (int64_t r = 0; r < nnz; ++r) {
    int64_t tx0, tx1, ty0, ty1;
    tile_range(aabb[2 * r] & 0xFFFFu, aabb[2 * r + 1] & 0xFFFFu, d->W, geo.tiles_x, &tx0, &tx1);
    tile_range(aabb[2 * r] >> 16, aabb[2 * r + 1] >> 16, d->H, geo.tiles_y, &ty0, &ty1);
    const int64_t base = (int64_t)row_cam[r] * geo.tiles_per_cam;
    for (int64_t ty = ty0; ty < ty1; ++ty)
      for (int64_t tx = tx0; tx < tx1; ++tx) {
        const int64_t t = base + ty * geo.tiles_x + tx;
        const int64_t s = slot[t];
        if (s < 0) continue;
        float depth32 = (float)screen[r * kRow + 9];
        uint32_t dbits;
        std::memcpy(&dbits, &depth32, 4);
        lists[s].push_back({((uint64_t)t << 32) | dbits, (uint32_t)r});
      }
  }
  out_off[0] = 0;
  for (int64_t i = 0; i < nsel; ++i) {
    std::stable_sort(lists[i].begin(), lists[i].end(),
                     [](const std::pair<uint64_t, uint32_t>& a, const std::pair<uint64_t, uint32_t>& b) {
                       return a.first < b.first;
                     });
    out_off[i + 1] = out_off[i] + (int64_t)lists[i].size();
  }
  if (out_off[nsel] > cap) return -2;
  for (int64_t i = 0; i < nsel; ++i)
    for (size_t k = 0; k < lists[i].size(); ++k) {
      out_keys[out_off[i] + k] = lists[i][k].first;
      out_vals[out_off[i] + k] = lists[i][k].second;
    }
  return 0;
}

// Forward rasterizer of the selected tiles from their lists (list i is
// vals[off[i]..off[i+1]) and starts at global sorted index start[i]).
// Outputs per selected tile: img [nsel][256][3], T [nsel][256], last [nsel][256]
// (pixels outside the image: T = 1, last = -2).
int orc_rasterize_tiles(const orc_dims* d, const double* screen, const uint32_t* vals, const int64_t* off,
                        const int64_t* sel, const int64_t* start, int64_t nsel, double* img, double* T_out,
                        int64_t* last_out, int nthreads) {
  set_threads(nthreads);
  Geo geo = geometry(d);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t q = 0; q < nsel * kTile * kTile; ++q) {
    const int64_t s = q / (kTile * kTile), pix = q % (kTile * kTile);
    const int64_t t = sel[s];
    const int64_t tr = t % geo.tiles_per_cam;
    const int64_t i = (tr % geo.tiles_x) * kTile + pix % kTile, j = (tr / geo.tiles_x) * kTile + pix / kTile;
    if (i >= d->W || j >= d->H) {
      for (int ch = 0; ch < 3; ++ch) img[3 * q + ch] = 0.0;
      T_out[q] = 1.0;
      last_out[q] = -2;
      continue;
    }
    float rgb[3], T;
    int64_t last;
    composite_pixel<float>(screen, vals, off[s], off[s + 1], (float)i + 0.5f, (float)j + 0.5f, rgb, &T, &last,
                           nullptr);
    for (int ch = 0; ch < 3; ++ch) img[3 * q + ch] = rgb[ch];
    T_out[q] = T;
    last_out[q] = last < 0 ? -1 : start[s] + (last - off[s]);
  }
  return 0;
}

// Backward rasterizer restricted to the selected rows: every pixel of the
// listed tiles (which must include all tiles those rows cover) is replayed in
// fp64 on top of its fp32 decisions, and only the selected rows' gradients are
// kept: v_rows [nrows][12].  row_slot[nnz] maps a row to its slot or -1.
int orc_raster_bwd_rows(const orc_dims* d, const double* screen, const uint32_t* vals, const int64_t* off,
                        const int64_t* sel, int64_t nsel, const double* v_img, const double* v_T,
                        const int64_t* row_slot, int64_t nrows, double* v_rows, int nthreads) {
  set_threads(nthreads);
  Geo geo = geometry(d);
  int nt = 1;
#ifdef _OPENMP
  nt = std::max(1, nthreads > 0 ? nthreads : omp_get_max_threads());
#endif
  std::vector<std::vector<double>> part((size_t)nt, std::vector<double>((size_t)nrows * kRow, 0.0));
#pragma omp parallel num_threads(nt)
  {
    int tid = 0;
#ifdef _OPENMP
    tid = omp_get_thread_num();
#endif
    std::vector<Contrib> list;
    std::vector<double> acc, lscreen;
    std::vector<uint32_t> local;
    std::vector<Contrib> ll;
#pragma omp for schedule(dynamic, 1)
    for (int64_t s = 0; s < nsel; ++s) {
      const int64_t t = sel[s];
      const int64_t c = t / geo.tiles_per_cam, tr = t % geo.tiles_per_cam;
      for (int64_t pix = 0; pix < kTile * kTile; ++pix) {
        const int64_t i = (tr % geo.tiles_x) * kTile + pix % kTile, j = (tr / geo.tiles_x) * kTile + pix / kTile;
        if (i >= d->W || j >= d->H) continue;
        float rgb[3], T;
        int64_t last;
        list.clear();
        composite_pixel<float>(screen, vals, off[s], off[s + 1], (float)i + 0.5f, (float)j + 0.5f, rgb, &T, &last,
                               &list);
        bool any = false;
        for (const Contrib& cb : list)
          if (row_slot[vals[cb.idx]] >= 0) any = true;
        if (!any) continue;
        const int64_t p = (c * d->H + j) * d->W + i;
        double g[3] = {v_img[3 * p], v_img[3 * p + 1], v_img[3 * p + 2]};
        double vT = v_T ? v_T[p] : 0.0;
        // replay this pixel's list on a local copy of its rows
        acc.assign(list.size() * kRow, 0.0);
        local.resize(list.size());
        ll.resize(list.size());
        lscreen.resize(list.size() * kRow);
        for (size_t k = 0; k < list.size(); ++k) {
          const uint32_t row = vals[list[k].idx];
          for (int q = 0; q < kRow; ++q) lscreen[k * kRow + q] = screen[(int64_t)row * kRow + q];
          local[k] = (uint32_t)k;
          ll[k] = {(int64_t)k, list[k].clamped};
        }
        pixel_backward(lscreen.data(), local.data(), ll, (double)i + 0.5, (double)j + 0.5, g, vT, acc.data());
        for (size_t k = 0; k < list.size(); ++k) {
          const int64_t sl = row_slot[vals[list[k].idx]];
          if (sl < 0) continue;
          for (int q = 0; q < kRow; ++q) part[tid][sl * kRow + q] += acc[k * kRow + q];
        }
      }
    }
  }
  for (int64_t q = 0; q < nrows * kRow; ++q) {
    double sum = 0.0;
    for (int t = 0; t < nt; ++t) sum += part[t][q];
    v_rows[q] = sum;
  }
  return 0;
}

// Projection backward of single rows: per-row gradient contributions
// [nrows][3+4+3+1+3K] (means, quats, scales, opacity, sh) in fp64, with the
// gates decided in fp32.  Summing a Gaussian's rows gives its gradient.
int orc_project_bwd_rows(const orc_dims* d, const double* cams, const double* means, const double* quats,
                         const double* scales, const double* opac, const double* sh, const int32_t* cam_of,
                         const int64_t* gauss_of, int64_t nrows, const double* v_rows, double* out) {
  const int K = (d->sh_degree + 1) * (d->sh_degree + 1);
  const int64_t w = 11 + 3 * K;
  for (int64_t q = 0; q < nrows * w; ++q) out[q] = 0.0;
  for (int64_t r = 0; r < nrows; ++r) {
    const int64_t c = cam_of[r], n = gauss_of[r];
    const double* cam = cams + 20 * c;
    const double *mu = means + 3 * n, *q = quats + 4 * n, *s = scales + 3 * n, *shn = sh + (int64_t)K * 3 * n;
    Gates gt = decide_gates<float>(cam, d, mu, q, s, opac[n], shn);
    Camera<double> k = make_camera<double>(cam, d->W, d->H);
    Gauss<double> g = make_gauss<double>(mu, q, s, opac[n]);
    Pair<double> P;
    project_pair<double>(k, g, d->W, d->H, d->near_plane, d->far_plane, P);
    double* o = out + r * w;
    pair_backward(k, g, P, gt, d->sh_degree, shn, v_rows + r * kRow, o, o + 3, o + 7, o + 10, o + 11);
  }
  return 0;
}

}  // extern "C"
