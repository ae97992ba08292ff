// Tile rasterizer, forward and backward ("Spirula Studio backward pass",
// section 4: the forward keeps tile offsets, the sorted intersection list,
// each pixel's last composited entry and its final transmittance; the backward
// reuses them without re-intersecting, splits each pixel's gradient by alpha
// contribution and sums per Gaussian with atomics).
//
// One CTA of 128 threads per 16x16 tile.  Each thread owns a vertical pair of
// pixels (same column, rows j and j+1), so the pair shares dx and the sigma and
// exp arithmetic runs on packed fp32 pairs (FFMA2/FMUL2/FADD2: each lane of the
// pair is rounded exactly like the scalar operation, so the canonical order is
// kept bit for bit).  Warp w owns the 16x4 region of rows 4w..4w+3.  Each batch
// of 256 sorted entries is gathered once into shared memory (three 16-byte
// loads per 48-byte screen row).  Per block of 32 staged entries each lane
// computes which of its warp's 64 pixels one entry can reach (outward-rounded
// ellipse chords, see entry_coverage) and a warp bit-transpose hands every
// lane the candidate entries of its own two pixels: the forward walks its own
// list, the backward steps its warp through the union of the lists (it needs
// the warp together for the gradient reduction).  The counting forward culls
// by region box (warp_culled).
#include "ss_common.cuh"
#include "ss_math.cuh"

namespace ss {

constexpr int kRThreads = 128;
constexpr int kBatch = 256;
constexpr int kRedF = 12;

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// sqrt(x) for x >= 0 through the approximate reciprocal square root (a few
// ulp); only the culling bounds use it, widened far beyond that error.
__device__ __forceinline__ float sqrt_approx(float x) { return x > 0.0f ? x * rsqrtf(x) : 0.0f; }
__device__ __forceinline__ float2 f2s(float a) { return make_float2(a, a); }

// Pixel-pair coordinates of this thread: column i, rows j and j+1.
__device__ __forceinline__ void tile_coords(const Geo& g, int64_t tile, int& c, int& tx0, int& ty0, int& i, int& j) {
  c = (int)(tile / g.tiles_per_cam);
  const int rem = (int)(tile - (int64_t)c * g.tiles_per_cam);
  const int ty = rem / g.tiles_x, tx = rem - ty * g.tiles_x;
  tx0 = tx * kTile;
  ty0 = ty * kTile;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  i = tx0 + (lane & 15);
  j = ty0 + 4 * warp + 2 * (lane >> 4);
}

// ---------------------------------------------------------------------------
// Staged entry.  thr is the entry's skip threshold: a pixel whose canonical
// sigma exceeds thr cannot reach alpha >= 1/255, so it skips the entry
// without the exp (the per-pixel definition skips it too).  For o <= 1 it is
// ln(255 o) plus a small margin, verified in the canonical arithmetic
// (o * E(-thr) < 1/255; E is monotone, so every larger sigma fails too) and
// capped at 5.6 (E(-5.6) < 1/255 holds for every o <= 1); -1 when o < 1/255
// (alpha <= o can never reach 1/255); +inf when o > 1.  The remaining fields
// bound where the entry can matter, all computed in fp32 and rounded outward:
// dql underestimates ca*cc - cb^2 (the fma error bound subtracted), so
// (hx, hy) over-cover the ellipse {sigma <= thr + kCullMargin} of the stored
// conic and the row chords below over-cover it too; +inf / "everything" when
// o > 1 or the conic is not safely positive definite.  The margin covers the
// fp32 rounding of the canonical sigma (at most 0.04 where the coverage is
// used, see warp_culled and entry_coverage).
constexpr float kCullMargin = 0.2f;

__device__ __forceinline__ float entry_threshold(float o, float amin) {
  if (!(o <= 1.0f)) return __int_as_float(0x7f800000);
  if (!(o >= amin)) return -1.0f;
  float thr = fminf(SS_SIGMA_SKIP, __logf(255.0f * o) + 2e-3f);
  if (!(mul(o, exp_neg(-thr)) < amin)) thr = SS_SIGMA_SKIP;
  return thr;
}

struct Stage {
  float4 a;  // x, y, 0.5*ca, cb
  float4 b;  // 0.5*cc, o, r, g
  float4 c;  // b, hx, hy, kterm = |ha| + |hc| + |cb|
  float4 d;  // thr, row (bits), P = 2*ca*(thr + margin), dql
  float4 e;  // 1/ca, cb/ca, bounded (1/0), depth
};

// The staged form of screen row r (r0..r2: its three 16-byte words).
__device__ __forceinline__ void stage_from(const float4 r0, const float4 r1, const float4 r2, uint32_t r, Stage& st) {
  const float ca = r0.z, cb = r0.w, cc = r1.x, o = r1.y;
  st.a = make_float4(r0.x, r0.y, mul(0.5f, ca), cb);
  st.b = make_float4(mul(0.5f, cc), o, r1.z, r1.w);
  const float inf = __int_as_float(0x7f800000);
  const float thr = entry_threshold(o, alpha_min());
  const float bb = cb * cb;
  const float dq = fmaf(ca, cc, -bb);
  const float dql = dq - 2e-7f * (bb + fabsf(dq)) - 1e-30f;
  float hx = inf, hy = inf, P = 0.0f, ica = 0.0f, cbr = 0.0f, bounded = 0.0f;
  if (thr < 0.0f) {
    // never composited: an empty box
    hx = hy = -1.0f;
    P = -1.0f;
    bounded = 1.0f;
  } else if (o <= 1.0f && ca > 0.0f && cc > 0.0f && dql > 0.0f) {
    const float L = thr + kCullMargin;
    // bounds only: the hardware's approximate root and divide (relative
    // error below 1e-6) stay inside the 1e-5 widening
    hx = sqrt_approx(__fdividef(2.0f * L * cc, dql)) * 1.00001f + 1e-3f;
    hy = sqrt_approx(__fdividef(2.0f * L * ca, dql)) * 1.00001f + 1e-3f;
    P = 2.0f * L * ca;
    ica = __fdividef(1.0f, ca);
    cbr = cb * ica;
    bounded = 1.0f;
  }
  const float kterm = 0.5f * fabsf(ca) + 0.5f * fabsf(cc) + fabsf(cb);
  st.c = make_float4(r2.x, hx, hy, kterm);
  st.d = make_float4(thr, __uint_as_float(r), P, dql);
  st.e = make_float4(ica, cbr, bounded, r2.y);
}

__device__ __forceinline__ void stage_row(const float* __restrict__ screen, uint32_t r, Stage& st) {
  const float4* row = reinterpret_cast<const float4*>(screen + (int64_t)r * kRowF);
  stage_from(row[0], row[1], row[2], r, st);
}

// Warp culling.  For an entry with o <= 1 every pixel whose computed sigma
// exceeds thr skips the entry.  A region outside the box (hx, hy) of the
// ellipse {sigma <= thr + 0.2} has exact sigma > thr + 0.2 at every pixel
// centre; when kterm*(Dx^2 + Dy^2) <= 8e4 (D: largest offset from the mean to
// the region) the canonical fp32 sigma differs from the exact one by less
// than 0.04, so every pixel of the region computes sigma > thr and would skip
// the entry: skipping it for the whole warp takes exactly the per-pixel
// decision.
__device__ __forceinline__ bool warp_culled(const Stage& st, float x_lo, float x_hi, float y_lo, float y_hi) {
  const float mx = st.a.x, my = st.a.y;
  const float ex = fmaxf(fmaxf(x_lo - mx, mx - x_hi), 0.0f);
  const float ey = fmaxf(fmaxf(y_lo - my, my - y_hi), 0.0f);
  if (!(ex > st.c.y || ey > st.c.z)) return false;
  const float Dx = fmaxf(fabsf(x_lo - mx), fabsf(x_hi - mx));
  const float Dy = fmaxf(fabsf(y_lo - my), fabsf(y_hi - my));
  return st.c.w * (Dx * Dx + Dy * Dy) <= 8e4f;
}

// sigma of the pixel pair in the canonical order (see gauss_sigma).
__device__ __forceinline__ float2 sigma_pair(const Stage& st, float dx, float2 dy) {
  const float t = mul(st.a.w, dx);                       // cb*dx
  float2 s = __fmul2_rn(f2s(t), dy);                     // (cb*dx)*dy
  s = __ffma2_rn(__fmul2_rn(f2s(st.b.x), dy), dy, s);    // fma(hc*dy, dy, s)
  const float v = mul(st.a.z, dx);                       // ha*dx
  return __ffma2_rn(f2s(v), f2s(dx), s);                 // fma(ha*dx, dx, s)
}

// exp_neg on a pair, each lane exactly as the scalar version.
__device__ __forceinline__ float2 exp_neg_pair(float2 x) {
  const float2 t = __fmul2_rn(x, f2s(0x1.715476p+0f));
  const float2 kf = f2(rintf(t.x), rintf(t.y));
  float2 r = __ffma2_rn(kf, f2s(-0x1.62e4p-1f), x);
  r = __ffma2_rn(kf, f2s(-0x1.7f7d1cp-20f), r);
  float2 p = f2s(0x1.a01a02p-13f);
  p = __ffma2_rn(p, r, f2s(0x1.6c16c2p-10f));
  p = __ffma2_rn(p, r, f2s(0x1.111112p-7f));
  p = __ffma2_rn(p, r, f2s(0x1.555556p-5f));
  p = __ffma2_rn(p, r, f2s(0x1.555556p-3f));
  p = __ffma2_rn(p, r, f2s(0.5f));
  p = __ffma2_rn(p, r, f2s(1.0f));
  p = __ffma2_rn(p, r, f2s(1.0f));
  const uint32_t ex = ((uint32_t)((int)kf.x + 127)) << 23, ey = ((uint32_t)((int)kf.y + 127)) << 23;
  float2 e = __fmul2_rn(p, f2(__uint_as_float(ex), __uint_as_float(ey)));
  if (x.x < -87.0f) e.x = 0.0f;
  if (x.y < -87.0f) e.y = 0.0f;
  return e;
}

// One pixel's front-to-back step for an entry whose sigma passed the tests;
// with EXT also the expected depth, accumulated with the colour's weight.
template <bool EXT = false>
__device__ __forceinline__ void composite(const Stage& st, float oe, float amin, int64_t idx, float& T, float& C0,
                                          float& C1, float& C2, float& D, int64_t& last, bool& done,
                                          unsigned long long& ncomp) {
  const float alpha = fminf(SS_ALPHA_MAX, oe);
  if (alpha < amin) return;
  const float Tn = mul(T, sub(1.0f, alpha));
  if (Tn < SS_T_STOP) {
    done = true;
    return;
  }
  const float w = mul(alpha, T);
  C0 = fma_(st.b.z, w, C0);
  C1 = fma_(st.b.w, w, C1);
  C2 = fma_(st.c.x, w, C2);
  if (EXT) D = fma_(st.e.w, w, D);
  T = Tn;
  last = idx;
  ++ncomp;
}

// COUNT adds work counters (measurement helper): entries evaluated per pixel
// (up to and including the stopping one), exps evaluated, entries composited,
// entries the backward replays (tile start to last_id) and exps among those.
// In COUNT mode no entry is culled, so the counts follow the per-pixel
// definition.
template <bool COUNT>
__global__ __launch_bounds__(kRThreads) void k_raster_fwd(Geo g, const float* __restrict__ screen,
                                                          const uint32_t* __restrict__ vals,
                                                          const int64_t* __restrict__ tile_off,
                                                          float* __restrict__ img, float* __restrict__ T_final,
                                                          int32_t* __restrict__ last_id,
                                                          unsigned long long* __restrict__ counts) {
  __shared__ Stage s_e[kBatch];
  const int lane = threadIdx.x & 31;
  const int64_t tile = blockIdx.x;
  int c, tx0, ty0, i, j;
  tile_coords(g, tile, c, tx0, ty0, i, j);
  const bool inA = i < g.W && j < g.H, inB = i < g.W && j + 1 < g.H;
  const float px = add((float)i, 0.5f);
  const float2 npy = f2(-add((float)j, 0.5f), -add((float)(j + 1), 0.5f));
  const float x_lo = (float)tx0 + 0.5f, x_hi = x_lo + 15.0f;
  const float y_lo = (float)(j - 2 * (lane >> 4)) + 0.5f, y_hi = y_lo + 3.0f;
  const int64_t beg = tile_off[tile], end = tile_off[tile + 1];
  const float amin = alpha_min();
  float TA = 1.0f, A0 = 0.0f, A1 = 0.0f, A2 = 0.0f, TB = 1.0f, B0 = 0.0f, B1 = 0.0f, B2 = 0.0f, DA = 0.0f,
        DB = 0.0f;
  int64_t lastA = -1, lastB = -1;
  bool doneA = !inA, doneB = !inB;
  unsigned long long n_eval = 0, n_exp = 0, n_comp = 0, n_expA_last = 0, n_expB_last = 0, n_expA = 0, n_expB = 0;
  for (int64_t b0 = beg; b0 < end; b0 += kBatch) {
    if (__syncthreads_count(doneA && doneB) == kRThreads) break;
    for (int t = threadIdx.x; t < kBatch; t += kRThreads)
      if (b0 + t < end) stage_row(screen, vals[b0 + t], s_e[t]);
    __syncthreads();
    if (__all_sync(0xffffffffu, doneA && doneB)) continue;
    const int cnt = (int)min64(kBatch, end - b0);
    for (int q = 0; q * 32 < cnt; ++q) {
      const int e = q * 32 + lane;
      uint32_t bits =
          __ballot_sync(0xffffffffu, e < cnt && (COUNT || !warp_culled(s_e[e], x_lo, x_hi, y_lo, y_hi)));
      while (bits) {
        const int k = q * 32 + __ffs(bits) - 1;
        bits &= bits - 1;
        if (doneA && doneB) continue;
        const Stage& st = s_e[k];
        if (COUNT) n_eval += (doneA ? 0 : 1) + (doneB ? 0 : 1);
        const float dx = sub(st.a.x, px);
        const float2 dy = __fadd2_rn(f2s(st.a.y), npy);
        const float2 sig = sigma_pair(st, dx, dy);
        const bool needA = !doneA && !(sig.x < 0.0f) && !(sig.x > st.d.x);
        const bool needB = !doneB && !(sig.y < 0.0f) && !(sig.y > st.d.x);
        if (!(needA || needB)) continue;
        const float2 ev = exp_neg_pair(f2(-sig.x, -sig.y));
        const float2 oe = __fmul2_rn(f2s(st.b.y), ev);
        const int64_t idx = b0 + k;
        if (needA) {
          if (COUNT) {
            ++n_exp;
            ++n_expA;
          }
          const int64_t before = lastA;
          composite(st, oe.x, amin, idx, TA, A0, A1, A2, DA, lastA, doneA, n_comp);
          if (COUNT && lastA != before) n_expA_last = n_expA;
        }
        if (needB) {
          if (COUNT) {
            ++n_exp;
            ++n_expB;
          }
          const int64_t before = lastB;
          composite(st, oe.y, amin, idx, TB, B0, B1, B2, DB, lastB, doneB, n_comp);
          if (COUNT && lastB != before) n_expB_last = n_expB;
        }
      }
      if (__all_sync(0xffffffffu, doneA && doneB)) break;
    }
  }
  const int64_t pixA = ((int64_t)c * g.H + j) * g.W + i;
  if (inA) {
    img[3 * pixA] = A0;
    img[3 * pixA + 1] = A1;
    img[3 * pixA + 2] = A2;
    T_final[pixA] = TA;
    last_id[pixA] = (int32_t)lastA;
  }
  if (inB) {
    const int64_t pixB = pixA + g.W;
    img[3 * pixB] = B0;
    img[3 * pixB + 1] = B1;
    img[3 * pixB + 2] = B2;
    T_final[pixB] = TB;
    last_id[pixB] = (int32_t)lastB;
  }
  if (COUNT) {
    const unsigned long long replay = (lastA >= 0 ? (unsigned long long)(lastA - beg + 1) : 0ull) +
                                      (lastB >= 0 ? (unsigned long long)(lastB - beg + 1) : 0ull);
    unsigned long long v[5] = {n_eval, n_exp, n_comp, replay, n_expA_last + n_expB_last};
#pragma unroll
    for (int q = 0; q < 5; ++q) {
      unsigned long long x = v[q];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      if (lane == 0 && x) atomicAdd(&counts[q], x);
    }
  }
}

// ---------------------------------------------------------------------------
// Per-pixel candidate masks.  For a block of 32 staged entries (one per lane)
// each lane computes which of the warp's 64 pixels its entry can reach: a
// pixel is left out only if its computed sigma provably exceeds the entry's
// threshold thr (exact sigma > thr + 0.2 outside the outward-rounded chord of
// the ellipse {sigma <= thr + 0.2}, and kterm*D^2 <= 8e4 bounds the fp32
// rounding of the canonical sigma by 0.04); such pixels skip the entry in the
// per-pixel definition too.  A 32x32 bit transpose across the warp then gives
// each lane the entries of the block that reach each of its two pixels.

// Lane i receives bit j = bit i of lane j's word.
template <int S, uint32_t M>
__device__ __forceinline__ uint32_t transpose_step(uint32_t x, int lane) {
  const uint32_t y = __shfl_xor_sync(0xffffffffu, x, S);
  return (lane & S) ? ((x & ~M) | ((y >> S) & M)) : ((x & M) | ((y << S) & ~M));
}

__device__ __forceinline__ uint32_t warp_transpose32(uint32_t x, int lane) {
  x = transpose_step<16, 0x0000FFFFu>(x, lane);
  x = transpose_step<8, 0x00FF00FFu>(x, lane);
  x = transpose_step<4, 0x0F0F0F0Fu>(x, lane);
  x = transpose_step<2, 0x33333333u>(x, lane);
  return transpose_step<1, 0x55555555u>(x, lane);
}

// 16-bit column mask of the pixels of row centre yc (columns x_lo + c,
// c = 0..15) inside the outward-rounded chord of {sigma <= L}, L = thr + 0.2:
// for a pixel row at offset dy the chord is centred at mx + (cb/ca)*dy with
// half-width sqrt(2*ca*L - dq*dy^2)/ca; dql <= dq and the margins make every
// fp32 rounding widen it.
__device__ __forceinline__ uint32_t chord_span(const Stage& st, float yc, float x_lo) {
  const float dy = st.a.y - yc;
  const float q = st.d.w * dy * dy;
  const float disc = st.d.z - q + 4e-7f * (st.d.z + q);
  if (disc < 0.0f) return 0u;
  if (!(disc >= 0.0f)) return 0xFFFFu;  // NaN: nothing can be concluded
  const float hw = sqrt_approx(disc) * st.e.x * 1.00001f + 2e-3f;
  const float off = st.e.y * dy;
  const float ctr = st.a.x + off;
  const float m = 1e-5f * (fabsf(st.a.x) + fabsf(off)) + 2e-3f;
  const float lo = ctr - hw - m - x_lo, hi = ctr + hw + m - x_lo;
  if (!(lo == lo && hi == hi)) return 0xFFFFu;
  if (hi < 0.0f || lo > 15.0f) return 0u;
  const int c0 = lo <= 0.0f ? 0 : (int)ceilf(lo);
  const int c1 = hi >= 15.0f ? 15 : (int)floorf(hi);
  if (c1 < c0) return 0u;
  return ((0xFFFFu >> (15 - c1)) >> c0) << c0;
}

// Coverage of this lane's entry over the warp's region: bit L of covA (covB)
// set when the entry can reach lane L's upper (lower) pixel.  A pixel left
// out has exact sigma > thr + 0.2, and kterm*D^2 <= 8e4 bounds the rounding
// of the canonical fp32 sigma by 0.04, so its computed sigma exceeds thr: it
// skips the entry in the per-pixel definition as well.
__device__ __forceinline__ void entry_coverage(const Stage& st, float x_lo, float y_lo, uint32_t& covA,
                                               uint32_t& covB) {
  const float x_hi = x_lo + 15.0f, y_hi = y_lo + 3.0f;
  const float mx = st.a.x, my = st.a.y;
  const float Dx = fmaxf(fabsf(x_lo - mx), fabsf(x_hi - mx));
  const float Dy = fmaxf(fabsf(y_lo - my), fabsf(y_hi - my));
  if (!(st.e.z > 0.0f && st.c.w * (Dx * Dx + Dy * Dy) <= 8e4f)) {
    covA = covB = 0xFFFFFFFFu;
    return;
  }
  const float ex = fmaxf(fmaxf(x_lo - mx, mx - x_hi), 0.0f);
  const float ey = fmaxf(fmaxf(y_lo - my, my - y_hi), 0.0f);
  if (ex > st.c.y || ey > st.c.z) {
    covA = covB = 0u;
    return;
  }
  const uint32_t s0 = chord_span(st, y_lo, x_lo), s1 = chord_span(st, y_lo + 1.0f, x_lo);
  const uint32_t s2 = chord_span(st, y_lo + 2.0f, x_lo), s3 = chord_span(st, y_lo + 3.0f, x_lo);
  covA = s0 | (s2 << 16);
  covB = s1 | (s3 << 16);
}

// EXT: also the expected depth (depth, nullable) and a background colour per
// camera (bg [C][3], nullable) blended as img = C + T_final * bg.
template <bool EXT>
__global__ __launch_bounds__(kRThreads) void k_raster_fwd_masked(Geo g, const float* __restrict__ screen,
                                                                 const uint32_t* __restrict__ vals,
                                                                 const int64_t* __restrict__ tile_off,
                                                                 float* __restrict__ img, float* __restrict__ T_final,
                                                                 int32_t* __restrict__ last_id,
                                                                 float* __restrict__ depth,
                                                                 const float* __restrict__ bg,
                                                                 const uint32_t* __restrict__ tile_order) {
  __shared__ Stage s_e[kBatch];
  const int lane = threadIdx.x & 31;
  const int64_t tile = tile_order ? (int64_t)tile_order[blockIdx.x] : (int64_t)blockIdx.x;
  if (tile >= g.n_tiles) return;  // not a tile index: nothing to draw
  int c, tx0, ty0, i, j;
  tile_coords(g, tile, c, tx0, ty0, i, j);
  const bool inA = i < g.W && j < g.H, inB = i < g.W && j + 1 < g.H;
  const float px = add((float)i, 0.5f);
  const float2 npy = f2(-add((float)j, 0.5f), -add((float)(j + 1), 0.5f));
  const float x_lo = (float)tx0 + 0.5f;
  const float y_lo = (float)(j - 2 * (lane >> 4)) + 0.5f;
  const int64_t beg = tile_off[tile], end = tile_off[tile + 1];
  const float amin = alpha_min();
  float TA = 1.0f, A0 = 0.0f, A1 = 0.0f, A2 = 0.0f, TB = 1.0f, B0 = 0.0f, B1 = 0.0f, B2 = 0.0f, DA = 0.0f,
        DB = 0.0f;
  int64_t lastA = -1, lastB = -1;
  bool doneA = !inA, doneB = !inB;
  unsigned long long ncomp = 0;
  for (int64_t b0 = beg; b0 < end; b0 += kBatch) {
    if (__syncthreads_count(doneA && doneB) == kRThreads) break;
    for (int t = threadIdx.x; t < kBatch; t += kRThreads)
      if (b0 + t < end) stage_row(screen, vals[b0 + t], s_e[t]);
    __syncthreads();
    if (__all_sync(0xffffffffu, doneA && doneB)) continue;
    const int cnt = (int)min64(kBatch, end - b0);
    for (int q = 0; q * 32 < cnt; ++q) {
      const int e = q * 32 + lane;
      uint32_t covA = 0u, covB = 0u;
      if (e < cnt) entry_coverage(s_e[e], x_lo, y_lo, covA, covB);
      uint32_t mA = warp_transpose32(covA, lane), mB = warp_transpose32(covB, lane);
      if (doneA) mA = 0u;
      if (doneB) mB = 0u;
      uint32_t m = mA | mB;
      while (m) {
        const int b = __ffs(m) - 1;
        m &= m - 1;
        const bool cA = !doneA && ((mA >> b) & 1u), cB = !doneB && ((mB >> b) & 1u);
        if (!(cA || cB)) continue;
        const int k = q * 32 + b;
        const Stage& st = s_e[k];
        const float dx = sub(st.a.x, px);
        const float2 dy = __fadd2_rn(f2s(st.a.y), npy);
        const float2 sig = sigma_pair(st, dx, dy);
        const bool needA = cA && !(sig.x < 0.0f) && !(sig.x > st.d.x);
        const bool needB = cB && !(sig.y < 0.0f) && !(sig.y > st.d.x);
        if (!(needA || needB)) continue;
        const float2 ev = exp_neg_pair(f2(-sig.x, -sig.y));
        const float2 oe = __fmul2_rn(f2s(st.b.y), ev);
        const int64_t idx = b0 + k;
        if (needA) composite<EXT>(st, oe.x, amin, idx, TA, A0, A1, A2, DA, lastA, doneA, ncomp);
        if (needB) composite<EXT>(st, oe.y, amin, idx, TB, B0, B1, B2, DB, lastB, doneB, ncomp);
      }
      if (__all_sync(0xffffffffu, doneA && doneB)) break;
    }
  }
  const int64_t pixA = ((int64_t)c * g.H + j) * g.W + i;
  if (EXT && bg) {
    const float b0 = bg[3 * c], b1 = bg[3 * c + 1], b2 = bg[3 * c + 2];
    A0 = fma_(TA, b0, A0);
    A1 = fma_(TA, b1, A1);
    A2 = fma_(TA, b2, A2);
    B0 = fma_(TB, b0, B0);
    B1 = fma_(TB, b1, B1);
    B2 = fma_(TB, b2, B2);
  }
  if (inA) {
    img[3 * pixA] = A0;
    img[3 * pixA + 1] = A1;
    img[3 * pixA + 2] = A2;
    T_final[pixA] = TA;
    last_id[pixA] = (int32_t)lastA;
    if (EXT && depth) depth[pixA] = DA;
  }
  if (inB) {
    const int64_t pixB = pixA + g.W;
    img[3 * pixB] = B0;
    img[3 * pixB + 1] = B1;
    img[3 * pixB + 2] = B2;
    T_final[pixB] = TB;
    last_id[pixB] = (int32_t)lastB;
    if (EXT && depth) depth[pixB] = DB;
  }
}

// Reduce-scatter of 8 values over a warp in 9 shuffles: afterwards lane L
// holds the warp sum of value ((L>>4)&1)*4 + ((L>>3)&1)*2 + ((L>>2)&1).
__device__ __forceinline__ float warp_reduce8(float* a, int lane) {
  bool up = lane & 16;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float send = up ? a[q] : a[q + 4];
    const float keep = up ? a[q + 4] : a[q];
    a[q] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
  up = lane & 8;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const float send = up ? a[q] : a[q + 2];
    const float keep = up ? a[q + 2] : a[q];
    a[q] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  up = lane & 4;
  {
    const float send = up ? a[0] : a[1];
    const float keep = up ? a[1] : a[0];
    a[0] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  a[0] += __shfl_xor_sync(0xffffffffu, a[0], 2);
  a[0] += __shfl_xor_sync(0xffffffffu, a[0], 1);
  return a[0];
}

// Two entries' eight sums reduced together: the exchange across lane bit 4
// leaves the first entry's partial sums in lanes 0-15 and the second's in
// lanes 16-31, and each half finishes as warp_reduce8 does over lane bits
// 3..1.  Lane l returns value 4*b3 + 2*b2 + b1 of entry b4 (bn: bit n of
// l), in 16 shuffles where two single reductions take 18.
__device__ __forceinline__ float warp_reduce8x2(float* a, const float* b, int lane) {
  bool up = lane & 16;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float send = up ? a[q] : b[q];
    const float keep = up ? b[q] : a[q];
    a[q] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
  up = lane & 8;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float send = up ? a[q] : a[q + 4];
    const float keep = up ? a[q + 4] : a[q];
    a[q] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  up = lane & 4;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const float send = up ? a[q] : a[q + 2];
    const float keep = up ? a[q + 2] : a[q];
    a[q] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  up = lane & 2;
  {
    const float send = up ? a[0] : a[1];
    const float keep = up ? a[1] : a[0];
    a[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  a[0] += __shfl_xor_sync(0xffffffffu, a[0], 1);
  return a[0];
}

// Warp sums of (a0, a1) for one entry and (b0, b1) for another: lane l
// returns value b3 of entry b4 (value 0: a0 or b0, value 1: a1 or b1).
// With `two` false only value 0 is reduced (lanes 0-15: a0, 16-31: b0).
template <bool two>
__device__ __forceinline__ float warp_sum_x2(float a0, float a1, float b0, float b1, int lane) {
  bool up = lane & 16;
  float v = (up ? b0 : a0) + __shfl_xor_sync(0xffffffffu, up ? a0 : b0, 16);
  if (two) {
    const float v1 = (up ? b1 : a1) + __shfl_xor_sync(0xffffffffu, up ? a1 : b1, 16);
    up = lane & 8;
    v = (up ? v1 : v) + __shfl_xor_sync(0xffffffffu, up ? v : v1, 8);
  } else {
    v += __shfl_xor_sync(0xffffffffu, v, 8);
  }
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Per-pixel backward state.
struct PixB {
  float T, Sg, g0, g1, g2, vTT, gD;  // gD: dL/d(expected depth), 0 unless requested
  int64_t last;
};

// Entries [qb, qb + 32) that a pixel with last composited entry `last`
// replays: bit b set when qb + b <= last.
__device__ __forceinline__ uint32_t live_bits(int64_t last, int64_t qb) {
  if (last < qb) return 0u;
  const int64_t d = last - qb;
  return d >= 31 ? 0xFFFFFFFFu : (2u << (int)d) - 1u;
}

// exp(x) of a pair through the hardware's fast exponential (relative error
// about 1e-6 on the sigma range the replay evaluates); see pair_grad for
// where the canonical E takes over.
__device__ __forceinline__ float2 exp_fast_pair(float2 x) { return f2(__expf(x.x), __expf(x.y)); }

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Reverse step of the thread's pixel pair for a replayed entry.  cA / cB say
// which pixels replay the entry with sigma within the skip threshold.  A
// pixel that does not take the entry (alpha < 1/255, the forward's decision
// in the same canonical arithmetic) gets alpha 0 below: ra = 1 and w = 0 keep
// its state.  Writes the pair's summed contribution to gr[0..8] (x, y, ca, cb,
// cc, o, r, g, b) and returns whether any pixel contributed.  The conic and
// mean terms are summed over the pair before the entry's coefficients
// multiply them: with v = dL/dsigma per pixel,
//   dL/dx = ca*dx*S0 + cb*S1,  dL/dy = cb*dx*S0 + cc*S1,
//   dL/dca = dx^2*S0/2,  dL/dcb = dx*S1,  dL/dcc = S2/2,
// where S0 = sum v, S1 = sum v*dy, S2 = sum v*dy^2 (dx is shared).
//
// The exponential comes from the fast hardware path; only the two decisions
// the forward took on it must come out the same (alpha >= 1/255, and
// whether o*E reached the 0.99 clamp), so wherever o*exp lies within 1e-5
// (relative) of either threshold, ten times the fast path's error, the pair
// is recomputed with the canonical E.  Elsewhere alpha and the recovered
// transmittance (an approximate reciprocal) differ from the forward's by a
// few ulps, which moves the gradients by about 1e-6 relative.
//
// EXT: the expected depth is a fourth channel composited with the same
// weights, so depth * gD joins the colour term of dL/dalpha and
// gr[9] = sum w * gD is the row's depth gradient.
template <bool EXT>
__device__ __forceinline__ bool pair_grad(const Stage& st, float dx, float2 dy, float2 sig, bool cA, bool cB,
                                          float amin, PixB& pa, PixB& pb, float* gr) {
  float2 ev = exp_fast_pair(f2(-sig.x, -sig.y));
  float2 oe = __fmul2_rn(f2s(st.b.y), ev);
  const bool nearA = fabsf(oe.x - amin) <= 1e-5f * amin || fabsf(oe.x - SS_ALPHA_MAX) <= 1e-5f;
  const bool nearB = fabsf(oe.y - amin) <= 1e-5f * amin || fabsf(oe.y - SS_ALPHA_MAX) <= 1e-5f;
  if ((cA && nearA) || (cB && nearB)) {
    ev = exp_neg_pair(f2(-sig.x, -sig.y));
    oe = __fmul2_rn(f2s(st.b.y), ev);
  }
  cA = cA && !(fminf(SS_ALPHA_MAX, oe.x) < amin);
  cB = cB && !(fminf(SS_ALPHA_MAX, oe.y) < amin);
  if (!(cA || cB)) return false;
  const float2 a = f2(cA ? fminf(SS_ALPHA_MAX, oe.x) : 0.0f, cB ? fminf(SS_ALPHA_MAX, oe.y) : 0.0f);
  const float2 ra = f2(rcp_approx(1.0f - a.x), rcp_approx(1.0f - a.y));
  const float2 Ti = __fmul2_rn(f2(pa.T, pb.T), ra);  // transmittance in front of the entry
  const float2 w = __fmul2_rn(a, Ti);
  const float2 G0 = f2(pa.g0, pb.g0), G1 = f2(pa.g1, pb.g1), G2 = f2(pa.g2, pb.g2);
  float2 rgbg = __fmul2_rn(f2s(st.b.z), G0);
  rgbg = __ffma2_rn(f2s(st.b.w), G1, rgbg);
  rgbg = __ffma2_rn(f2s(st.c.x), G2, rgbg);
  if (EXT) rgbg = __ffma2_rn(f2s(st.e.w), f2(pa.gD, pb.gD), rgbg);
  const float2 Sg = f2(pa.Sg, pb.Sg);
  const float2 behind = __fadd2_rn(Sg, f2(pa.vTT, pb.vTT));
  const float2 va = __ffma2_rn(Ti, rgbg, __fmul2_rn(f2(-ra.x, -ra.y), behind));  // dL/dalpha
  const float2 Sg1 = __ffma2_rn(w, rgbg, Sg);
  pa.Sg = Sg1.x;
  pb.Sg = Sg1.y;
  pa.T = Ti.x;
  pb.T = Ti.y;
  const float2 w0 = __fmul2_rn(w, G0), w1 = __fmul2_rn(w, G1), w2 = __fmul2_rn(w, G2);
  gr[6] = w0.x + w0.y;
  gr[7] = w1.x + w1.y;
  gr[8] = w2.x + w2.y;
  if (EXT) {
    const float2 wd = __fmul2_rn(w, f2(pa.gD, pb.gD));
    gr[9] = wd.x + wd.y;
  }
  // sigma and opacity gradients only where alpha was not clamped at 0.99
  const bool gA = cA && oe.x < SS_ALPHA_MAX, gB = cB && oe.y < SS_ALPHA_MAX;
  const float2 vs0 = __fmul2_rn(f2(-a.x, -a.y), va);
  const float2 ea = __fmul2_rn(ev, va);
  const float2 v = f2(gA ? vs0.x : 0.0f, gB ? vs0.y : 0.0f);
  gr[5] = (gA ? ea.x : 0.0f) + (gB ? ea.y : 0.0f);
  const float2 vdy = __fmul2_rn(v, dy);
  const float2 vdy2 = __fmul2_rn(vdy, dy);
  const float S0 = v.x + v.y, S1 = vdy.x + vdy.y, S2 = vdy2.x + vdy2.y;
  const float ca = 2.0f * st.a.z, cb = st.a.w, cc = 2.0f * st.b.x;  // staged halves doubled exactly
  const float dS0 = dx * S0;
  gr[0] = fmaf(ca, dS0, cb * S1);
  gr[1] = fmaf(cb, dS0, cc * S1);
  gr[2] = 0.5f * dx * dS0;
  gr[3] = dx * S1;
  gr[4] = 0.5f * S2;
  return true;
}

// The warp's sums of an entry when a single lane contributed: that lane's
// values, stored by it (the row's pad words stay zero).
template <bool EXT>
__device__ __forceinline__ void store_sums(float* row, const float* gr) {
  reinterpret_cast<float4*>(row)[0] = make_float4(gr[0], gr[1], gr[2], gr[3]);
  reinterpret_cast<float4*>(row)[1] = make_float4(gr[4], gr[5], gr[6], gr[7]);
  reinterpret_cast<float2*>(row)[4] = make_float2(gr[8], EXT ? gr[9] : 0.0f);
}

// One replayed entry (bit hb of the lanes' candidate masks mA, mB) for the
// thread's pixel pair: sigma and exp where a pixel is a candidate, then the
// reverse step.  gr[0..9] is zero when neither pixel contributes.
template <bool EXT>
__device__ __forceinline__ bool entry_grad(const Stage& st, uint32_t mA, uint32_t mB, int hb, float px, float2 npy,
                                           float amin, PixB& pa, PixB& pb, float* gr) {
  bool contrib = false;
  const bool liveA = (mA >> hb) & 1u, liveB = (mB >> hb) & 1u;
  if (liveA || liveB) {
    const float dx = sub(st.a.x, px);
    const float2 dy = __fadd2_rn(f2s(st.a.y), npy);
    const float2 sig = sigma_pair(st, dx, dy);
    const bool needA = liveA && !(sig.x < 0.0f) && !(sig.x > st.d.x);
    const bool needB = liveB && !(sig.y < 0.0f) && !(sig.y > st.d.x);
    if (needA || needB) contrib = pair_grad<EXT>(st, dx, dy, sig, needA, needB, amin, pa, pb, gr);
  }
  if (!contrib) {
#pragma unroll
    for (int t = 0; t < 10; ++t) gr[t] = 0.0f;
  }
  return contrib;
}

// EXT: v_depth (nullable, per pixel) and bg (nullable, [C][3]; the blend
// img = C + T_final * bg adds g . bg to dL/dT_final).
//
// Each warp replays its own 16x4 region independently (no CTA barrier): it
// walks the tile's entries from the last one any of its pixels composited
// down to the tile's first, 32 at a time, lane l holding entry
// top - 32k - 31 + l of block k.  The screen rows of block k + 1 are copied
// into the warp's second row buffer (asynchronous 16-byte copies) while
// block k runs, with the row ids of block k + 2 loaded meanwhile.  A
// touched entry's warp sums go to v_screen with three 16-byte atomics from
// the lane that holds the entry.
template <bool EXT>
__global__ __launch_bounds__(kRThreads, 6) void k_raster_bwd(Geo g, const float* __restrict__ screen,
                                                          const uint32_t* __restrict__ vals,
                                                          const int64_t* __restrict__ tile_off,
                                                          const float* __restrict__ T_final,
                                                          const int32_t* __restrict__ last_id,
                                                          const float* __restrict__ v_img,
                                                          const float* __restrict__ v_T,
                                                          const float* __restrict__ v_depth,
                                                          const float* __restrict__ bg,
                                                          const uint32_t* __restrict__ tile_order,
                                                          float* __restrict__ v_screen) {
  constexpr int kWarps = kRThreads / 32;
  __shared__ __align__(16) float s_raw[kWarps][2][32][kRowF];  // rows of the block in work and the next
  __shared__ Stage s_e[kWarps][32];
  // the warp's sums of each entry of the block (plain stores: a warp visits
  // an entry once; slots 10 and 11, and 9 without EXT, stay zero)
  __shared__ __align__(16) float red[kWarps][32][kRedF];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t tile = tile_order ? (int64_t)tile_order[blockIdx.x] : (int64_t)blockIdx.x;
  if (tile >= g.n_tiles) return;  // not a tile index: nothing to replay
  int c, tx0, ty0, i, j;
  tile_coords(g, tile, c, tx0, ty0, i, j);
  const bool inA = i < g.W && j < g.H, inB = i < g.W && j + 1 < g.H;
  const float px = add((float)i, 0.5f);
  const float2 npy = f2(-add((float)j, 0.5f), -add((float)(j + 1), 0.5f));
  const float x_lo = (float)tx0 + 0.5f;
  const float y_lo = (float)(j - 2 * (lane >> 4)) + 0.5f;
  const int64_t beg = tile_off[tile];
  const float amin = alpha_min();
  float* rw = &red[warp][lane][0];
#pragma unroll
  for (int t = 0; t < kRedF; ++t) rw[t] = 0.0f;
  PixB pa{1.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, -1}, pb{1.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, -1};
  const int64_t pixA = ((int64_t)c * g.H + j) * g.W + i, pixB = pixA + g.W;
  if (inA) {
    pa.last = last_id[pixA];
    pa.T = T_final[pixA];
    pa.g0 = v_img[3 * pixA];
    pa.g1 = v_img[3 * pixA + 1];
    pa.g2 = v_img[3 * pixA + 2];
    float vt = v_T ? v_T[pixA] : 0.0f;
    if (EXT && bg) vt += pa.g0 * bg[3 * c] + pa.g1 * bg[3 * c + 1] + pa.g2 * bg[3 * c + 2];
    if (EXT && v_depth) pa.gD = v_depth[pixA];
    pa.vTT = mul(vt, pa.T);
  }
  if (inB) {
    pb.last = last_id[pixB];
    pb.T = T_final[pixB];
    pb.g0 = v_img[3 * pixB];
    pb.g1 = v_img[3 * pixB + 1];
    pb.g2 = v_img[3 * pixB + 2];
    float vt = v_T ? v_T[pixB] : 0.0f;
    if (EXT && bg) vt += pb.g0 * bg[3 * c] + pb.g1 * bg[3 * c + 1] + pb.g2 * bg[3 * c + 2];
    if (EXT && v_depth) pb.gD = v_depth[pixB];
    pb.vTT = mul(vt, pb.T);
  }
  int64_t top = max64(pa.last, pb.last);  // the warp's last replayed entry
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) top = max64(top, __shfl_xor_sync(0xffffffffu, top, o));
  if (top < beg) return;
  const int nblk = (int)((top - beg) / 32 + 1);
  // row id of this lane's entry in block k (~0u: none)
  auto row_of = [&](int k) -> uint32_t {
    const int64_t e = top - 32 * (int64_t)k - 31 + lane;
    return (k < nblk && e >= beg) ? vals[e] : ~0u;
  };
  auto fetch = [&](int k, uint32_t r) {
    if (r != ~0u) {
      const float* src = screen + (int64_t)r * kRowF;
      float* dst = &s_raw[warp][k & 1][lane][0];
      cp_async16(dst, src);
      cp_async16(dst + 4, src + 4);
      cp_async16(dst + 8, src + 8);
    }
    cp_async_commit();
  };
  uint32_t rcur = row_of(0);
  fetch(0, rcur);
  uint32_t rnext = row_of(1);
  for (int k = 0; k < nblk; ++k) {
    const uint32_t rnext2 = row_of(k + 2);
    fetch(k + 1, rnext);
    cp_async_wait_group<1>();  // this lane's rows of block k have landed
    const int64_t qb = top - 32 * (int64_t)k - 31;
    uint32_t covA = 0u, covB = 0u;
    if (rcur != ~0u) {
      const float4* raw = reinterpret_cast<const float4*>(&s_raw[warp][k & 1][lane][0]);
      Stage st;
      stage_from(raw[0], raw[1], raw[2], rcur, st);
      s_e[warp][lane] = st;
      entry_coverage(st, x_lo, y_lo, covA, covB);
    }
    __syncwarp();
    // candidate masks as in the forward: bit b of mA (mB) set when entry
    // qb + b can reach this lane's upper (lower) pixel and the pixel replays
    // it; the warp steps through the union of its lanes' masks
    const uint32_t mA = warp_transpose32(covA, lane) & live_bits(pa.last, qb);
    const uint32_t mB = warp_transpose32(covB, lane) & live_bits(pb.last, qb);
    uint32_t bits = __reduce_or_sync(0xffffffffu, mA | mB);
    uint32_t touched = 0u;  // warp-uniform: entries whose sums were stored
    while (bits) {
      int hb = 31 - __clz(bits);
      bits &= ~(1u << hb);
      float gr[10];
      bool cA;
      uint32_t balA;
      const uint32_t mAB = mA | mB;
      if (bits) {
        // the next candidate of the warp: its pixel step follows this
        // one's, and the two entries' sums are reduced together
        const int hb2 = 31 - __clz(bits);
        bits &= ~(1u << hb2);
        float gr2[10];
        bool cB;
        const bool inA2 = (mAB >> hb) & 1u, inB2 = (mAB >> hb2) & 1u;
        if (!__any_sync(0xffffffffu, inA2 && inB2)) {
          // no pixel pair of the warp is a candidate of both entries: each
          // lane steps through the one entry it has (if any), so both
          // entries take one pixel step between them
          const int hx = inA2 ? hb : hb2;
          float g1[10];
          const bool c1 = entry_grad<EXT>(s_e[warp][hx], mA, mB, hx, px, npy, amin, pa, pb, g1);
          cA = inA2 && c1;
          cB = !inA2 && c1;
#pragma unroll
          for (int t = 0; t < 10; ++t) {
            gr[t] = inA2 ? g1[t] : 0.0f;
            gr2[t] = inA2 ? 0.0f : g1[t];
          }
        } else {
          cA = entry_grad<EXT>(s_e[warp][hb], mA, mB, hb, px, npy, amin, pa, pb, gr);
          cB = entry_grad<EXT>(s_e[warp][hb2], mA, mB, hb2, px, npy, amin, pa, pb, gr2);
        }
        balA = __ballot_sync(0xffffffffu, cA);
        const uint32_t balB = __ballot_sync(0xffffffffu, cB);
        touched |= (balA ? 1u << hb : 0u) | (balB ? 1u << hb2 : 0u);
        if ((balA & (balA - 1u)) == 0u && (balB & (balB - 1u)) == 0u) {
          // at most one lane contributes to each entry: its pixel pair's
          // sums are the warp's, stored as they are
          if (cA) store_sums<EXT>(red[warp][hb], gr);
          if (cB) store_sums<EXT>(red[warp][hb2], gr2);
          continue;
        }
        if (balA && balB) {
          const float s8 = warp_reduce8x2(gr, gr2, lane);
          const float s2 = warp_sum_x2<EXT>(gr[8], gr[9], gr2[8], gr2[9], lane);
          const int kl = (lane & 16) ? hb2 : hb;
          if ((lane & 1) == 0) red[warp][kl][((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1)] = s8;
          if ((lane & 15) == 0) red[warp][kl][8] = s2;
          if (EXT && (lane & 15) == 8) red[warp][kl][9] = s2;
          continue;
        }
        if (balB) {
#pragma unroll
          for (int t = 0; t < 10; ++t) gr[t] = gr2[t];
          hb = hb2;
          cA = cB;
          balA = balB;
        }
      } else {
        cA = entry_grad<EXT>(s_e[warp][hb], mA, mB, hb, px, npy, amin, pa, pb, gr);
        balA = __ballot_sync(0xffffffffu, cA);
        touched |= balA ? 1u << hb : 0u;
      }
      if ((balA & (balA - 1u)) == 0u) {
        if (cA) store_sums<EXT>(red[warp][hb], gr);
      } else {
        const float s8 = warp_reduce8(gr, lane);
        const float sb = warp_sum(gr[8]);
        const float sd = EXT ? warp_sum(gr[9]) : 0.0f;
        if ((lane & 3) == 0) red[warp][hb][((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1)] = s8;
        if (lane == 0) {
          red[warp][hb][8] = sb;
          if (EXT) red[warp][hb][9] = sd;
        }
      }
    }
    __syncwarp();
    if ((touched >> lane) & 1u) {
      const float4* src = reinterpret_cast<const float4*>(rw);
      float4* dst = reinterpret_cast<float4*>(v_screen + (int64_t)rcur * kRowF);
      atomicAdd(dst, src[0]);
      atomicAdd(dst + 1, src[1]);
      atomicAdd(dst + 2, src[2]);
    }
    __syncwarp();
    rcur = rnext;
    rnext = rnext2;
  }
  cp_async_wait_group<0>();
}

// ----- tile order: heaviest tiles first ------------------------------------
// The rasterizers take one CTA per tile, and tiles differ in their entry
// counts by orders of magnitude (most are empty, a few hold thousands of
// entries).  The block scheduler hands out CTAs in index order, so a heavy
// tile that comes late runs on after the rest have finished; taking tiles in
// decreasing order of entry count (longest first) keeps the SMs busy to the
// end.  The order is a counting sort over bins of the count: four bins per
// power of two (the two bits below the leading one), heavier bins first,
// empty tiles last; the order inside a bin is the order the atomic cursor
// hands out (any order draws the same images).
constexpr int kOrderBins = 128;

__device__ __forceinline__ int order_bin(int64_t cnt) {
  if (cnt <= 0) return kOrderBins - 1;
  const int msb = 63 - __clzll((long long)cnt);
  const int key = msb < 2 ? (int)cnt : 4 * msb + (int)((cnt >> (msb - 2)) & 3);  // non-decreasing in cnt
  return max(0, kOrderBins - 2 - key);
}

__global__ __launch_bounds__(256) void k_order_hist(const int64_t* __restrict__ tile_off, int64_t n_tiles,
                                                    uint32_t* __restrict__ hist) {
  __shared__ uint32_t h[kOrderBins];
  for (int i = threadIdx.x; i < kOrderBins; i += blockDim.x) h[i] = 0;
  __syncthreads();
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n_tiles; t += (int64_t)gridDim.x * blockDim.x)
    atomicAdd(&h[order_bin(tile_off[t + 1] - tile_off[t])], 1u);
  __syncthreads();
  for (int i = threadIdx.x; i < kOrderBins; i += blockDim.x)
    if (h[i]) atomicAdd(&hist[i], h[i]);
}

// hist -> exclusive prefix in place (the bins' write cursors); one warp.
__global__ void k_order_scan(uint32_t* __restrict__ hist) {
  const int lane = threadIdx.x;
  uint32_t carry = 0;
  for (int b0 = 0; b0 < kOrderBins; b0 += 32) {
    const uint32_t v = hist[b0 + lane];
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += x;
    }
    hist[b0 + lane] = carry + inc - v;
    carry += __shfl_sync(0xffffffffu, inc, 31);
  }
}

// One cursor atomic per (warp, bin): lanes with equal bins share it.
__global__ __launch_bounds__(256) void k_order_scatter(const int64_t* __restrict__ tile_off, int64_t n_tiles,
                                                       uint32_t* __restrict__ cursor,
                                                       uint32_t* __restrict__ tile_order) {
  const int lane = threadIdx.x & 31;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x; base < n_tiles; base += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = base + threadIdx.x;
    const bool valid = t < n_tiles;
    const int bin = valid ? order_bin(tile_off[t + 1] - tile_off[t]) : -1 - lane;
    const uint32_t peers = __match_any_sync(0xffffffffu, bin);
    const int leader = __ffs(peers) - 1;
    uint32_t first = 0;
    if (valid && lane == leader) first = atomicAdd(&cursor[bin], (uint32_t)__popc(peers));
    first = __shfl_sync(0xffffffffu, first, leader);
    if (valid) tile_order[first + __popc(peers & ((1u << lane) - 1u))] = (uint32_t)t;
  }
}

size_t tile_order_temp_bytes() { return kOrderBins * sizeof(uint32_t); }

}  // namespace ss

using namespace ss;

extern "C" ss_status ss_tile_order(const ss_dims* dims, const int64_t* tile_off, uint32_t* tile_order, void* temp,
                                   size_t temp_bytes, void* stream) {
  if (!dims_ok(dims)) return invalid("dims");
  if (!tile_off || !tile_order) return invalid("null pointer");
  if (!temp || temp_bytes < tile_order_temp_bytes()) return invalid("temp too small");
  const Geo g = geometry(*dims);
  cudaStream_t st = as_stream(stream);
  uint32_t* hist = reinterpret_cast<uint32_t*>(temp);
  ss_status s = cuda_status(cudaMemsetAsync(hist, 0, tile_order_temp_bytes(), st), "memset");
  if (s) return s;
  const unsigned grid = (unsigned)max64(1, min64(ceil_div(g.n_tiles, 256), 148 * 4));
  k_order_hist<<<grid, 256, 0, st>>>(tile_off, g.n_tiles, hist);
  k_order_scan<<<1, 32, 0, st>>>(hist);
  k_order_scatter<<<grid, 256, 0, st>>>(tile_off, g.n_tiles, hist, tile_order);
  return cuda_status(cudaGetLastError(), "tile order");
}

extern "C" ss_status ss_rasterize_fwd(const ss_dims* dims, const float* screen, const uint32_t* vals,
                                      const int64_t* tile_off, const uint32_t* tile_order, float* img,
                                      float* T_final, int32_t* last_id, float* depth, const float* bg,
                                      void* stream) {
  if (!dims_ok(dims)) return invalid("dims");
  if (!tile_off || !img || !T_final || !last_id) return invalid("null pointer");
  if (((uintptr_t)screen & 15) != 0) return invalid("screen must be 16-byte aligned");
  const Geo g = geometry(*dims);
  cudaStream_t st = as_stream(stream);
  if (depth || bg) {
    k_raster_fwd_masked<true><<<(unsigned)g.n_tiles, kRThreads, 0, st>>>(g, screen, vals, tile_off, img, T_final,
                                                                         last_id, depth, bg, tile_order);
  } else {
    k_raster_fwd_masked<false><<<(unsigned)g.n_tiles, kRThreads, 0, st>>>(g, screen, vals, tile_off, img, T_final,
                                                                          last_id, nullptr, nullptr, tile_order);
  }
  return cuda_status(cudaGetLastError(), "rasterize fwd");
}

extern "C" ss_status ss_rasterize_fwd_counts(const ss_dims* dims, const float* screen, const uint32_t* vals,
                                             const int64_t* tile_off, float* img, float* T_final, int32_t* last_id,
                                             uint64_t* counts, void* stream) {
  if (!dims_ok(dims)) return invalid("dims");
  if (!tile_off || !img || !T_final || !last_id || !counts) return invalid("null pointer");
  if (((uintptr_t)screen & 15) != 0) return invalid("screen must be 16-byte aligned");
  const Geo g = geometry(*dims);
  cudaStream_t st = as_stream(stream);
  ss_status s = cuda_status(cudaMemsetAsync(counts, 0, 5 * sizeof(uint64_t), st), "memset");
  if (s) return s;
  k_raster_fwd<true><<<(unsigned)g.n_tiles, kRThreads, 0, st>>>(g, screen, vals, tile_off, img, T_final, last_id,
                                                                reinterpret_cast<unsigned long long*>(counts));
  return cuda_status(cudaGetLastError(), "rasterize fwd (counted)");
}

extern "C" ss_status ss_rasterize_bwd(const ss_dims* dims, const float* screen, const uint32_t* vals,
                                      const int64_t* tile_off, const uint32_t* tile_order, const float* T_final,
                                      const int32_t* last_id, const float* v_img, const float* v_T,
                                      const float* v_depth, const float* bg, float* v_screen, int64_t nnz,
                                      void* stream) {
  if (!dims_ok(dims)) return invalid("dims");
  if (nnz < 0) return invalid("nnz < 0");
  if (!tile_off || !T_final || !last_id || !v_img || (nnz > 0 && !v_screen)) return invalid("null pointer");
  if (((uintptr_t)screen & 15) != 0 || ((uintptr_t)v_screen & 15) != 0) return invalid("rows must be 16-byte aligned");
  const Geo g = geometry(*dims);
  cudaStream_t st = as_stream(stream);
  if (nnz > 0) {
    ss_status s = cuda_status(cudaMemsetAsync(v_screen, 0, (size_t)nnz * kRowF * sizeof(float), st), "memset");
    if (s) return s;
  }
  if (v_depth || bg) {
    k_raster_bwd<true><<<(unsigned)g.n_tiles, kRThreads, 0, st>>>(g, screen, vals, tile_off, T_final, last_id, v_img,
                                                                  v_T, v_depth, bg, tile_order, v_screen);
  } else {
    k_raster_bwd<false><<<(unsigned)g.n_tiles, kRThreads, 0, st>>>(g, screen, vals, tile_off, T_final, last_id,
                                                                   v_img, v_T, nullptr, nullptr, tile_order,
                                                                   v_screen);
  }
  return cuda_status(cudaGetLastError(), "rasterize bwd");
}
