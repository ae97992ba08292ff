// Tile rasterizer, forward and backward ("Spirula Studio backward pass",
// section 4: the forward keeps tile offsets, the sorted intersection list,
// each pixel's last composited entry and its final transmittance; the backward
// reuses them without re-intersecting, splits each pixel's gradient by alpha
// contribution and sums per Gaussian with atomics).
//
// One CTA per 16x16 tile, one thread per pixel.  Each batch of the tile's
// sorted entries is gathered once into shared memory (three 16-byte loads per
// 48-byte screen row) and evaluated by all 256 pixels.
#include "ss_common.cuh"
#include "ss_math.cuh"

namespace ss {

constexpr int kPix = kTile * kTile;  // 256 threads
constexpr int kFwdBatch = 256;
constexpr int kBwdBatch = 64;

__device__ __forceinline__ void tile_coords(const Geo& g, int64_t tile, int& c, int& i, int& j) {
  c = (int)(tile / g.tiles_per_cam);
  const int rem = (int)(tile - (int64_t)c * g.tiles_per_cam);
  const int ty = rem / g.tiles_x, tx = rem - ty * g.tiles_x;
  i = tx * kTile + (threadIdx.x & (kTile - 1));
  j = ty * kTile + (threadIdx.x >> 4);
}

// ---------------------------------------------------------------------------
// Warp culling.  A warp owns a 16x2 strip of the tile (rows 2w, 2w+1).  For an
// entry with o <= 1 every pixel whose computed sigma exceeds 5.6 is skipped by
// the per-pixel test anyway (o*exp(-sigma) < 1/255).  The staged half-extents
// (hx, hy) bound the ellipse {sigma <= 5.7} of the stored conic exactly
// (computed in fp64 with a margin); a strip outside that box has exact sigma
// > 5.7 at every pixel, and when kterm*(Dx^2 + Dy^2) <= 1e5 the fp32 rounding
// of the canonical sigma is below 0.04, so the computed sigma exceeds 5.6 too:
// skipping the entry for the whole warp takes exactly the per-pixel decision.
struct Stage {
  float4 a;  // x, y, 0.5*ca, cb
  float4 b;  // 0.5*cc, o, r, g
  float4 c;  // b, hx, hy, kterm
};

__device__ __forceinline__ void stage_row(const float* __restrict__ screen, uint32_t r, Stage& st) {
  const float4* row = reinterpret_cast<const float4*>(screen + (int64_t)r * kRowF);
  const float4 r0 = row[0], r1 = row[1], r2 = row[2];
  st.a = make_float4(r0.x, r0.y, mul(0.5f, r0.z), r0.w);
  st.b = make_float4(mul(0.5f, r1.x), r1.y, r1.z, r1.w);
  float hx = __int_as_float(0x7f800000), hy = hx;
  const double dq = (double)r0.z * (double)r1.x - (double)r0.w * (double)r0.w;
  if (r1.y <= 1.0f && dq > 0.0) {
    hx = (float)(sqrt(11.4 * (double)r1.x / dq) * 1.001 + 1e-3);
    hy = (float)(sqrt(11.4 * (double)r0.z / dq) * 1.001 + 1e-3);
  }
  const float kterm = 0.5f * fabsf(r0.z) + 0.5f * fabsf(r1.x) + fabsf(r0.w);
  st.c = make_float4(r2.x, hx, hy, kterm);
}

// True when the entry can be skipped by the whole warp (see above).
__device__ __forceinline__ bool warp_culled(const Stage& st, float x_lo, float x_hi, float y_lo, float y_hi) {
  const float mx = st.a.x, my = st.a.y;
  const float ex = fmaxf(fmaxf(x_lo - mx, mx - x_hi), 0.0f);
  const float ey = fmaxf(fmaxf(y_lo - my, my - y_hi), 0.0f);
  if (!(ex > st.c.y || ey > st.c.z)) return false;
  const float Dx = fmaxf(fabsf(x_lo - mx), fabsf(x_hi - mx));
  const float Dy = fmaxf(fabsf(y_lo - my), fabsf(y_hi - my));
  return st.c.w * (Dx * Dx + Dy * Dy) <= 1e5f;
}

// COUNT adds per-pixel work counters (measurement helper): entries evaluated,
// exps evaluated, entries composited; and for the backward replay (entries up
// to last_id): entries replayed and exps evaluated.  The counts follow the
// per-pixel definition (warp culling does not change them).
template <bool COUNT>
__global__ __launch_bounds__(kPix) void k_raster_fwd(Geo g, const float* __restrict__ screen,
                                                     const uint32_t* __restrict__ vals,
                                                     const int64_t* __restrict__ tile_off, float* __restrict__ img,
                                                     float* __restrict__ T_final, int32_t* __restrict__ last_id,
                                                     unsigned long long* __restrict__ counts) {
  __shared__ Stage s_e[kFwdBatch];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t tile = blockIdx.x;
  int c, i, j;
  tile_coords(g, tile, c, i, j);
  const bool inside = i < g.W && j < g.H;
  const float px = add((float)i, 0.5f), py = add((float)j, 0.5f);
  const float x_lo = (float)(i - (i & (kTile - 1))) + 0.5f, x_hi = x_lo + 15.0f;
  const float y_lo = (float)(j - (j & 1)) + 0.5f, y_hi = y_lo + 1.0f;
  const int64_t beg = tile_off[tile], end = tile_off[tile + 1];
  const float amin = alpha_min();
  float T = 1.0f, C0 = 0.0f, C1 = 0.0f, C2 = 0.0f;
  int64_t last = -1;
  bool done = !inside;
  unsigned long long n_eval = 0, n_exp = 0, n_comp = 0, n_exp_last = 0;
  for (int64_t b0 = beg; b0 < end; b0 += kFwdBatch) {
    if (__syncthreads_count(done) == kPix) break;
    const int64_t idx = b0 + threadIdx.x;
    if (idx < end) stage_row(screen, vals[idx], s_e[threadIdx.x]);
    __syncthreads();
    if (__all_sync(0xffffffffu, done)) continue;
    const int cnt = (int)min64(kFwdBatch, end - b0);
    for (int q = 0; q < kFwdBatch / 32; ++q) {
      if (q * 32 >= cnt) break;
      const int e = q * 32 + lane;
      uint32_t bits = __ballot_sync(0xffffffffu, e < cnt && (COUNT || !warp_culled(s_e[e], x_lo, x_hi, y_lo, y_hi)));
      while (bits) {
        const int k = q * 32 + __ffs(bits) - 1;
        bits &= bits - 1;
        if (done) continue;
        if (COUNT) ++n_eval;
        const Stage& st = s_e[k];
        const float dx = sub(st.a.x, px), dy = sub(st.a.y, py);
        const float sig = gauss_sigma(st.a.z, st.a.w, st.b.x, dx, dy);
        if (sig < 0.0f) continue;
        if (sig > SS_SIGMA_SKIP && st.b.y <= 1.0f) continue;  // o*exp(-sig) < 1/255 guaranteed
        if (COUNT) ++n_exp;
        const float ev = exp_neg(-sig);
        const float alpha = fminf(SS_ALPHA_MAX, mul(st.b.y, ev));
        if (alpha < amin) continue;
        const float Tn = mul(T, sub(1.0f, alpha));
        if (Tn < SS_T_STOP) {
          done = true;
          continue;
        }
        const float w = mul(alpha, T);
        C0 = fma_(st.b.z, w, C0);
        C1 = fma_(st.b.w, w, C1);
        C2 = fma_(st.c.x, w, C2);
        T = Tn;
        last = b0 + k;
        if (COUNT) {
          ++n_comp;
          n_exp_last = n_exp;
        }
      }
      if (__all_sync(0xffffffffu, done)) break;
    }
  }
  if (inside) {
    const int64_t pix = ((int64_t)c * g.H + j) * g.W + i;
    img[3 * pix] = C0;
    img[3 * pix + 1] = C1;
    img[3 * pix + 2] = C2;
    T_final[pix] = T;
    last_id[pix] = (int32_t)last;
  }
  if (COUNT) {
    const unsigned long long replay = last >= 0 ? (unsigned long long)(last - beg + 1) : 0ull;
    unsigned long long v[5] = {n_eval, n_exp, n_comp, replay, n_exp_last};
#pragma unroll
    for (int q = 0; q < 5; ++q) {
      unsigned long long x = v[q];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      if (lane == 0 && x) atomicAdd(&counts[q], x);
    }
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

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Gradient slots per entry in the shared reduction buffer (12 = 3 float4).
constexpr int kRedF = 12;

__global__ __launch_bounds__(kPix) void k_raster_bwd(Geo g, const float* __restrict__ screen,
                                                     const uint32_t* __restrict__ vals,
                                                     const int64_t* __restrict__ tile_off,
                                                     const float* __restrict__ T_final,
                                                     const int32_t* __restrict__ last_id,
                                                     const float* __restrict__ v_img, const float* __restrict__ v_T,
                                                     float* __restrict__ v_screen) {
  __shared__ Stage s_e[kBwdBatch];
  __shared__ uint32_t s_row[kBwdBatch];
  __shared__ uint32_t s_wmask[kBwdBatch];  // warps that contributed to each entry
  __shared__ __align__(16) float red[kPix / 32][kBwdBatch][kRedF];
  __shared__ int s_maxlast;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t tile = blockIdx.x;
  int c, i, j;
  tile_coords(g, tile, c, i, j);
  const bool inside = i < g.W && j < g.H;
  const float px = add((float)i, 0.5f), py = add((float)j, 0.5f);
  const float x_lo = (float)(i - (i & (kTile - 1))) + 0.5f, x_hi = x_lo + 15.0f;
  const float y_lo = (float)(j - (j & 1)) + 0.5f, y_hi = y_lo + 1.0f;
  const int64_t beg = tile_off[tile];
  const float amin = alpha_min();
  float T = 1.0f, Tfin = 1.0f, g0 = 0.0f, g1 = 0.0f, g2 = 0.0f, vT = 0.0f, Sg = 0.0f;
  int64_t last = -1;
  if (threadIdx.x == 0) s_maxlast = -1;
  __syncthreads();
  if (inside) {
    const int64_t pix = ((int64_t)c * g.H + j) * g.W + i;
    last = last_id[pix];
    Tfin = T_final[pix];
    T = Tfin;
    g0 = v_img[3 * pix];
    g1 = v_img[3 * pix + 1];
    g2 = v_img[3 * pix + 2];
    vT = v_T ? v_T[pix] : 0.0f;
    if (last >= 0) atomicMax(&s_maxlast, (int)last);
  }
  __syncthreads();
  const int64_t stop = (int64_t)s_maxlast + 1;  // entries [beg, stop) can matter
  // the warp's own last entry: entries above it need no work from this warp
  int64_t wlast = last;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wlast = max64(wlast, __shfl_xor_sync(0xffffffffu, wlast, o));
  const float vTT = mul(vT, Tfin);
  for (int64_t b1 = stop; b1 > beg; b1 -= kBwdBatch) {
    const int64_t b0 = max64(beg, b1 - kBwdBatch);
    const int cnt = (int)(b1 - b0);
    __syncthreads();
    if (threadIdx.x < cnt) {
      const uint32_t r = vals[b0 + threadIdx.x];
      stage_row(screen, r, s_e[threadIdx.x]);
      s_row[threadIdx.x] = r;
      s_wmask[threadIdx.x] = 0u;
    }
    __syncthreads();
    if (b0 <= wlast) {
      for (int q = (cnt - 1) / 32; q >= 0; --q) {
        const int e = q * 32 + lane;
        uint32_t bits = __ballot_sync(0xffffffffu, e < cnt && b0 + e <= wlast &&
                                                      !warp_culled(s_e[e], x_lo, x_hi, y_lo, y_hi));
        while (bits) {
          const int hb = 31 - __clz(bits);
          bits &= ~(1u << hb);
          const int k = q * 32 + hb;
          const int64_t idx = b0 + k;
          float gr[9];
#pragma unroll
          for (int t = 0; t < 9; ++t) gr[t] = 0.0f;
          bool contrib = false;
          if (idx <= last) {
            const Stage& st = s_e[k];
            const float dx = sub(st.a.x, px), dy = sub(st.a.y, py);
            const float sig = gauss_sigma(st.a.z, st.a.w, st.b.x, dx, dy);
            if (sig >= 0.0f && !(sig > SS_SIGMA_SKIP && st.b.y <= 1.0f)) {
              const float ev = exp_neg(-sig);
              const float oe = mul(st.b.y, ev);
              const float alpha = fminf(SS_ALPHA_MAX, oe);
              if (alpha >= amin) {
                contrib = true;
                const float ra = 1.0f / (1.0f - alpha);
                const float Ti = T * ra;
                const float w = alpha * Ti;
                gr[6] = w * g0;
                gr[7] = w * g1;
                gr[8] = w * g2;
                const float rgbg = st.b.z * g0 + st.b.w * g1 + st.c.x * g2;
                const float v_alpha = Ti * rgbg - ra * (Sg + vTT);
                Sg += w * rgbg;
                T = Ti;
                if (oe < SS_ALPHA_MAX) {
                  const float v_sig = -alpha * v_alpha;
                  gr[5] = ev * v_alpha;
                  gr[2] = v_sig * 0.5f * dx * dx;
                  gr[3] = v_sig * dx * dy;
                  gr[4] = v_sig * 0.5f * dy * dy;
                  gr[0] = v_sig * (2.0f * st.a.z * dx + st.a.w * dy);
                  gr[1] = v_sig * (st.a.w * dx + 2.0f * st.b.x * dy);
                }
              }
            }
          }
          if (__any_sync(0xffffffffu, contrib)) {
            const float s8 = warp_reduce8(gr, lane);
            const float sb = warp_sum(gr[8]);
            if ((lane & 3) == 0) red[warp][k][((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1)] = s8;
            if (lane == 0) {
              red[warp][k][8] = sb;
              atomicOr(&s_wmask[k], 1u << warp);
            }
          }
        }
      }
    }
    __syncthreads();
    // cross-warp sum over the contributing warps, one vector atomic per (entry, 16-byte quarter)
    for (int t = threadIdx.x; t < cnt * 3; t += kPix) {
      const int k = t / 3, q = t - 3 * k;
      uint32_t m = s_wmask[k];
      if (!m) continue;
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
      while (m) {
        const int w = __ffs(m) - 1;
        m &= m - 1;
        if (q < 2) {
          const float4 v = *reinterpret_cast<const float4*>(&red[w][k][4 * q]);
          sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
        } else {
          sum.x += red[w][k][8];
        }
      }
      atomicAdd(reinterpret_cast<float4*>(v_screen + (int64_t)s_row[k] * kRowF + 4 * q), sum);
    }
  }
}

}  // namespace ss

using namespace ss;

extern "C" ss_status ss_rasterize_fwd(const ss_dims* dims, const float* screen, const uint32_t* vals,
                                      const int64_t* tile_off, float* img, float* T_final, int32_t* last_id,
                                      void* stream) {
  if (!dims_ok(dims)) return invalid("dims");
  if (!tile_off || !img || !T_final || !last_id) return invalid("null pointer");
  if (((uintptr_t)screen & 15) != 0) return invalid("screen must be 16-byte aligned");
  const Geo g = geometry(*dims);
  cudaStream_t st = as_stream(stream);
  k_raster_fwd<false><<<(unsigned)g.n_tiles, kPix, 0, st>>>(g, screen, vals, tile_off, img, T_final, last_id,
                                                            nullptr);
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
  k_raster_fwd<true><<<(unsigned)g.n_tiles, kPix, 0, st>>>(g, screen, vals, tile_off, img, T_final, last_id,
                                                           reinterpret_cast<unsigned long long*>(counts));
  return cuda_status(cudaGetLastError(), "rasterize fwd (counted)");
}

extern "C" ss_status ss_rasterize_bwd(const ss_dims* dims, const float* screen, const uint32_t* vals,
                                      const int64_t* tile_off, const float* T_final, const int32_t* last_id,
                                      const float* v_img, const float* v_T, float* v_screen, int64_t nnz,
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
  k_raster_bwd<<<(unsigned)g.n_tiles, kPix, 0, st>>>(g, screen, vals, tile_off, T_final, last_id, v_img, v_T,
                                                    v_screen);
  return cuda_status(cudaGetLastError(), "rasterize bwd");
}
