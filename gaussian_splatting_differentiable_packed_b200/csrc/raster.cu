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

// COUNT adds per-pixel work counters (measurement helper): entries evaluated,
// exps evaluated, entries composited; and for the backward replay (entries up
// to last_id): entries replayed and exps evaluated.
template <bool COUNT>
__global__ __launch_bounds__(kPix) void k_raster_fwd(Geo g, const float* __restrict__ screen,
                                                     const uint32_t* __restrict__ vals,
                                                     const int64_t* __restrict__ tile_off, float* __restrict__ img,
                                                     float* __restrict__ T_final, int32_t* __restrict__ last_id,
                                                     unsigned long long* __restrict__ counts) {
  __shared__ float4 s_a[kFwdBatch];  // x, y, 0.5*ca, cb
  __shared__ float4 s_b[kFwdBatch];  // 0.5*cc, o, r, g
  __shared__ float s_c[kFwdBatch];   // b
  const int64_t tile = blockIdx.x;
  int c, i, j;
  tile_coords(g, tile, c, i, j);
  const bool inside = i < g.W && j < g.H;
  const float px = add((float)i, 0.5f), py = add((float)j, 0.5f);
  const int64_t beg = tile_off[tile], end = tile_off[tile + 1];
  const float amin = alpha_min();
  float T = 1.0f, C0 = 0.0f, C1 = 0.0f, C2 = 0.0f;
  int64_t last = -1;
  bool done = !inside;
  unsigned long long n_eval = 0, n_exp = 0, n_comp = 0, n_exp_last = 0;
  for (int64_t b0 = beg; b0 < end; b0 += kFwdBatch) {
    if (__syncthreads_count(done) == kPix) break;
    const int64_t idx = b0 + threadIdx.x;
    if (idx < end) {
      const float4* row = reinterpret_cast<const float4*>(screen + (int64_t)vals[idx] * kRowF);
      const float4 r0 = row[0], r1 = row[1], r2 = row[2];
      s_a[threadIdx.x] = make_float4(r0.x, r0.y, mul(0.5f, r0.z), r0.w);
      s_b[threadIdx.x] = make_float4(mul(0.5f, r1.x), r1.y, r1.z, r1.w);
      s_c[threadIdx.x] = r2.x;
    }
    __syncthreads();
    if (!done) {
      const int cnt = (int)min64(kFwdBatch, end - b0);
      for (int k = 0; k < cnt; ++k) {
        if (COUNT) ++n_eval;
        const float4 A = s_a[k];
        const float dx = sub(A.x, px), dy = sub(A.y, py);
        const float4 B = s_b[k];
        const float sig = gauss_sigma(A.z, A.w, B.x, dx, dy);
        if (sig < 0.0f) continue;
        if (sig > SS_SIGMA_SKIP && B.y <= 1.0f) continue;  // o*exp(-sig) < 1/255 guaranteed
        if (COUNT) ++n_exp;
        const float e = exp_neg(-sig);
        const float alpha = fminf(SS_ALPHA_MAX, mul(B.y, e));
        if (alpha < amin) continue;
        const float Tn = mul(T, sub(1.0f, alpha));
        if (Tn < SS_T_STOP) {
          done = true;
          break;
        }
        const float w = mul(alpha, T);
        C0 = fma_(B.z, w, C0);
        C1 = fma_(B.w, w, C1);
        C2 = fma_(s_c[k], w, C2);
        T = Tn;
        last = b0 + k;
        if (COUNT) {
          ++n_comp;
          n_exp_last = n_exp;
        }
      }
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
      if ((threadIdx.x & 31) == 0 && x) atomicAdd(&counts[q], x);
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
  __shared__ float4 s_a[kBwdBatch];  // x, y, 0.5*ca, cb
  __shared__ float4 s_b[kBwdBatch];  // 0.5*cc, o, r, g
  __shared__ float s_c[kBwdBatch];   // b
  __shared__ uint32_t s_row[kBwdBatch];
  __shared__ __align__(16) float red[kPix / 32][kBwdBatch][kRedF];
  __shared__ int s_maxlast;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t tile = blockIdx.x;
  int c, i, j;
  tile_coords(g, tile, c, i, j);
  const bool inside = i < g.W && j < g.H;
  const float px = add((float)i, 0.5f), py = add((float)j, 0.5f);
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
  const float vTT = mul(vT, Tfin);
  for (int64_t b1 = stop; b1 > beg; b1 -= kBwdBatch) {
    const int64_t b0 = max64(beg, b1 - kBwdBatch);
    const int cnt = (int)(b1 - b0);
    __syncthreads();
    if (threadIdx.x < cnt) {
      const uint32_t r = vals[b0 + threadIdx.x];
      const float4* row = reinterpret_cast<const float4*>(screen + (int64_t)r * kRowF);
      const float4 r0 = row[0], r1 = row[1], r2 = row[2];
      s_a[threadIdx.x] = make_float4(r0.x, r0.y, mul(0.5f, r0.z), r0.w);
      s_b[threadIdx.x] = make_float4(mul(0.5f, r1.x), r1.y, r1.z, r1.w);
      s_c[threadIdx.x] = r2.x;
      s_row[threadIdx.x] = r;
    }
    __syncthreads();
    for (int k = cnt - 1; k >= 0; --k) {
      const int64_t idx = b0 + k;
      float gr[9];
#pragma unroll
      for (int q = 0; q < 9; ++q) gr[q] = 0.0f;
      bool contrib = false;
      if (idx <= last) {
        const float4 A = s_a[k];
        const float dx = sub(A.x, px), dy = sub(A.y, py);
        const float4 B = s_b[k];
        const float sig = gauss_sigma(A.z, A.w, B.x, dx, dy);
        if (sig >= 0.0f && !(sig > SS_SIGMA_SKIP && B.y <= 1.0f)) {
          const float e = exp_neg(-sig);
          const float oe = mul(B.y, e);
          const float alpha = fminf(SS_ALPHA_MAX, oe);
          if (alpha >= amin) {
            contrib = true;
            const float ra = 1.0f / (1.0f - alpha);
            const float Ti = T * ra;
            const float w = alpha * Ti;
            const float rb = s_c[k];
            gr[6] = w * g0;
            gr[7] = w * g1;
            gr[8] = w * g2;
            const float rgbg = B.z * g0 + B.w * g1 + rb * g2;
            const float v_alpha = Ti * rgbg - ra * (Sg + vTT);
            Sg += w * rgbg;
            T = Ti;
            if (oe < SS_ALPHA_MAX) {
              const float v_sig = -alpha * v_alpha;
              gr[5] = e * v_alpha;
              gr[2] = v_sig * 0.5f * dx * dx;
              gr[3] = v_sig * dx * dy;
              gr[4] = v_sig * 0.5f * dy * dy;
              gr[0] = v_sig * (2.0f * A.z * dx + A.w * dy);
              gr[1] = v_sig * (A.w * dx + 2.0f * B.x * dy);
            }
          }
        }
      }
      if (__any_sync(0xffffffffu, contrib)) {
        const float s8 = warp_reduce8(gr, lane);
        const float sb = warp_sum(gr[8]);
        if ((lane & 3) == 0) red[warp][k][((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1)] = s8;
        if (lane == 0) red[warp][k][8] = sb;
      } else if (lane < 9) {
        red[warp][k][lane] = 0.0f;
      }
    }
    __syncthreads();
    // cross-warp sum and one vector atomic per (entry, 16-byte quarter)
    for (int t = threadIdx.x; t < cnt * 3; t += kPix) {
      const int k = t / 3, q = t - 3 * k;
      float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < kPix / 32; ++w) {
        if (q < 2) {
          const float4 v = *reinterpret_cast<const float4*>(&red[w][k][4 * q]);
          s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
        } else {
          s.x += red[w][k][8];
        }
      }
      if (s.x != 0.0f || s.y != 0.0f || s.z != 0.0f || s.w != 0.0f)
        atomicAdd(reinterpret_cast<float4*>(v_screen + (int64_t)s_row[k] * kRowF + 4 * q), s);
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
