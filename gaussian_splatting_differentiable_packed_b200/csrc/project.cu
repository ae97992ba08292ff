// Packed projection ("Spirula Studio VRAM deep-dive", section "bitmask
// compaction"; "16-bit packed AABB"; projection chain from the "Spirula Studio
// backward pass" page, section 5).
//
// Pass 1 (k_project_mask): one thread per Gaussian, 128 threads per CTA, loops
// over the cameras so each Gaussian's parameters are read once.  For camera c
// the CTA's 128 pairs are bits [c*n_pad + 128*blk, +128) of the mask: each warp
// writes its ballot word and the CTA writes one popcount (block_count).
// Scan: block_off = exclusive scan of block_count (int64), nnz at the end.
// Pass 2 (k_project_rows): same geometry; a thread whose bit is set re-projects
// its pair and writes row = block_off[block] + popc(earlier words of the block)
// + popc(bits below it in its word).
#include "ss_common.cuh"
#include "ss_math.cuh"

namespace ss {

constexpr int kCamChunk = 32;

struct GaussIn {
  float mx, my, mz;
  Cov3 S;
};

__device__ __forceinline__ GaussIn load_gauss(const float* means, const float* quats, const float* scales, int64_t n) {
  GaussIn g;
  g.mx = means[3 * n]; g.my = means[3 * n + 1]; g.mz = means[3 * n + 2];
  float4 q = reinterpret_cast<const float4*>(quats)[n];
  QuatRot r = quat_rot(q.x, q.y, q.z, q.w);
  g.S = cov3(r, scales[3 * n], scales[3 * n + 1], scales[3 * n + 2]);
  return g;
}

__global__ __launch_bounds__(kBlock) void k_project_mask(Geo g, const float* __restrict__ cams,
                                                         const float* __restrict__ means,
                                                         const float* __restrict__ quats,
                                                         const float* __restrict__ scales, uint32_t* __restrict__ mask,
                                                         uint32_t* __restrict__ block_count) {
  __shared__ Cam scam[kCamChunk];
  __shared__ uint32_t wcnt[kCamChunk][kBlock / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t blk = blockIdx.x;
  const int64_t n = blk * kBlock + threadIdx.x;
  const bool valid = n < g.N;
  GaussIn gi{};
  if (valid) gi = load_gauss(means, quats, scales, n);
  for (int c0 = 0; c0 < g.C; c0 += kCamChunk) {
    const int nc = min(kCamChunk, g.C - c0);
    __syncthreads();
    if (threadIdx.x < nc) scam[threadIdx.x] = load_cam(cams + 20 * (int64_t)(c0 + threadIdx.x), g.W, g.H);
    __syncthreads();
    for (int cc = 0; cc < nc; ++cc) {
      bool vis = false;
      if (valid) {
        const Cam& k = scam[cc];
        Proj P;
        cam_point(k, gi.mx, gi.my, gi.mz, P.px, P.py, P.pz);
        if (g.near_plane < P.pz && P.pz < g.far_plane) {
          project_rest(k, gi.S, g.W, g.H, P);
          vis = P.vis;
        }
      }
      const uint32_t word = __ballot_sync(0xffffffffu, vis);
      if (lane == 0) {
        const int64_t c = c0 + cc;
        mask[(c * g.n_pad + blk * kBlock) / 32 + warp] = word;
        wcnt[cc][warp] = __popc(word);
      }
    }
    __syncthreads();
    if (threadIdx.x < nc) {
      const int64_t c = c0 + threadIdx.x;
      uint32_t s = 0;
#pragma unroll
      for (int w = 0; w < kBlock / 32; ++w) s += wcnt[threadIdx.x][w];
      block_count[c * g.blocks_per_cam + blk] = s;
    }
  }
}

// Shared-memory layout of a CTA's SH block.  With 3(D+1)^2 a multiple of 4
// (degrees 1 and 3) a row is copied and read in 16-byte words and its stride
// is an odd number of them, so the 8 lanes of a quarter-warp that read 16
// bytes each from 8 different rows hit 8 different bank groups.  Otherwise
// the stride is an odd number of words (word accesses of 32 rows conflict-
// free).
template <int DEG>
__host__ __device__ constexpr bool rows_sh_vec() {
  return (3 * (DEG + 1) * (DEG + 1)) % 4 == 0;
}
template <int DEG>
__host__ __device__ constexpr int rows_sh_stride() {
  constexpr int K3 = 3 * (DEG + 1) * (DEG + 1);
  if (rows_sh_vec<DEG>()) return ((K3 / 4) % 2 == 1) ? K3 : K3 + 4;
  return (K3 % 2 == 0) ? K3 + 1 : K3;
}

// A visible (camera, Gaussian) pair waiting in the CTA's work queue.
struct RowItem {
  int64_t row;
  int cam;  // camera within the current chunk
  int g;    // Gaussian within the CTA
};

// Pass 2 keeps its 128 threads busy whatever the visibility pattern.  For a
// chunk of cameras the CTA stages each warp's mask word per camera and an
// exclusive prefix of their popcounts in camera-major order; the chunk's
// visible pairs are then items 0..total-1 of a virtual list, and thread t
// decodes item i (t, t + 128, ...) by itself: the (camera, warp) slot by
// binary search in the prefix, the lane as the rank-th set bit of the slot's
// word, the row as the camera's block offset plus the rank among the
// camera's set bits.  Consecutive items are consecutive rows.
template <int DEG>
__global__ __launch_bounds__(kBlock) void k_project_rows(Geo g, const float* __restrict__ cams,
                                                         const float* __restrict__ means,
                                                         const float* __restrict__ quats,
                                                         const float* __restrict__ scales,
                                                         const float* __restrict__ opacities,
                                                         const float* __restrict__ sh,
                                                         const uint32_t* __restrict__ mask,
                                                         const int64_t* __restrict__ block_off,
                                                         float* __restrict__ screen, uint32_t* __restrict__ aabb16,
                                                         float* __restrict__ row_depth, int64_t ahead) {
  constexpr int K = (DEG + 1) * (DEG + 1);
  constexpr int K3 = 3 * K;
  constexpr int KP = rows_sh_stride<DEG>();
  constexpr int kWarps = kBlock / 32;
  constexpr int kSlots = kCamChunk * kWarps;
  __shared__ Cam scam[kCamChunk];
  __shared__ __align__(16) float sh_s[kBlock * KP];
  __shared__ GaussIn s_g[kBlock];
  __shared__ float s_o[kBlock];
  __shared__ uint32_t s_word[kSlots];  // [camera][warp]
  __shared__ int s_pre[kSlots + 1];    // exclusive prefix of the words' popcounts
  __shared__ int64_t s_row0[kCamChunk];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t blk = blockIdx.x;
  const int64_t n0 = blk * kBlock;
  const int64_t n = n0 + threadIdx.x;
  const int cnt = (int)min64(kBlock, g.N - n0);
  const bool prefetch_ahead = ahead > 0 && blk + ahead < (int64_t)gridDim.x;
  if (prefetch_ahead && threadIdx.x == 0) {
    // the parameters and the SH block of the block that starts about a wave
    // later, into L2
    const int64_t m0 = (blk + ahead) * kBlock;
    const int mc = (int)min64(kBlock, g.N - m0);
    prefetch_l2(means + 3 * m0, (uint32_t)(mc * 12));
    prefetch_l2(quats + 4 * m0, (uint32_t)(mc * 16));
    prefetch_l2(scales + 3 * m0, (uint32_t)(mc * 12));
    prefetch_l2(opacities + m0, (uint32_t)(mc * 4));
    prefetch_l2(sh + m0 * K3, (uint32_t)(mc * K3 * 4));
  }
  // A chunk's cameras, first rows and each warp's mask word per camera.  The
  // first chunk is loaded before the parameters and the SH block so that its
  // loads are in flight together with theirs.
  auto load_chunk = [&](int c0) {
    const int nc = min(kCamChunk, g.C - c0);
    if (threadIdx.x < nc) {
      scam[threadIdx.x] = load_cam(cams + 20 * (int64_t)(c0 + threadIdx.x), g.W, g.H);
      s_row0[threadIdx.x] = block_off[(int64_t)(c0 + threadIdx.x) * g.blocks_per_cam + blk];
    }
    if (threadIdx.x < nc * kWarps) {
      const int64_t c = c0 + threadIdx.x / kWarps;
      s_word[threadIdx.x] = mask[(c * g.n_pad + blk * kBlock) / 32 + threadIdx.x % kWarps];
    }
  };
  load_chunk(0);
  if (n < g.N) {
    s_g[threadIdx.x] = load_gauss(means, quats, scales, n);
    s_o[threadIdx.x] = opacities[n];
  }
  // exclusive prefix of the chunk's ns <= 128 slot popcounts into s_pre,
  // 4 consecutive slots a lane (one warp)
  auto chunk_prefix = [&](int ns) {
    int v[4], sum = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int sl = 4 * lane + u;
      v[u] = sl < ns ? __popc(s_word[sl]) : 0;
      sum += v[u];
    }
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += x;
    }
    int run = inc - sum;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int sl = 4 * lane + u;
      if (sl < ns) s_pre[sl] = run;
      run += v[u];
    }
    if (lane == 31) s_pre[ns] = inc;  // the chunk's total
  };
  __syncthreads();  // the first chunk's cameras, rows and words
  // Each warp copies the SH rows of its own 32 Gaussians that some camera
  // sees (a third of the Gaussians of the 15M-Gaussian workload are seen by
  // none; with every camera in the first chunk the words just staged tell,
  // otherwise every row is copied) into the padded shared layout by
  // asynchronous copies: all in flight together, no register staging
  // (which would cap the CTAs per SM), consecutive lanes on consecutive
  // 16-byte (or 4-byte) words.  Warp 0 meanwhile scans the first chunk.
  {
    const uint32_t seen_w =
        g.C <= kCamChunk ? __reduce_or_sync(0xffffffffu, lane < g.C ? s_word[lane * kWarps + warp] : 0u)
                         : 0xFFFFFFFFu;
    const int wrows = max(0, min(32, cnt - 32 * warp));
    const float* src = sh + (n0 + 32 * warp) * K3;
    float* dst = sh_s + 32 * warp * KP;
    if constexpr (rows_sh_vec<DEG>()) {
      constexpr int Q = K3 / 4;  // 16-byte words a row
#pragma unroll 4
      for (int v = lane; v < wrows * Q; v += 32) {
        const int gi = v / Q, qq = v - gi * Q;
        if ((seen_w >> gi) & 1u) cp_async16(&dst[gi * KP + 4 * qq], src + 4 * v);
      }
    } else {
#pragma unroll 8
      for (int f = lane; f < wrows * K3; f += 32) {
        const int gi = f / K3, qq = f - gi * K3;
        if ((seen_w >> gi) & 1u) cp_async4(&dst[gi * KP + qq], src + f);
      }
    }
    if (warp == 0) chunk_prefix(min(kCamChunk, g.C) * kWarps);
    cp_async_wait_all();
  }
  __syncthreads();  // every warp's rows, the parameters and the first chunk's prefix
  auto process = [&](const RowItem& it) {
    const Cam& k = scam[it.cam];
    const GaussIn& gi = s_g[it.g];
    const float* shn = sh_s + it.g * KP;
    Proj P;
    cam_point(k, gi.mx, gi.my, gi.mz, P.px, P.py, P.pz);
    project_rest(k, gi.S, g.W, g.H, P);
    const float idet = rcp_(P.det);
    const float ca = mul(P.c, idet), cb = -mul(P.b, idet), cc2 = mul(P.a, idet);
    float b[16];
    float X = 0.0f, Y = 0.0f, Z = 0.0f, il;
    if (DEG > 0) view_dir(k, gi.mx, gi.my, gi.mz, X, Y, Z, il);
    sh_basis(DEG, X, Y, Z, b);
    float rgb[3];
    if constexpr (rows_sh_vec<DEG>()) {
      // coefficient e = 3 kk + ch in increasing e: each channel's terms come
      // in increasing kk, the canonical order
      float acc[3] = {0.0f, 0.0f, 0.0f};
      const float4* sh4 = reinterpret_cast<const float4*>(shn);
#pragma unroll
      for (int q = 0; q < K3 / 4; ++q) {
        const float4 w = sh4[q];
        const float e4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = 4 * q + u, kk = e / 3, ch = e - 3 * kk;
          acc[ch] = kk == 0 ? mul(e4[u], b[0]) : add(acc[ch], mul(e4[u], b[kk]));
        }
      }
#pragma unroll
      for (int ch = 0; ch < 3; ++ch) rgb[ch] = fmaxf(add(acc[ch], 0.5f), 0.0f);
    } else {
#pragma unroll
      for (int ch = 0; ch < 3; ++ch) {
        float acc = mul(shn[ch], b[0]);
#pragma unroll
        for (int kk = 1; kk < K; ++kk) acc = add(acc, mul(shn[3 * kk + ch], b[kk]));
        rgb[ch] = fmaxf(add(acc, 0.5f), 0.0f);
      }
    }
    float4* out = reinterpret_cast<float4*>(screen + it.row * kRowF);
    out[0] = make_float4(P.mx, P.my, ca, cb);
    out[1] = make_float4(cc2, s_o[it.g], rgb[0], rgb[1]);
    out[2] = make_float4(rgb[2], P.pz, 0.0f, 0.0f);
    const float x0 = fmaxf(sub(P.mx, P.r), 0.0f), x1 = fminf(add(P.mx, P.r), (float)g.W);
    const float y0 = fmaxf(sub(P.my, P.r), 0.0f), y1 = fminf(add(P.my, P.r), (float)g.H);
    uint2 qq;
    qq.x = q16_floor(x0, g.W) | (q16_floor(y0, g.H) << 16);
    qq.y = q16_ceil(x1, g.W) | (q16_ceil(y1, g.H) << 16);
    reinterpret_cast<uint2*>(aabb16)[it.row] = qq;
    row_depth[it.row] = P.pz;
  };
  for (int c0 = 0; c0 < g.C; c0 += kCamChunk) {
    const int nc = min(kCamChunk, g.C - c0);
    const int ns = nc * kWarps;
    if (c0 > 0) {  // the first chunk was loaded and scanned above
      __syncthreads();
      load_chunk(c0);
      __syncthreads();
      if (warp == 0) chunk_prefix(ns);
      __syncthreads();
    }
    const int total = s_pre[ns];
    for (int i = threadIdx.x; i < total; i += kBlock) {
      int lo = 0, hi = ns;  // largest slot j with s_pre[j] <= i
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_pre[mid] <= i) lo = mid; else hi = mid;
      }
      const int cc = lo / kWarps, w = lo - cc * kWarps;
      const int rank = i - s_pre[lo];
      RowItem it;
      it.cam = cc;
      it.g = w * 32 + (int)__fns(s_word[lo], 0, rank + 1);
      it.row = s_row0[cc] + (s_pre[lo] - s_pre[cc * kWarps]) + rank;
      process(it);
    }
  }
}

template <int DEG>
void launch_rows(const Geo& g, unsigned grid, cudaStream_t st, const float* cams, const float* means,
                 const float* quats, const float* scales, const float* opacities, const float* sh,
                 const uint32_t* mask, const int64_t* block_off, float* screen, uint32_t* aabb16,
                 float* row_depth) {
  const int64_t ahead = wave_blocks(k_project_rows<DEG>, kBlock, 0);
  k_project_rows<DEG><<<grid, kBlock, 0, st>>>(g, cams, means, quats, scales, opacities, sh, mask, block_off, screen,
                                               aabb16, row_depth, ahead);
}

size_t cap_temp_bytes(int C);
ss_status apply_visible_cap(const Geo& g, const float* opacities, uint32_t* mask, uint32_t* block_count,
                            const int64_t* block_off, int64_t cap, void* temp, cudaStream_t st, bool* changed);

size_t project_temp_bytes(const Geo& g) {
  return scan_temp_bytes(max64(g.mask_blocks, 1)) + cap_temp_bytes(g.C);
}

}  // namespace ss

using namespace ss;

extern "C" ss_status ss_project_packed(const ss_dims* dims, const float* cams, const float* means,
                                       const float* quats, const float* scales, const float* opacities,
                                       const float* sh, uint32_t* mask, uint32_t* block_count, int64_t* block_off,
                                       float* screen, uint32_t* aabb16, float* row_depth, int64_t cap_rows,
                                       int64_t cap_visible, void* temp,
                                       size_t temp_bytes, int64_t* nnz_out, void* stream) {
  if (!dims_ok(dims)) return invalid("dims");
  if (!nnz_out) return invalid("nnz_out is NULL");
  const Geo g = geometry(*dims);
  cudaStream_t st = as_stream(stream);
  if (!block_off) return invalid("block_off is NULL");
  if (g.N == 0) {
    ss_status s = cuda_status(cudaMemsetAsync(block_off, 0, sizeof(int64_t), st), "memset");
    if (s) return s;
    *nnz_out = 0;
    return SS_OK;
  }
  if (!cams || !means || !quats || !scales || !mask || !block_count) return invalid("null input");
  if (((uintptr_t)quats & 15) != 0 || ((uintptr_t)sh & 15) != 0) return invalid("quats and sh must be 16-byte aligned");
  if (!temp || temp_bytes < ss_workspace_bytes(dims, SS_WS_PROJECT, 0)) return invalid("temp too small");
  const unsigned grid = (unsigned)g.blocks_per_cam;
  k_project_mask<<<grid, kBlock, 0, st>>>(g, cams, means, quats, scales, mask, block_count);
  ss_status s = cuda_status(cudaGetLastError(), "project pass 1");
  if (s) return s;
  ScanSrc src{};
  src.kind = SCAN_U32;
  src.u32 = block_count;
  s = scan_phase1(src, g.mask_blocks, temp, block_off + g.mask_blocks, st);
  if (s) return s;
  s = scan_phase2<int64_t>(src, g.mask_blocks, temp, block_off, st);
  if (s) return s;
  if (cap_visible >= 0) {
    if (!opacities) return invalid("the visible cap needs the opacities");
    if (g.N > (int64_t(1) << 32)) return invalid("the visible cap needs N <= 2^32");
    bool changed = false;
    void* cap_temp = reinterpret_cast<char*>(temp) + scan_temp_bytes(max64(g.mask_blocks, 1));
    s = apply_visible_cap(g, opacities, mask, block_count, block_off, cap_visible, cap_temp, st, &changed);
    if (s) return s;
    if (changed) {
      s = scan_phase1(src, g.mask_blocks, temp, block_off + g.mask_blocks, st);
      if (s) return s;
      s = scan_phase2<int64_t>(src, g.mask_blocks, temp, block_off, st);
      if (s) return s;
    }
  }
  int64_t nnz = 0;
  s = cuda_status(cudaMemcpyAsync(&nnz, block_off + g.mask_blocks, sizeof(int64_t), cudaMemcpyDeviceToHost, st),
                  "copy nnz");
  if (s) return s;
  s = cuda_status(cudaStreamSynchronize(st), "project pass 1 / scan");
  if (s) return s;
  *nnz_out = nnz;
  if (!screen) return SS_OK;
  if (nnz > cap_rows) {
    set_error("ss_project_packed: nnz exceeds cap_rows");
    return SS_ERR_CAPACITY;
  }
  if (!opacities || !sh || !aabb16 || !row_depth) return invalid("null row input/output");
  if (((uintptr_t)screen & 15) != 0 || ((uintptr_t)aabb16 & 7) != 0) return invalid("row buffers misaligned");
  switch (g.deg) {
    case 0: launch_rows<0>(g, grid, st, cams, means, quats, scales, opacities, sh, mask, block_off, screen, aabb16,
                            row_depth);
            break;
    case 1: launch_rows<1>(g, grid, st, cams, means, quats, scales, opacities, sh, mask, block_off, screen, aabb16,
                            row_depth);
            break;
    case 2: launch_rows<2>(g, grid, st, cams, means, quats, scales, opacities, sh, mask, block_off, screen, aabb16,
                            row_depth);
            break;
    default: launch_rows<3>(g, grid, st, cams, means, quats, scales, opacities, sh, mask, block_off, screen, aabb16,
                            row_depth);
  }
  return cuda_status(cudaGetLastError(), "project pass 2");
}
