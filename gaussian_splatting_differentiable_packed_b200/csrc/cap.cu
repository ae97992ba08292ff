// Per-image visible cap ("Spirula Studio VRAM deep-dive", practical guide:
// --cap-max, the cap on the visible splats of each image, which holds down
// nnz and with it the screen rows, the AABBs and the intersection list).
//
// The page gives no selection rule.  Reading: in each camera whose visible
// pairs exceed the cap, keep the cap of highest opacity, ties going to the
// lower Gaussian index.  Each visible pair (c, n) gets the 64-bit priority
//   key(o_n) << 32 | (2^32 - 1 - n),
// key = the IEEE total order of the fp32 opacity as an unsigned word, so the
// priorities of one camera are distinct and the kept set is exactly the cap
// largest.  A radix select finds, per capped camera, the cap-th largest
// priority T_c, 8 bits per pass from the top (k_cap_hist: per-camera digit
// histograms of the pairs whose priority matches the prefix found so far;
// k_cap_pick: the digit where the running count from the top reaches the
// number still to keep).  k_cap_apply then clears the mask bits of pairs below
// T_c and recounts the 128-pair blocks; the caller scans the counts again.
#include <vector>

#include "ss_common.cuh"

namespace ss {

constexpr int kCapDigits = 8;  // 64-bit priority, 8 bits a pass

struct CapState {
  uint32_t* hist;      // [C][256]
  uint64_t* prefix;    // [C] priority bits found so far
  int64_t* remaining;  // [C] pairs still to keep among those matching prefix
  int64_t* cam_off;    // [C + 1] first row of each camera (block_off gather)
  uint32_t* active;    // [C] 1 where the cap binds
};

size_t cap_temp_bytes(int C) {
  return align_up((size_t)C * 256 * 4, 256) + 3 * align_up((size_t)(C + 1) * 8, 256) +
         align_up((size_t)C * 4, 256);
}

CapState cap_state(void* temp, int C) {
  char* p = reinterpret_cast<char*>(temp);
  CapState s;
  s.hist = reinterpret_cast<uint32_t*>(p);
  p += align_up((size_t)C * 256 * 4, 256);
  s.prefix = reinterpret_cast<uint64_t*>(p);
  p += align_up((size_t)(C + 1) * 8, 256);
  s.remaining = reinterpret_cast<int64_t*>(p);
  p += align_up((size_t)(C + 1) * 8, 256);
  s.cam_off = reinterpret_cast<int64_t*>(p);
  p += align_up((size_t)(C + 1) * 8, 256);
  s.active = reinterpret_cast<uint32_t*>(p);
  return s;
}

__device__ __forceinline__ uint64_t cap_priority(float o, int64_t n) {
  const uint32_t b = __float_as_uint(o);
  const uint32_t key = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)n);
}

// cam_off[c] = block_off[c * blocks_per_cam], c = 0..C.
__global__ void k_cap_cam_off(const int64_t* __restrict__ block_off, int C, int64_t blocks_per_cam,
                              int64_t* __restrict__ cam_off) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c <= C) cam_off[c] = block_off[(int64_t)c * blocks_per_cam];
}

// Visible count of each camera against the cap: sets active, remaining = cap,
// prefix = 0, clears the histograms.
__global__ void k_cap_init(const int64_t* __restrict__ cam_off, int C, int64_t cap, uint32_t* __restrict__ hist,
                           uint64_t* __restrict__ prefix, int64_t* __restrict__ remaining,
                           uint32_t* __restrict__ active) {
  const int c = blockIdx.x;
  if (threadIdx.x == 0) {
    active[c] = cam_off[c + 1] - cam_off[c] > cap ? 1u : 0u;
    prefix[c] = 0;
    remaining[c] = cap;
  }
  for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[c * 256 + i] = 0;
}

// Digit histogram of pass `pass` (digit = priority bits [56 - 8 pass, 64 - 8 pass))
// over the visible pairs of active cameras whose higher bits equal the prefix.
// grid (x: strides over the camera's 128-pair blocks, y: camera).
__global__ __launch_bounds__(kBlock) void k_cap_hist(Geo g, const float* __restrict__ opacities,
                                                     const uint32_t* __restrict__ mask,
                                                     const uint32_t* __restrict__ active,
                                                     const uint64_t* __restrict__ prefix, int pass,
                                                     uint32_t* __restrict__ hist) {
  __shared__ uint32_t h[256];
  const int c = blockIdx.y;
  if (!active[c]) return;
  for (int i = threadIdx.x; i < 256; i += kBlock) h[i] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint64_t pre = prefix[c];
  const int shift = 56 - 8 * pass;
  for (int64_t blk = blockIdx.x; blk < g.blocks_per_cam; blk += gridDim.x) {
    const uint32_t word = mask[(c * g.n_pad + blk * kBlock) / 32 + warp];
    if ((word >> lane) & 1u) {
      const int64_t n = blk * kBlock + threadIdx.x;
      const uint64_t p = cap_priority(opacities[n], n);
      if (pass == 0 || (p >> (shift + 8)) == pre) atomicAdd(&h[(p >> shift) & 0xFFu], 1u);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 256; i += kBlock)
    if (h[i]) atomicAdd(&hist[c * 256 + i], h[i]);
}

// Per active camera: the digit d where the count of matching pairs with digit
// > d is below `remaining` and with digit >= d reaches it; prefix gains d,
// remaining drops by the count above d; the histogram is cleared for the next
// pass.  One CTA of 256 threads per camera (thread t holds digit 255 - t).
__global__ __launch_bounds__(256) void k_cap_pick(const uint32_t* __restrict__ active, uint32_t* __restrict__ hist,
                                                  uint64_t* __restrict__ prefix, int64_t* __restrict__ remaining) {
  __shared__ uint32_t wsum[8];
  const int c = blockIdx.x;
  if (!active[c]) return;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int d = 255 - t;
  const uint32_t v = hist[c * 256 + d];
  uint32_t inc = v;  // inclusive count of digits >= d
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += x;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  uint32_t before = 0;
  for (int w = 0; w < warp; ++w) before += wsum[w];
  inc += before;
  const uint32_t above = inc - v;  // count of digits > d
  const int64_t rem = remaining[c];
  __syncthreads();
  if ((int64_t)above < rem && (int64_t)inc >= rem) {
    prefix[c] = (prefix[c] << 8) | (uint64_t)d;
    remaining[c] = rem - (int64_t)above;
  }
  hist[c * 256 + d] = 0;
}

// Clears the mask bits of pairs of active cameras whose priority is below the
// threshold (every pair when the cap is 0) and recounts their blocks.
__global__ __launch_bounds__(kBlock) void k_cap_apply(Geo g, const float* __restrict__ opacities,
                                                      const uint32_t* __restrict__ active,
                                                      const uint64_t* __restrict__ prefix, int64_t cap,
                                                      uint32_t* __restrict__ mask,
                                                      uint32_t* __restrict__ block_count) {
  __shared__ uint32_t wc[kBlock / 32];
  const int c = blockIdx.y;
  if (!active[c]) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint64_t thr = prefix[c];
  for (int64_t blk = blockIdx.x; blk < g.blocks_per_cam; blk += gridDim.x) {
    const int64_t wi = (c * g.n_pad + blk * kBlock) / 32 + warp;
    const uint32_t word = mask[wi];
    bool keep = false;
    if ((word >> lane) & 1u) {
      const int64_t n = blk * kBlock + threadIdx.x;
      keep = cap > 0 && cap_priority(opacities[n], n) >= thr;
    }
    const uint32_t nw = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) {
      mask[wi] = nw;
      wc[warp] = __popc(nw);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t s = 0;
#pragma unroll
      for (int w = 0; w < kBlock / 32; ++w) s += wc[w];
      block_count[c * g.blocks_per_cam + blk] = s;
    }
    __syncthreads();
  }
}

// Applies the cap after pass 1 and the first scan; *changed says whether any
// camera exceeded it (then the caller scans block_count again).  Reads the
// cameras' first rows on the host (one small copy, stream sync) to see
// whether the cap binds anywhere.
ss_status apply_visible_cap(const Geo& g, const float* opacities, uint32_t* mask, uint32_t* block_count,
                            const int64_t* block_off, int64_t cap, void* temp, cudaStream_t st, bool* changed) {
  *changed = false;
  CapState s = cap_state(temp, g.C);
  k_cap_cam_off<<<(unsigned)ceil_div(g.C + 1, 256), 256, 0, st>>>(block_off, g.C, g.blocks_per_cam, s.cam_off);
  k_cap_init<<<(unsigned)g.C, 256, 0, st>>>(s.cam_off, g.C, cap, s.hist, s.prefix, s.remaining, s.active);
  ss_status e = cuda_status(cudaGetLastError(), "visible cap set-up");
  if (e) return e;
  std::vector<int64_t> off((size_t)g.C + 1);
  e = cuda_status(cudaMemcpyAsync(off.data(), s.cam_off, off.size() * 8, cudaMemcpyDeviceToHost, st),
                  "copy camera offsets");
  if (e) return e;
  e = cuda_status(cudaStreamSynchronize(st), "visible cap counts");
  if (e) return e;
  bool any = false;
  for (int c = 0; c < g.C; ++c) any = any || off[c + 1] - off[c] > cap;
  if (!any) return SS_OK;
  const unsigned gx = (unsigned)max64(1, min64(g.blocks_per_cam, ceil_div(148 * 8, g.C)));
  const dim3 grid(gx, (unsigned)g.C);
  if (cap > 0) {
    for (int pass = 0; pass < kCapDigits; ++pass) {
      k_cap_hist<<<grid, kBlock, 0, st>>>(g, opacities, mask, s.active, s.prefix, pass, s.hist);
      k_cap_pick<<<(unsigned)g.C, 256, 0, st>>>(s.active, s.hist, s.prefix, s.remaining);
    }
  }
  k_cap_apply<<<grid, kBlock, 0, st>>>(g, opacities, s.active, s.prefix, cap, mask, block_count);
  e = cuda_status(cudaGetLastError(), "visible cap");
  if (e) return e;
  *changed = true;
  return SS_OK;
}

}  // namespace ss
