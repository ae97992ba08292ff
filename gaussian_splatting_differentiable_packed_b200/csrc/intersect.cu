// Tile intersections ("Spirula Studio VRAM deep-dive", section "4 GiB rule and
// 2^31 limit": the count pass sums an exact 64-bit total, the host checks it
// before the offsets are written, and the write pass never writes past the
// allocation; key format (tile_id << 32 | depth) from the buffer-cost table).
//
// Count: per-row tiles from the AABB16 by integer arithmetic, CTA sums and a
// single-CTA scan of the sums give the exact int64 total (no atomics, so the
// total is deterministic).  Offsets: block scan per 4096 rows.  Write: load
// balanced over output slots — each thread owns 8 consecutive slots, finds
// the row of its first slot by binary search in the offsets and walks on, so
// stores are contiguous whatever the per-row tile counts.
#include "ss_common.cuh"
#include "ss_math.cuh"

namespace ss {

constexpr int kWrThreads = 256;
constexpr int kWrItems = 8;
constexpr int64_t kWrTile = (int64_t)kWrThreads * kWrItems;

// Largest r in [lo, hi) with off[r] <= s (off non-decreasing, off[lo] <= s).
__device__ __forceinline__ int64_t find_row(const int64_t* off, int64_t lo, int64_t hi, int64_t s) {
  while (hi - lo > 1) {
    int64_t mid = lo + ((hi - lo) >> 1);
    if (off[mid] <= s) lo = mid; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ int find_cam(const int64_t* block_off, int64_t blocks_per_cam, int C, int64_t r) {
  int lo = 0, hi = C;
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (block_off[(int64_t)mid * blocks_per_cam] <= r) lo = mid; else hi = mid;
  }
  return lo;
}

__global__ __launch_bounds__(kWrThreads) void k_isect_write(Geo g, const float* __restrict__ screen,
                                                            const uint32_t* __restrict__ aabb16,
                                                            const int64_t* __restrict__ block_off,
                                                            const int64_t* __restrict__ off, int64_t nnz,
                                                            int64_t limit, uint64_t* __restrict__ keys,
                                                            uint32_t* __restrict__ vals) {
  __shared__ int64_t s_lo, s_hi;
  const int64_t s0 = (int64_t)blockIdx.x * kWrTile;
  if (threadIdx.x == 0) s_lo = find_row(off, 0, nnz, s0);
  if (threadIdx.x == 1) s_hi = find_row(off, 0, nnz, min(s0 + kWrTile, limit) - 1) + 1;
  __syncthreads();
  int64_t s = s0 + (int64_t)threadIdx.x * kWrItems;
  if (s >= limit) return;
  int64_t r = find_row(off, s_lo, s_hi, s);
  int c = find_cam(block_off, g.blocks_per_cam, g.C, r);
  int64_t r_end = off[r + 1];
  int tx0, tx1, ty0, ty1, w;
  uint32_t dbits;
  auto decode = [&](int64_t row) {
    const uint2 q = reinterpret_cast<const uint2*>(aabb16)[row];
    tile_span(q.x & 0xFFFFu, q.y & 0xFFFFu, g.W, g.tiles_x, tx0, tx1);
    tile_span(q.x >> 16, q.y >> 16, g.H, g.tiles_y, ty0, ty1);
    w = tx1 - tx0;
    dbits = __float_as_uint(screen[row * kRowF + 9]);
  };
  decode(r);
  int64_t k = s - off[r];
  const int64_t s_stop = min(s + kWrItems, limit);
  for (; s < s_stop; ++s, ++k) {
    while (s >= r_end) {  // next row with at least one tile
      ++r;
      r_end = off[r + 1];
      k = 0;
      while (c + 1 < g.C && block_off[(int64_t)(c + 1) * g.blocks_per_cam] <= r) ++c;
      decode(r);
    }
    const int ty = ty0 + (int)(k / w), tx = tx0 + (int)(k % w);
    const uint64_t tile = (uint64_t)c * (uint64_t)g.tiles_per_cam + (uint64_t)ty * g.tiles_x + (uint64_t)tx;
    keys[s] = (tile << 32) | dbits;
    vals[s] = (uint32_t)r;
  }
}

}  // namespace ss

using namespace ss;

extern "C" ss_status ss_intersect_tiles(const ss_dims* dims, const float* screen, const uint32_t* aabb16,
                                        const int64_t* block_off, int64_t nnz, int64_t* isect_off, uint64_t* keys,
                                        uint32_t* vals, int64_t cap_isects, void* temp, size_t temp_bytes,
                                        uint64_t* n_isects_out, void* stream) {
  if (!dims_ok(dims)) return invalid("dims");
  if (!n_isects_out || !isect_off) return invalid("null output");
  if (nnz < 0) return invalid("nnz < 0");
  const Geo g = geometry(*dims);
  cudaStream_t st = as_stream(stream);
  if (nnz == 0) {
    ss_status s = cuda_status(cudaMemsetAsync(isect_off, 0, sizeof(int64_t), st), "memset");
    if (s) return s;
    *n_isects_out = 0;
    return SS_OK;
  }
  if (!screen || !aabb16 || !block_off) return invalid("null input");
  if (!temp || temp_bytes < ss_workspace_bytes(dims, SS_WS_INTERSECT, nnz)) return invalid("temp too small");
  ScanSrc src{};
  src.kind = SCAN_TILES;
  src.aabb16 = aabb16;
  src.W = g.W; src.H = g.H; src.tiles_x = g.tiles_x; src.tiles_y = g.tiles_y;
  ss_status s = scan_phase1(src, nnz, temp, isect_off + nnz, st);
  if (s) return s;
  int64_t total = 0;
  s = cuda_status(cudaMemcpyAsync(&total, isect_off + nnz, sizeof(int64_t), cudaMemcpyDeviceToHost, st),
                  "copy n_isects");
  if (s) return s;
  s = cuda_status(cudaStreamSynchronize(st), "intersect count");
  if (s) return s;
  *n_isects_out = (uint64_t)total;
  if (total > cap_isects) {
    set_error("ss_intersect_tiles: n_isects exceeds cap_isects");
    return SS_ERR_CAPACITY;
  }
  if (total >= (int64_t(1) << 31)) {
    set_error("ss_intersect_tiles: n_isects >= 2^31 (32-bit values and last_id)");
    return SS_ERR_OVERFLOW;
  }
  s = scan_phase2<int64_t>(src, nnz, temp, isect_off, st);
  if (s) return s;
  if (total == 0) return SS_OK;
  if (!keys || !vals) return invalid("null keys/vals");
  const int64_t limit = min64(total, cap_isects);
  const unsigned grid = (unsigned)ceil_div(limit, kWrTile);
  k_isect_write<<<grid, kWrThreads, 0, st>>>(g, screen, aabb16, block_off, isect_off, nnz, limit, keys, vals);
  return cuda_status(cudaGetLastError(), "intersect write");
}
