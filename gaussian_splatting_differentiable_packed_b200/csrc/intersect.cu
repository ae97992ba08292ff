// Tile intersections ("Spirula Studio VRAM deep-dive", section "4 GiB rule and
// 2^31 limit": the count pass sums an exact 64-bit total, the host checks it
// before the offsets are written, and the write pass never writes past the
// allocation; key format (tile_id << 32 | depth) from the buffer-cost table).
//
// Count: per-row tiles from the AABB16 by integer arithmetic, CTA sums and a
// single-CTA scan of the sums give the exact int64 total (no atomics, so the
// total is deterministic).  Offsets: block scan per 4096 rows.  Write: load
// balanced over output slots — each thread owns 8 consecutive slots of a
// 2048-slot chunk, finds the row of its first slot by binary search in the
// chunk's row range (each chunk's first row comes from one pass over the
// rows) and walks on; the chunk is staged in shared memory and stored
// contiguously, whatever the per-row tile counts.
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

// Slots [s, s_stop) of rows starting at row r, into the CTA's staging arrays.
__device__ __forceinline__ void slot_run(const Geo& g, const float* __restrict__ screen,
                                         const uint32_t* __restrict__ aabb16, const int64_t* __restrict__ block_off,
                                         const int64_t* __restrict__ off, int64_t r, int64_t s, int64_t s_stop,
                                         int64_t s0, uint64_t* s_key, uint32_t* s_val) {
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
    const int64_t i = s - s0;
    s_key[i + i / kWrItems] = (tile << 32) | dbits;
    s_val[i + i / kWrItems] = (uint32_t)r;
  }
}

// first[k] = the row holding slot k * kWrTile, for every chunk start below
// limit (one thread per row; a row spanning several chunk starts writes each).
__global__ void k_chunk_first(const int64_t* __restrict__ off, int64_t nnz, int64_t limit,
                              int64_t* __restrict__ first) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= nnz) return;
  const int64_t a = off[r], b = min64(off[r + 1], limit);
  for (int64_t k = (a + kWrTile - 1) / kWrTile; k * kWrTile < b; ++k) first[k] = r;
}

// One CTA per 2048-slot chunk; the chunk's rows are first[blk] .. first[blk+1].
__global__ __launch_bounds__(kWrThreads) void k_isect_write(Geo g, const float* __restrict__ screen,
                                                            const uint32_t* __restrict__ aabb16,
                                                            const int64_t* __restrict__ block_off,
                                                            const int64_t* __restrict__ off, int64_t nnz,
                                                            int64_t limit, const int64_t* __restrict__ first,
                                                            uint64_t* __restrict__ keys, uint32_t* __restrict__ vals) {
  // the chunk's slots, written back coalesced; one pad word after every
  // kWrItems so that a thread's run of kWrItems slots does not share banks
  // with its neighbours' runs
  __shared__ uint64_t s_key[kWrTile + kWrThreads];
  __shared__ uint32_t s_val[kWrTile + kWrThreads];
  const int64_t blk = blockIdx.x;
  const int64_t nch = (limit + kWrTile - 1) / kWrTile;
  const int64_t s0 = blk * kWrTile;
  const int64_t s_end = min64(s0 + kWrTile, limit);
  const int64_t lo = first[blk], hi = blk + 1 < nch ? first[blk + 1] + 1 : nnz;
  const int64_t s = s0 + (int64_t)threadIdx.x * kWrItems;
  if (s < s_end)
    slot_run(g, screen, aabb16, block_off, off, find_row(off, lo, hi, s), s, min64(s + kWrItems, s_end), s0, s_key,
             s_val);
  __syncthreads();
  const int cnt = (int)(s_end - s0);
  for (int i = threadIdx.x; i < cnt; i += kWrThreads) {
    keys[s0 + i] = s_key[i + i / kWrItems];
    vals[s0 + i] = s_val[i + i / kWrItems];
  }
}

// Workspace: the scan's scratch, then first[] for the largest chunk count
// (n_isects < 2^31).
constexpr int64_t kMaxChunks = ((int64_t(1) << 31) + kWrTile - 1) / kWrTile;
size_t isect_temp_bytes(int64_t nnz) {
  return scan_temp_bytes(nnz) + align_up((size_t)(kMaxChunks + 1) * sizeof(int64_t), 256);
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
  const int64_t nch = ceil_div(limit, kWrTile);
  int64_t* first = reinterpret_cast<int64_t*>(reinterpret_cast<char*>(temp) + scan_temp_bytes(nnz));
  k_chunk_first<<<(unsigned)ceil_div(nnz, 256), 256, 0, st>>>(isect_off, nnz, limit, first);
  k_isect_write<<<(unsigned)nch, kWrThreads, 0, st>>>(g, screen, aabb16, block_off, isect_off, nnz, limit, first, keys,
                                                      vals);
  return cuda_status(cudaGetLastError(), "intersect write");
}
