// Tile intersections ("Spirula Studio VRAM deep-dive", section "4 GiB rule and
// 2^31 limit": the count pass sums an exact 64-bit total, the host checks it
// before the offsets are written, and the write pass never writes past the
// allocation; key format (tile_id << 32 | depth) from the buffer-cost table).
//
// Count: per-row tiles from the AABB16 by integer arithmetic, CTA sums per
// 4096 rows and a single-CTA scan of the sums give the exact int64 total (no
// atomics, so the total is deterministic).  Write (k_isect_fused, after the
// host check): one CTA per 4096-row block of the count pass.  It decodes its
// rows once into shared memory (first tile id, tile columns, depth bits; the
// depth comes from the compact per-row array the projection writes, 4 bytes a
// row instead of a 48-byte screen row), scans their tile counts into per-row
// offsets (written to isect_off with the block's base from the count pass),
// then expands the block's slots: slot s belongs to the last row whose offset
// is <= s (binary search in shared memory), and consecutive threads write
// consecutive slots, so every store is coalesced whatever the per-row counts.
#include "ss_common.cuh"
#include "ss_math.cuh"

namespace ss {

constexpr int kIxThreads = 512;
constexpr int kIxRows = (int)kScanTile;  // rows per CTA: the count pass's tiling
constexpr int kIxPer = kIxRows / kIxThreads;
static_assert(kIxRows % kIxThreads == 0, "rows per thread");

struct IxSmem {
  uint32_t off[kIxRows + 1];  // slot offset of each row within the block
  uint32_t t0[kIxRows];       // first tile id of the row's range
  uint32_t dep[kIxRows];      // depth bits
  uint16_t w[kIxRows];        // tile columns of the row's range
  uint32_t wsum[kIxThreads / 32];
};

__global__ __launch_bounds__(kIxThreads) void k_isect_fused(Geo g, const float* __restrict__ row_depth,
                                                            const uint32_t* __restrict__ aabb16,
                                                            const int64_t* __restrict__ block_off,
                                                            const int64_t* __restrict__ partial, int64_t nnz,
                                                            int64_t limit, int64_t* __restrict__ isect_off,
                                                            uint64_t* __restrict__ keys,
                                                            uint32_t* __restrict__ vals) {
  extern __shared__ __align__(16) unsigned char ix_raw[];
  IxSmem& S = *reinterpret_cast<IxSmem*>(ix_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t r0 = (int64_t)blockIdx.x * kIxRows;
  const int nr = (int)min64(kIxRows, nnz - r0);
  // camera of the block's first row (rows are camera-major; camera c starts
  // at block_off[c * blocks_per_cam])
  int c_first = 0;
  {
    int lo = 0, hi = g.C;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (block_off[(int64_t)mid * g.blocks_per_cam] <= r0) lo = mid; else hi = mid;
    }
    c_first = lo;
  }
  // decode the rows, coalesced (row i = k * kIxThreads + tid); counts go to
  // S.off for the scan below
#pragma unroll
  for (int k = 0; k < kIxPer; ++k) {
    const int i = k * kIxThreads + tid;
    uint32_t cnt = 0;
    if (i < nr) {
      const int64_t r = r0 + i;
      const uint2 q = reinterpret_cast<const uint2*>(aabb16)[r];
      int tx0, tx1, ty0, ty1;
      tile_span(q.x & 0xFFFFu, q.y & 0xFFFFu, g.W, g.tiles_x, tx0, tx1);
      tile_span(q.x >> 16, q.y >> 16, g.H, g.tiles_y, ty0, ty1);
      int c = c_first;
      while (c + 1 < g.C && block_off[(int64_t)(c + 1) * g.blocks_per_cam] <= r) ++c;
      const int w = tx1 - tx0;
      cnt = (uint32_t)w * (uint32_t)(ty1 - ty0);
      S.t0[i] = (uint32_t)((uint64_t)c * (uint64_t)g.tiles_per_cam + (uint64_t)ty0 * g.tiles_x + (uint64_t)tx0);
      S.w[i] = (uint16_t)w;
      S.dep[i] = __float_as_uint(row_depth[r]);
    }
    S.off[i] = cnt;
  }
  __syncthreads();
  // exclusive scan of the counts in row order: thread t owns rows
  // [t * kIxPer, (t + 1) * kIxPer); the block's total is < 2^31 (host check)
  uint32_t v[kIxPer], sum = 0;
#pragma unroll
  for (int k = 0; k < kIxPer; ++k) {
    v[k] = S.off[tid * kIxPer + k];
    sum += v[k];
  }
  uint32_t inc = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += x;
  }
  if (lane == 31) S.wsum[warp] = inc;
  __syncthreads();
  uint32_t before = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kIxThreads / 32; ++w) {
    const uint32_t t = S.wsum[w];
    before += w < warp ? t : 0u;
    total += t;
  }
  uint32_t run = before + inc - sum;
#pragma unroll
  for (int k = 0; k < kIxPer; ++k) {
    S.off[tid * kIxPer + k] = run;
    run += v[k];
  }
  if (tid == 0) S.off[kIxRows] = total;
  __syncthreads();
  const int64_t base = partial[blockIdx.x];
  for (int i = tid; i < nr; i += kIxThreads) isect_off[r0 + i] = base + (int64_t)S.off[i];
  // expand the block's slots; rows past nr have offset == total and are never
  // found for s < total
  const uint32_t stop = (uint32_t)min64((int64_t)total, limit - base);
  for (uint32_t s = tid; (int64_t)s < (int64_t)stop; s += kIxThreads) {
    int lo = 0, hi = nr;  // largest i with S.off[i] <= s
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (S.off[mid] <= s) lo = mid; else hi = mid;
    }
    const uint32_t k = s - S.off[lo], w = S.w[lo];
    const uint32_t ty = k / w, tx = k - ty * w;
    const uint64_t tile = (uint64_t)S.t0[lo] + (uint64_t)ty * (uint64_t)g.tiles_x + tx;
    keys[base + s] = (tile << 32) | S.dep[lo];
    vals[base + s] = (uint32_t)(r0 + lo);
  }
}

size_t isect_temp_bytes(int64_t nnz) { return scan_temp_bytes(nnz); }

}  // namespace ss

using namespace ss;

extern "C" ss_status ss_intersect_tiles(const ss_dims* dims, const float* row_depth, const uint32_t* aabb16,
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
  if (!row_depth || !aabb16 || !block_off) return invalid("null input");
  if (((uintptr_t)aabb16 & 7) != 0) return invalid("aabb16 must be 8-byte aligned");
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
  if (total > 0 && (!keys || !vals)) return invalid("null keys/vals");
  const int64_t limit = min64(total, cap_isects);
  const int64_t* partial = reinterpret_cast<const int64_t*>(temp);
  s = cuda_status(cudaFuncSetAttribute(k_isect_fused, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sizeof(IxSmem)),
                  "set smem attribute");
  if (s) return s;
  k_isect_fused<<<(unsigned)ceil_div(nnz, kIxRows), kIxThreads, sizeof(IxSmem), st>>>(
      g, row_depth, aabb16, block_off, partial, nnz, limit, isect_off, keys, vals);
  return cuda_status(cudaGetLastError(), "intersect write");
}
