// Tile intersections ("Spirula Studio VRAM deep-dive", section "4 GiB rule and
// 2^31 limit": the count pass sums an exact 64-bit total, the host checks it
// before any key is written, and the write pass never writes past the
// allocation; key format (tile_id << 32 | depth) from the buffer-cost table).
//
// Rows are written in order of depth.  The sorted keys are ordered by tile,
// then depth, then row; a row's keys all carry its depth, so if the rows are
// visited in (depth, row) order, every tile's keys come out in the right
// order and the key sort needs only the tile-id bytes: a stable sort of the
// nnz rows' 32-bit depths (4 byte passes over 12 bytes a row) replaces the 4
// depth passes over the 12-byte keys (2.2 keys a row on the 15M-Gaussian
// workload, 59 on the 7680^2 one).
//
//   k_row_keys      (depth bits, row) of every row
//   radix sort      stable, by depth (sort.cu)
//   count           per-row tiles from the AABB16 by integer arithmetic, in
//                   depth order: CTA sums per 4096 rows and a single-CTA scan
//                   give the exact int64 total (no atomics: deterministic)
//   k_isect_fused   (after the host check) one CTA per 4096 rows of the depth
//                   order: decodes its rows once into shared memory (first
//                   tile id, tile columns, depth bits), scans their tile
//                   counts into offsets (written to isect_off with the block's
//                   base from the count), then expands the block's slots: slot
//                   s belongs to the last row whose offset is <= s (binary
//                   search in shared memory), and consecutive threads write
//                   consecutive slots, so every store is coalesced whatever
//                   the per-row counts.
#include "ss_common.cuh"
#include "ss_math.cuh"

namespace ss {

size_t sort_temp_bytes(int64_t n);
ss_status radix_sort_pairs(uint64_t* ka, uint32_t* va, uint64_t* kb, uint32_t* vb, int64_t n, int lo_bytes,
                           int hi_bytes, void* temp, cudaStream_t st, bool* in_b);
ss_status radix_sort_flag(const void* temp, cudaStream_t st, bool* flagged);

constexpr int kIxThreads = 512;
constexpr int kIxRows = (int)kScanTile;  // rows per CTA: the count pass's tiling
constexpr int kIxPer = kIxRows / kIxThreads;
static_assert(kIxRows % kIxThreads == 0, "rows per thread");

struct IxSmem {
  uint32_t off[kIxRows + 1];  // slot offset of each row within the block
  uint32_t t0[kIxRows];       // first tile id of the row's range
  uint32_t dep[kIxRows];      // depth bits
  uint32_t row[kIxRows];      // row index
  uint16_t w[kIxRows];        // tile columns of the row's range
  uint32_t wsum[kIxThreads / 32];
};

__global__ void k_row_keys(const float* __restrict__ row_depth, int64_t nnz, uint64_t* __restrict__ keys,
                           uint32_t* __restrict__ rows) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= nnz) return;
  keys[r] = (uint64_t)__float_as_uint(row_depth[r]);
  rows[r] = (uint32_t)r;
}

__device__ __forceinline__ int camera_of_row(const int64_t* __restrict__ block_off, int64_t blocks_per_cam, int C,
                                             int64_t r) {
  int lo = 0, hi = C;  // camera c starts at row block_off[c * blocks_per_cam]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (block_off[(int64_t)mid * blocks_per_cam] <= r) lo = mid; else hi = mid;
  }
  return lo;
}

__global__ __launch_bounds__(kIxThreads) void k_isect_fused(Geo g, const uint64_t* __restrict__ dkeys,
                                                            const uint32_t* __restrict__ rows,
                                                            const uint32_t* __restrict__ aabb16,
                                                            const int64_t* __restrict__ block_off,
                                                            const int64_t* __restrict__ partial, int64_t nnz,
                                                            int64_t limit, int64_t* __restrict__ isect_off,
                                                            uint64_t* __restrict__ keys,
                                                            uint32_t* __restrict__ vals) {
  extern __shared__ __align__(16) unsigned char ix_raw[];
  IxSmem& S = *reinterpret_cast<IxSmem*>(ix_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t p0 = (int64_t)blockIdx.x * kIxRows;
  const int nr = (int)min64(kIxRows, nnz - p0);
  // decode the rows of positions p0 .. p0 + nr of the depth order, coalesced
  // in position (row i = k * kIxThreads + tid); counts go to S.off for the scan
#pragma unroll
  for (int k = 0; k < kIxPer; ++k) {
    const int i = k * kIxThreads + tid;
    uint32_t cnt = 0;
    if (i < nr) {
      const uint32_t r = rows[p0 + i];
      const uint2 q = reinterpret_cast<const uint2*>(aabb16)[r];
      int tx0, tx1, ty0, ty1;
      tile_span(q.x & 0xFFFFu, q.y & 0xFFFFu, g.W, g.tiles_x, tx0, tx1);
      tile_span(q.x >> 16, q.y >> 16, g.H, g.tiles_y, ty0, ty1);
      const int c = camera_of_row(block_off, g.blocks_per_cam, g.C, (int64_t)r);
      const int w = tx1 - tx0;
      cnt = (uint32_t)w * (uint32_t)(ty1 - ty0);
      S.t0[i] = (uint32_t)((uint64_t)c * (uint64_t)g.tiles_per_cam + (uint64_t)ty0 * g.tiles_x + (uint64_t)tx0);
      S.w[i] = (uint16_t)w;
      S.dep[i] = (uint32_t)dkeys[p0 + i];
      S.row[i] = r;
    }
    S.off[i] = cnt;
  }
  __syncthreads();
  // exclusive scan of the counts in position order: thread t owns positions
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
  for (int i = tid; i < nr; i += kIxThreads) isect_off[p0 + i] = base + (int64_t)S.off[i];
  // expand the block's slots; positions past nr have offset == total and are
  // never found for s < total
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
    vals[base + s] = S.row[lo];
  }
}

// Workspace: the count's scratch | row depth keys a, b (u64) | row ids a, b
// (u32) | the row sort's scratch.
struct IxTemp {
  void* scan;
  uint64_t *dk_a, *dk_b;
  uint32_t *rows_a, *rows_b;
  void* sort;
};

IxTemp isect_temp(void* temp, int64_t nnz) {
  char* p = reinterpret_cast<char*>(temp);
  IxTemp t;
  t.scan = p;
  p += scan_temp_bytes(nnz);
  t.dk_a = reinterpret_cast<uint64_t*>(p);
  p += align_up((size_t)nnz * 8, 256);
  t.dk_b = reinterpret_cast<uint64_t*>(p);
  p += align_up((size_t)nnz * 8, 256);
  t.rows_a = reinterpret_cast<uint32_t*>(p);
  p += align_up((size_t)nnz * 4, 256);
  t.rows_b = reinterpret_cast<uint32_t*>(p);
  p += align_up((size_t)nnz * 4, 256);
  t.sort = p;
  return t;
}

size_t isect_temp_bytes(int64_t nnz) {
  return scan_temp_bytes(nnz) + 2 * align_up((size_t)nnz * 8, 256) + 2 * align_up((size_t)nnz * 4, 256) +
         sort_temp_bytes(nnz);
}

}  // namespace ss

using namespace ss;

extern "C" ss_status ss_intersect_tiles(const ss_dims* dims, const float* row_depth, const uint32_t* aabb16,
                                        const int64_t* block_off, int64_t nnz, int64_t* isect_off, uint64_t* keys,
                                        uint32_t* vals, int64_t cap_isects, void* temp, size_t temp_bytes,
                                        uint64_t* n_isects_out, void* stream) {
  if (!dims_ok(dims)) return invalid("dims");
  if (!n_isects_out || !isect_off) return invalid("null output");
  if (nnz < 0) return invalid("nnz < 0");
  if (nnz >= (int64_t(1) << 32)) return invalid("nnz >= 2^32 (32-bit row ids)");
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
  const IxTemp t = isect_temp(temp, nnz);
  // the rows in depth order (ties by row index: the sort is stable)
  k_row_keys<<<(unsigned)ceil_div(nnz, 256), 256, 0, st>>>(row_depth, nnz, t.dk_a, t.rows_a);
  ss_status s = cuda_status(cudaGetLastError(), "row keys");
  if (s) return s;
  bool in_b = false;
  s = radix_sort_pairs(t.dk_a, t.rows_a, t.dk_b, t.rows_b, nnz, 4, 0, t.sort, st, &in_b);
  if (s) return s;
  const uint64_t* dkeys = in_b ? t.dk_b : t.dk_a;
  const uint32_t* rows = in_b ? t.rows_b : t.rows_a;
  // the exact total, counted in that order
  ScanSrc src{};
  src.kind = SCAN_TILES_ORDERED;
  src.aabb16 = aabb16;
  src.rows = rows;
  src.W = g.W; src.H = g.H; src.tiles_x = g.tiles_x; src.tiles_y = g.tiles_y;
  s = scan_phase1(src, nnz, t.scan, isect_off + nnz, st);
  if (s) return s;
  int64_t total = 0;
  s = cuda_status(cudaMemcpyAsync(&total, isect_off + nnz, sizeof(int64_t), cudaMemcpyDeviceToHost, st),
                  "copy n_isects");
  if (s) return s;
  bool flagged = false;
  s = radix_sort_flag(t.sort, st, &flagged);  // synchronises the stream
  if (s) return s;
  if (flagged) {
    set_error("ss_intersect_tiles: the depth sort's look-back wait exceeded its limit");
    return SS_ERR_DEVICE_CHECK;
  }
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
  const int64_t* partial = reinterpret_cast<const int64_t*>(t.scan);
  s = cuda_status(cudaFuncSetAttribute(k_isect_fused, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sizeof(IxSmem)),
                  "set smem attribute");
  if (s) return s;
  k_isect_fused<<<(unsigned)ceil_div(nnz, kIxRows), kIxThreads, sizeof(IxSmem), st>>>(
      g, dkeys, rows, aabb16, block_off, partial, nnz, limit, isect_off, keys, vals);
  return cuda_status(cudaGetLastError(), "intersect write");
}
