// Tile intersections ("Spirula Studio VRAM deep-dive", section "4 GiB rule and
// 2^31 limit": the count pass sums an exact 64-bit total, the host checks it
// before any key is written, and the write pass never writes past the
// allocation; key format (tile_id << 32 | depth) from the buffer-cost table).
//
// Rows are written in order of depth.  The sorted keys are ordered by tile,
// then depth, then row; a row's keys all carry its depth, so if the rows are
// visited in (depth, row) order, every tile's keys come out in the right
// order and the key sort needs only the tile-id bytes: a stable sort of the
// nnz rows' 32-bit depths replaces the depth passes over the keys (2.2 keys a
// row on the 15M-Gaussian workload, 59 on the 7680^2 one).
//
//   k_row_keys      (depth bits << 32 | row) of every row, the exact int64
//                   total of tiles covered (integer atomics, one per CTA:
//                   the sum is the same in any order) and the depth bytes'
//                   digit counts, so the depth sort reads no histogram
//   radix sort      keys only, by the depth word (sort.cu; the row index in
//                   the low word rides along, ties stay in row order)
//   (host)          checks the total against the capacity and 2^31
//   k_isect_fused   one CTA per 4096 positions of the depth order, blocks
//                   taken by ticket: decodes its rows once into shared memory
//                   (first tile id and tile columns, from the row's AABB16;
//                   the depth bits and the row id are the row's depth key,
//                   read again at the write), scans their tile counts,
//                   publishes the block's total and looks back over earlier
//                   blocks for its base (decoupled look-back, bounded spin),
//                   writes the rows' offsets to isect_off, then expands the
//                   block's slots 8192 at a time: slot s belongs to the last
//                   row whose offset is <= s (a binary search in shared
//                   memory between the rows of its 64-slot cell, found
//                   first), and consecutive threads write consecutive slots,
//                   so every store is coalesced whatever the per-row counts.
#include "ss_common.cuh"
#include "ss_math.cuh"

namespace ss {

size_t sort_temp_bytes(int64_t n);
ss_status radix_sort_pairs(uint64_t* ka, uint32_t* va, uint64_t* kb, uint32_t* vb, int64_t n, int lo_bytes,
                           int hi_bytes, const uint32_t* given_hist, void* temp, cudaStream_t st, bool* in_b,
                           int64_t* tile_off, int64_t ntiles, bool* ranged);
ss_status radix_sort_flag(const void* temp, cudaStream_t st, bool* flagged);
int tile_bits(int64_t ntiles);

constexpr int kIxThreads = 512;
constexpr int kIxRows = 4096;  // positions of the depth order per CTA
constexpr int kIxPer = kIxRows / kIxThreads;
static_assert(kIxRows % kIxThreads == 0, "rows per thread");
constexpr int kRowKeyThreads = 256;
constexpr int kIxCams = 256;  // cameras whose first rows the write kernel keeps in shared memory
constexpr int kIxChunk = 8192;  // slots expanded per round of the write kernel
constexpr int kIxCell = 64;     // slots per search cell

// Block status of the look-back: flag in the top two bits, count below.
constexpr uint64_t kIxAgg = 1ull << 62;
constexpr uint64_t kIxPre = 2ull << 62;
constexpr uint64_t kIxVal = (1ull << 62) - 1;
constexpr int kIxSpinLimit = 1 << 20;

struct IxSmem {
  uint32_t off[kIxRows + 1];  // slot offset of each row within the block
  uint32_t t0[kIxRows];       // first tile id of the row's range
  uint16_t w[kIxRows];        // tile columns of the row's range
  uint32_t wsum[kIxThreads / 32];
  int64_t cam_row0[kIxCams];  // first row of each camera
  uint32_t cell[kIxChunk / kIxCell + 1];  // row of every kIxCell-th slot of the chunk
  uint32_t hist[4][256];  // digit counts of the written keys' tile-id bytes
  int64_t base;
  uint32_t blk;
};

// Scratch: total (int64) | ticket (u32) | error flag (u32) | block status
// (u64 per block) | the depth keys' digit counts ([4][256] u32), then the
// keys' two buffers and the sort's scratch.
struct IxTemp {
  int64_t* total;
  uint32_t* ticket;
  uint32_t* err;
  uint64_t* status;
  uint32_t* dhist;    // [4][256] digit counts of the depth keys' high word
  size_t head_bytes;  // total .. dhist, cleared per call
  uint64_t *dk_a, *dk_b;
  void* sort;
};

IxTemp isect_temp(void* temp, int64_t nnz) {
  char* p = reinterpret_cast<char*>(temp);
  IxTemp t;
  t.total = reinterpret_cast<int64_t*>(p);
  t.ticket = reinterpret_cast<uint32_t*>(p + 8);
  t.err = reinterpret_cast<uint32_t*>(p + 12);
  t.status = reinterpret_cast<uint64_t*>(p + 16);
  t.dhist = reinterpret_cast<uint32_t*>(p + 16 + (size_t)ceil_div(nnz, kIxRows) * 8);
  t.head_bytes = align_up(16 + (size_t)ceil_div(nnz, kIxRows) * 8 + 4 * 256 * 4, 256);
  p += t.head_bytes;
  t.dk_a = reinterpret_cast<uint64_t*>(p);
  p += align_up((size_t)nnz * 8, 256);
  t.dk_b = reinterpret_cast<uint64_t*>(p);
  p += align_up((size_t)nnz * 8, 256);
  t.sort = p;
  return t;
}

size_t isect_temp_bytes(int64_t nnz) {
  return align_up(16 + (size_t)ceil_div(nnz, kIxRows) * 8 + 4 * 256 * 4, 256) + 2 * align_up((size_t)nnz * 8, 256) +
         sort_temp_bytes(nnz);
}

__device__ __forceinline__ uint32_t row_tiles(const Geo& g, uint2 q, int& tx0, int& ty0, int& w) {
  int tx1, ty1;
  tile_span(q.x & 0xFFFFu, q.y & 0xFFFFu, g.W, g.tiles_x, tx0, tx1);
  tile_span(q.x >> 16, q.y >> 16, g.H, g.tiles_y, ty0, ty1);
  w = tx1 - tx0;
  return (uint32_t)w * (uint32_t)(ty1 - ty0);
}

// Grid-stride over the rows (a few CTAs per SM): one 64-bit atomic per CTA
// for the total, not one per 256 rows.
__global__ __launch_bounds__(kRowKeyThreads) void k_row_keys(Geo g, const float* __restrict__ row_depth,
                                                             const uint32_t* __restrict__ aabb16, int64_t nnz,
                                                             uint64_t* __restrict__ keys,
                                                             int64_t* __restrict__ total,
                                                             uint32_t* __restrict__ dhist) {
  __shared__ unsigned long long ws[kRowKeyThreads / 32];
  __shared__ uint32_t h[4][256];  // the depth bytes' digit counts, for the depth sort
  for (int i = threadIdx.x; i < 4 * 256; i += kRowKeyThreads) (&h[0][0])[i] = 0u;
  __syncthreads();
  unsigned long long cnt = 0;
  for (int64_t r = (int64_t)blockIdx.x * kRowKeyThreads + threadIdx.x; r < nnz;
       r += (int64_t)gridDim.x * kRowKeyThreads) {
    const uint32_t d = __float_as_uint(row_depth[r]);
    keys[r] = ((uint64_t)d << 32) | (uint64_t)r;
#pragma unroll
    for (int b = 0; b < 4; ++b) atomicAdd(&h[b][(d >> (8 * b)) & 0xFFu], 1u);
    int tx0, ty0, w;
    cnt += row_tiles(g, reinterpret_cast<const uint2*>(aabb16)[r], tx0, ty0, w);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long s = 0;
#pragma unroll
    for (int w = 0; w < kRowKeyThreads / 32; ++w) s += ws[w];
    if (s) atomicAdd(reinterpret_cast<unsigned long long*>(total), s);
  }
  for (int i = threadIdx.x; i < 4 * 256; i += kRowKeyThreads) {
    const uint32_t c = (&h[0][0])[i];
    if (c) atomicAdd(dhist + i, c);
  }
}

// Camera of row r: camera c's rows start at block_off[c * blocks_per_cam];
// cam_row0 holds those starts in shared memory for the first kIxCams cameras.
__device__ __forceinline__ int camera_of_row(const int64_t* __restrict__ block_off, const int64_t* cam_row0,
                                             int64_t blocks_per_cam, int C, int64_t r) {
  int lo = 0, hi = C;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    const int64_t start = mid < kIxCams ? cam_row0[mid] : block_off[(int64_t)mid * blocks_per_cam];
    if (start <= r) lo = mid; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ uint64_t ld_volatile(const uint64_t* p) {
  return *reinterpret_cast<const volatile unsigned long long*>(p);
}

__global__ __launch_bounds__(kIxThreads) void k_isect_fused(Geo g, const uint64_t* __restrict__ dkeys,
                                                            const uint32_t* __restrict__ aabb16,
                                                            const int64_t* __restrict__ block_off, int64_t nnz,
                                                            int64_t limit, uint64_t* __restrict__ status,
                                                            uint32_t* __restrict__ ticket, uint32_t* __restrict__ err,
                                                            int64_t* __restrict__ isect_off,
                                                            uint64_t* __restrict__ keys,
                                                            uint32_t* __restrict__ vals,
                                                            uint32_t* __restrict__ key_hist, int hist_bytes) {
  extern __shared__ __align__(16) unsigned char ix_raw[];
  IxSmem& S = *reinterpret_cast<IxSmem*>(ix_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // blocks by ticket: every block this one looks back on belongs to a CTA
  // that is already running
  if (tid == 0) S.blk = atomicAdd(ticket, 1u);
  if (key_hist)
    for (int i = tid; i < 4 * 256; i += kIxThreads) (&S.hist[0][0])[i] = 0u;
  for (int c = tid; c < min(g.C, kIxCams); c += kIxThreads) S.cam_row0[c] = block_off[(int64_t)c * g.blocks_per_cam];
  __syncthreads();
  const int64_t blk = S.blk;
  const int64_t p0 = blk * kIxRows;
  const int nr = (int)min64(kIxRows, nnz - p0);
  // decode the rows of positions p0 .. p0 + nr of the depth order, coalesced
  // in position (row i = k * kIxThreads + tid); counts go to S.off for the scan
#pragma unroll
  for (int k = 0; k < kIxPer; ++k) {
    const int i = k * kIxThreads + tid;
    uint32_t cnt = 0;
    if (i < nr) {
      const uint64_t key = dkeys[p0 + i];
      const uint32_t r = (uint32_t)key;
      int tx0, ty0, w;
      cnt = row_tiles(g, reinterpret_cast<const uint2*>(aabb16)[r], tx0, ty0, w);
      const int c = camera_of_row(block_off, S.cam_row0, g.blocks_per_cam, g.C, (int64_t)r);
      const uint32_t t0 =
          (uint32_t)((uint64_t)c * (uint64_t)g.tiles_per_cam + (uint64_t)ty0 * g.tiles_x + (uint64_t)tx0);
      S.t0[i] = t0;
      S.w[i] = (uint16_t)w;
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
  if (warp == 0) {
    // publish the block's total, then look back: lane j reads block
    // blk - 1 - j of the current window; the nearest inclusive prefix ends
    // the walk, a block that has not published makes the warp wait (bounded)
    if (lane == 0)
      atomicExch(reinterpret_cast<unsigned long long*>(status + blk), (blk == 0 ? kIxPre : kIxAgg) | total);
    int64_t prefix = 0;
    if (blk > 0) {
      int64_t t = blk - 1;
      int spins = 0;
      while (true) {
        const int64_t b = t - lane;
        const uint64_t sv = b >= 0 ? ld_volatile(status + b) : kIxPre;  // before block 0: prefix 0
        const uint32_t pre = __ballot_sync(0xffffffffu, (sv & kIxPre) != 0);
        const uint32_t none = __ballot_sync(0xffffffffu, (sv & (kIxPre | kIxAgg)) == 0);
        // lanes up to the first inclusive one, if no lane before it is unpublished
        const int first_pre = pre ? __ffs(pre) - 1 : 32;
        const int first_none = none ? __ffs(none) - 1 : 32;
        // the published counts before the first unpublished block, up to and
        // including the first inclusive prefix (64-bit sums: prefixes pass 2^32)
        const int take = first_none < first_pre ? first_none : first_pre + 1;
        uint64_t s = lane < take && b >= 0 ? (sv & kIxVal) : 0ull;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        prefix += (int64_t)s;
        if (first_none < first_pre) {
          // block t - first_none has not published yet: wait for it (bounded)
          t -= first_none;
          if (++spins > kIxSpinLimit) {
            if (lane == 0) atomicOr(err, 1u);
            break;
          }
          __nanosleep(64);
          continue;
        }
        if (first_pre < 32) break;
        t -= 32;
      }
      if (lane == 0)
        atomicExch(reinterpret_cast<unsigned long long*>(status + blk), kIxPre | (uint64_t)(prefix + total));
    }
    if (lane == 0) S.base = prefix;
  }
  __syncthreads();
  const int64_t base = S.base;
  for (int i = tid; i < nr; i += kIxThreads) isect_off[p0 + i] = base + (int64_t)S.off[i];
  if (tid == 0 && p0 + nr == nnz) isect_off[nnz] = base + (int64_t)total;  // the last block: the total
  // expand the block's slots, kIxChunk at a time.  A slot's row is the last
  // row whose offset is <= the slot; every kIxCell-th slot of the chunk has
  // its row found first (one binary search per cell over the whole block),
  // so a slot searches only between its cell's bounding rows (about 29 rows
  // on the 15M-Gaussian workload, one or two on the 7680^2 one).  Positions
  // past nr have offset == total and are never found for s < total.
  const uint32_t stop = (uint32_t)max64(0, min64((int64_t)total, limit - base));
  for (uint32_t c0 = 0; c0 < stop; c0 += kIxChunk) {
    __syncthreads();  // the previous chunk's cells are read no more
    for (int j = tid; j <= kIxChunk / kIxCell; j += kIxThreads) {
      const uint32_t sc = min(c0 + (uint32_t)(j * kIxCell), total - 1u);
      int lo = 0, hi = nr;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (S.off[mid] <= sc) lo = mid; else hi = mid;
      }
      S.cell[j] = (uint32_t)lo;
    }
    __syncthreads();
    const uint32_t c1 = min(stop, c0 + (uint32_t)kIxChunk);
    // warp-uniform rounds: a warp's lanes take 32 consecutive slots
    for (uint32_t s0 = c0 + (uint32_t)(warp * 32); s0 < c1; s0 += kIxThreads) {
      const uint32_t s = s0 + (uint32_t)lane;
      const bool live = s < c1;
      uint32_t tile32 = 0;
      if (live) {
        const int j = (int)((s - c0) / kIxCell);
        int lo = (int)S.cell[j], hi = (int)S.cell[j + 1];  // the row is in [lo, hi]
        while (hi > lo) {
          const int mid = (lo + hi + 1) >> 1;
          if (S.off[mid] <= s) lo = mid; else hi = mid - 1;
        }
        const uint32_t k = s - S.off[lo], w = S.w[lo];
        // k / w through the hardware's approximate reciprocal (relative error
        // below 2^-22 with the product's rounding): k < 2^24 is exact in fp32
        // and the quotient is below 2^22, so the estimate's floor is off by at
        // most one, and one correction each way makes it exact
        float rw;
        asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(rw) : "f"((float)w));
        uint32_t ty = (uint32_t)__fmul_rz((float)k, rw);
        if (ty * w > k) --ty;
        if ((ty + 1) * w <= k) ++ty;
        const uint32_t tx = k - ty * w;
        // tile ids fit 32 bits (a key's high word)
        tile32 = S.t0[lo] + ty * (uint32_t)g.tiles_x + tx;
        // the row's depth key (L1-resident): depth bits and row index
        const uint64_t dk = dkeys[p0 + lo];
        keys[base + s] = ((uint64_t)tile32 << 32) | (dk >> 32);
        vals[base + s] = (uint32_t)dk;
      }
      if (key_hist) {
        // the keys' tile-id bytes, counted for the sort: neighbouring slots
        // share their upper bytes (a row's tiles are consecutive ids), so
        // each run of equal digits is added by its first lane
        const uint32_t vmask = __ballot_sync(0xffffffffu, live);
        const uint32_t end_all = 32u - (uint32_t)__clz(vmask);
        const uint32_t above = ~((2u << lane) - 1u);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          if (b >= hist_bytes) break;
          const uint32_t d = (tile32 >> (8 * b)) & 0xFFu;
          const uint32_t prev = __shfl_up_sync(0xffffffffu, d, 1);
          const bool head = live && (lane == 0 || d != prev);
          const uint32_t after = __ballot_sync(0xffffffffu, head) & above;
          if (head) atomicAdd(&S.hist[b][d], (after ? (uint32_t)(__ffs(after) - 1) : end_all) - (uint32_t)lane);
        }
      }
    }
  }
  if (key_hist) {
    __syncthreads();
    for (int i = tid; i < hist_bytes * 256; i += kIxThreads) {
      const uint32_t c = (&S.hist[0][0])[i];
      if (c) atomicAdd(key_hist + i, c);
    }
  }
}

}  // namespace ss

using namespace ss;

extern "C" ss_status ss_intersect_tiles(const ss_dims* dims, const float* row_depth, const uint32_t* aabb16,
                                        const int64_t* block_off, int64_t nnz, int64_t* isect_off, uint64_t* keys,
                                        uint32_t* vals, uint32_t* key_hist, int64_t cap_isects, void* temp,
                                        size_t temp_bytes, uint64_t* n_isects_out, void* stream) {
  if (!dims_ok(dims)) return invalid("dims");
  if (!n_isects_out || !isect_off) return invalid("null output");
  if (nnz < 0) return invalid("nnz < 0");
  if (nnz >= (int64_t(1) << 32)) return invalid("nnz >= 2^32 (32-bit row ids)");
  const Geo g = geometry(*dims);
  cudaStream_t st = as_stream(stream);
  if (key_hist) {
    ss_status s = cuda_status(cudaMemsetAsync(key_hist, 0, 4 * 256 * sizeof(uint32_t), st), "memset");
    if (s) return s;
  }
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
  ss_status s = cuda_status(cudaMemsetAsync(t.total, 0, t.head_bytes, st), "memset");
  if (s) return s;
  // the rows' depth keys and the exact total
  k_row_keys<<<(unsigned)min64(ceil_div(nnz, kRowKeyThreads), 148 * 8), kRowKeyThreads, 0, st>>>(
      g, row_depth, aabb16, nnz, t.dk_a, t.total, t.dhist);
  s = cuda_status(cudaGetLastError(), "row keys");
  if (s) return s;
  // the rows in depth order (ties by row index: the sort is stable and the
  // row index is the key's low word)
  bool in_b = false;
  s = radix_sort_pairs(t.dk_a, nullptr, t.dk_b, nullptr, nnz, 0, 4, t.dhist, t.sort, st, &in_b, nullptr, 0,
                       nullptr);
  if (s) return s;
  const uint64_t* dkeys = in_b ? t.dk_b : t.dk_a;
  int64_t total = 0;
  s = cuda_status(cudaMemcpyAsync(&total, t.total, sizeof(int64_t), cudaMemcpyDeviceToHost, st), "copy n_isects");
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
  s = cuda_status(cudaFuncSetAttribute(k_isect_fused, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sizeof(IxSmem)),
                  "set smem attribute");
  if (s) return s;
  k_isect_fused<<<(unsigned)ceil_div(nnz, kIxRows), kIxThreads, sizeof(IxSmem), st>>>(
      g, dkeys, aabb16, block_off, nnz, limit, t.status, t.ticket, t.err, isect_off, keys, vals, key_hist,
      max(1, (tile_bits(g.n_tiles) + 7) / 8));
  s = cuda_status(cudaGetLastError(), "intersect write");
  if (s) return s;
  // the write's look-back flag (stream sync)
  uint32_t herr = 0;
  s = cuda_status(cudaMemcpyAsync(&herr, t.err, 4, cudaMemcpyDeviceToHost, st), "copy flag");
  if (s) return s;
  s = cuda_status(cudaStreamSynchronize(st), "intersect write");
  if (s) return s;
  if (herr) {
    set_error("ss_intersect_tiles: the write's look-back wait exceeded its limit");
    return SS_ERR_DEVICE_CHECK;
  }
  return SS_OK;
}
