// Stable LSD radix sort of (key, value) pairs on the (tile_id << 32 | depth)
// keys ("Spirula Studio VRAM deep-dive", buffer-cost table: double-buffered
// isect.ids_a/b; the reference's CUDA backend calls a library sort, this one is
// written here).  8-bit digits over the 31 depth bits (depth > 0, so bit 31 is
// zero) and over the bits the tile ids need.  Per pass, reduce-then-scan:
//   k_radix_hist     per 4096-key tile: digit histogram -> counts[digit][tile]
//   scan             exclusive scan of counts (digit-major) -> offsets
//   k_radix_scatter  per tile: stable rank of each key among equal digits
//                    (warp match + per-warp counters), keys staged in shared
//                    memory in digit order, then written out in contiguous runs
// No CTA waits on another.  Equal keys keep their input order.
#include <algorithm>
#include <utility>

#include "ss_common.cuh"

namespace ss {

constexpr int kSortThreads = 256;
constexpr int kSortItems = 16;
constexpr int kSortTile = kSortThreads * kSortItems;  // 4096 keys per CTA
constexpr int kRadix = 256;
constexpr int kSortWarps = kSortThreads / 32;

__global__ __launch_bounds__(kSortThreads) void k_radix_hist(const uint64_t* __restrict__ keys, int64_t n, int shift,
                                                             uint32_t* __restrict__ counts, int64_t ntiles) {
  __shared__ uint32_t h[kSortWarps][kRadix];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kSortWarps * kRadix; i += kSortThreads) (&h[0][0])[i] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kSortTile + warp * (kSortTile / kSortWarps);
#pragma unroll 4
  for (int r = 0; r < kSortItems; ++r) {
    const int64_t i = base + r * 32 + lane;
    const bool valid = i < n;
    const uint32_t d = valid ? (uint32_t)(keys[i] >> shift) & 0xFFu : 0x100u;
    const uint32_t peers = __match_any_sync(0xffffffffu, d);
    if (valid && lane == 31 - __clz(peers)) h[warp][d] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  uint32_t s = 0;
#pragma unroll
  for (int w = 0; w < kSortWarps; ++w) s += h[w][threadIdx.x];
  counts[(int64_t)threadIdx.x * ntiles + blockIdx.x] = s;
}

struct ScatterSmem {
  uint32_t wcnt[kSortWarps][kRadix];
  uint32_t dstart[kRadix];
  uint32_t gbase[kRadix];
  uint32_t wtot[kSortWarps + 1];
  uint64_t k[kSortTile];
  uint32_t v[kSortTile];
};

__global__ __launch_bounds__(kSortThreads) void k_radix_scatter(const uint64_t* __restrict__ kin,
                                                                const uint32_t* __restrict__ vin,
                                                                uint64_t* __restrict__ kout,
                                                                uint32_t* __restrict__ vout, int64_t n, int shift,
                                                                const uint32_t* __restrict__ offs, int64_t ntiles) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ScatterSmem& S = *reinterpret_cast<ScatterSmem*>(smem_raw);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kSortWarps * kRadix; i += kSortThreads) (&S.wcnt[0][0])[i] = 0;
  __syncthreads();
  const int64_t tile0 = (int64_t)blockIdx.x * kSortTile;
  const int64_t base = tile0 + warp * (kSortTile / kSortWarps);
  const uint32_t lt = (1u << lane) - 1u;
  uint64_t kk[kSortItems];
  uint32_t vv[kSortItems];
  uint32_t pos[kSortItems];
#pragma unroll
  for (int r = 0; r < kSortItems; ++r) {
    const int64_t i = base + r * 32 + lane;
    const bool valid = i < n;
    kk[r] = valid ? kin[i] : 0ull;
    vv[r] = valid ? vin[i] : 0u;
    const uint32_t d = valid ? (uint32_t)(kk[r] >> shift) & 0xFFu : 0x100u;
    const uint32_t peers = __match_any_sync(0xffffffffu, d);
    const uint32_t before = valid ? S.wcnt[warp][d] : 0u;
    __syncwarp();
    if (valid && lane == 31 - __clz(peers)) S.wcnt[warp][d] = before + __popc(peers);
    __syncwarp();
    pos[r] = valid ? before + __popc(peers & lt) : 0xFFFFFFFFu;
  }
  __syncthreads();
  // per digit: exclusive prefix over warps, digit totals, then exclusive scan over digits
  {
    const int d = threadIdx.x;
    uint32_t run = 0;
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) {
      const uint32_t t = S.wcnt[w][d];
      S.wcnt[w][d] = run;
      run += t;
    }
    // block exclusive scan of run over the 256 digits
    uint32_t inc = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += x;
    }
    if (lane == 31) S.wtot[warp] = inc;
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t a = 0;
      for (int w = 0; w < kSortWarps; ++w) {
        const uint32_t t = S.wtot[w];
        S.wtot[w] = a;
        a += t;
      }
    }
    __syncthreads();
    S.dstart[d] = S.wtot[warp] + inc - run;
    S.gbase[d] = offs[(int64_t)d * ntiles + blockIdx.x];
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kSortItems; ++r) {
    if (pos[r] == 0xFFFFFFFFu) continue;
    const uint32_t d = (uint32_t)(kk[r] >> shift) & 0xFFu;
    const uint32_t lp = S.dstart[d] + S.wcnt[warp][d] + pos[r];
    S.k[lp] = kk[r];
    S.v[lp] = vv[r];
  }
  __syncthreads();
  const int cnt = (int)min64(kSortTile, n - tile0);
  for (int i = threadIdx.x; i < cnt; i += kSortThreads) {
    const uint64_t key = S.k[i];
    const uint32_t d = (uint32_t)(key >> shift) & 0xFFu;
    const int64_t gpos = (int64_t)S.gbase[d] + (i - (int64_t)S.dstart[d]);
    kout[gpos] = key;
    vout[gpos] = S.v[i];
  }
}

// tile_off[t] = first sorted index whose tile id is >= t; tile_off[ntiles] = n.
__global__ void k_tile_ranges(const uint64_t* __restrict__ keys, int64_t n, int64_t ntiles,
                              int64_t* __restrict__ tile_off) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i > n) return;
  const int64_t prev = i == 0 ? -1 : (int64_t)(keys[i - 1] >> 32);
  const int64_t cur = i == n ? ntiles : (int64_t)(keys[i] >> 32);
  for (int64_t t = prev + 1; t <= cur && t <= ntiles; ++t) tile_off[t] = i;
}

int tile_bits(int64_t ntiles) {
  int b = 0;
  while ((int64_t(1) << b) < ntiles) ++b;
  return b;
}

int sort_passes(int64_t ntiles) { return 4 + (tile_bits(ntiles) + 7) / 8; }

size_t sort_temp_bytes(int64_t n) {
  const int64_t tiles = ceil_div(max64(n, 1), kSortTile);
  const size_t counts = align_up((size_t)tiles * kRadix * 4, 256);
  return 2 * counts + scan_temp_bytes(tiles * kRadix) + 256;
}

}  // namespace ss

using namespace ss;

extern "C" ss_status ss_sort_isects(const ss_dims* dims, uint64_t* keys_a, uint32_t* vals_a, uint64_t* keys_b,
                                    uint32_t* vals_b, int64_t n, void* temp, size_t temp_bytes, int64_t* tile_off,
                                    int* result_in_b_out, void* stream) {
  if (!dims_ok(dims)) return invalid("dims");
  if (!result_in_b_out || !tile_off) return invalid("null output");
  if (n < 0) return invalid("n < 0");
  if (n >= (int64_t(1) << 31)) {
    set_error("ss_sort_isects: n >= 2^31");
    return SS_ERR_OVERFLOW;
  }
  const Geo g = geometry(*dims);
  cudaStream_t st = as_stream(stream);
  const int passes = sort_passes(g.n_tiles);
  *result_in_b_out = passes & 1;
  if (n == 0) return cuda_status(cudaMemsetAsync(tile_off, 0, sizeof(int64_t) * (g.n_tiles + 1), st), "memset");
  if (!keys_a || !vals_a || !keys_b || !vals_b) return invalid("null keys/vals");
  if (!temp || temp_bytes < sort_temp_bytes(n)) return invalid("temp too small");
  static bool attr_set = false;
  if (!attr_set) {
    ss_status s = cuda_status(cudaFuncSetAttribute(k_radix_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)sizeof(ScatterSmem)),
                              "set smem attribute");
    if (s) return s;
    attr_set = true;
  }
  const int64_t tiles = ceil_div(n, kSortTile);
  const size_t counts_b = align_up((size_t)tiles * kRadix * 4, 256);
  uint32_t* counts = reinterpret_cast<uint32_t*>(temp);
  uint32_t* offs = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(temp) + counts_b);
  char* scan_tmp = reinterpret_cast<char*>(temp) + 2 * counts_b;
  int64_t* scan_total = reinterpret_cast<int64_t*>(scan_tmp + scan_temp_bytes(tiles * kRadix));
  uint64_t* kin = keys_a;
  uint32_t* vin = vals_a;
  uint64_t* kout = keys_b;
  uint32_t* vout = vals_b;
  const int tb = tile_bits(g.n_tiles);
  for (int p = 0; p < passes; ++p) {
    const int shift = p < 4 ? 8 * p : 32 + 8 * (p - 4);
    (void)tb;
    k_radix_hist<<<(unsigned)tiles, kSortThreads, 0, st>>>(kin, n, shift, counts, tiles);
    ss_status s = cuda_status(cudaGetLastError(), "radix histogram");
    if (s) return s;
    ScanSrc src{};
    src.kind = SCAN_U32;
    src.u32 = counts;
    s = scan_phase1(src, tiles * kRadix, scan_tmp, scan_total, st);
    if (s) return s;
    s = scan_phase2<uint32_t>(src, tiles * kRadix, scan_tmp, offs, st);
    if (s) return s;
    k_radix_scatter<<<(unsigned)tiles, kSortThreads, sizeof(ScatterSmem), st>>>(kin, vin, kout, vout, n, shift,
                                                                                offs, tiles);
    s = cuda_status(cudaGetLastError(), "radix scatter");
    if (s) return s;
    std::swap(kin, kout);
    std::swap(vin, vout);
  }
  const unsigned grid = (unsigned)ceil_div(n + 1, 256);
  k_tile_ranges<<<grid, 256, 0, st>>>(kin, n, g.n_tiles, tile_off);
  return cuda_status(cudaGetLastError(), "tile ranges");
}
