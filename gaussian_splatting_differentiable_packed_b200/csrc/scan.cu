// Device-wide exclusive scan with a 64-bit running total, reduce-then-scan:
//   k_partials  one CTA per 4096 items: the tile's sum (int64)
//   k_scan_tops one CTA: exclusive scan of the tile sums, total -> *total
//   k_offsets   one CTA per 4096 items: block scan + tile offset -> out[i]
// No inter-CTA waiting.  Used for the block-count scan of the packed
// projection ("Spirula Studio VRAM deep-dive", section "bitmask compaction":
// only C*N/128 counts are scanned) and for the per-row tile counts of the
// intersection pass (section "4 GiB rule": exact 64-bit totals).
#include "ss_common.cuh"
#include "ss_math.cuh"

namespace ss {

__device__ __forceinline__ int64_t item_count(const ScanSrc& s, int64_t i) {
  if (s.kind == SCAN_U32) return (int64_t)s.u32[i];
  uint32_t w0 = s.aabb16[2 * i], w1 = s.aabb16[2 * i + 1];
  int tx0, tx1, ty0, ty1;
  tile_span(w0 & 0xFFFFu, w1 & 0xFFFFu, s.W, s.tiles_x, tx0, tx1);
  tile_span(w0 >> 16, w1 >> 16, s.H, s.tiles_y, ty0, ty1);
  return (int64_t)(tx1 - tx0) * (int64_t)(ty1 - ty0);
}

__device__ __forceinline__ int64_t warp_incl_scan(int64_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int64_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Exclusive block scan of one value per thread (blockDim = kScanThreads).
__device__ __forceinline__ int64_t block_excl_scan(int64_t v, int64_t* warp_tot, int64_t& block_total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t inc = warp_incl_scan(v);
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int64_t t = lane < kScanThreads / 32 ? warp_tot[lane] : 0;
    int64_t ti = warp_incl_scan(t);
    if (lane < kScanThreads / 32) warp_tot[lane] = ti - t;
    if (lane == kScanThreads / 32 - 1) warp_tot[kScanThreads / 32] = ti;
  }
  __syncthreads();
  int64_t ex = warp_tot[warp] + inc - v;
  block_total = warp_tot[kScanThreads / 32];
  __syncthreads();
  return ex;
}

__global__ __launch_bounds__(kScanThreads) void k_partials(ScanSrc src, int64_t n, int64_t* partial) {
  __shared__ int64_t wt[kScanThreads / 32 + 1];
  const int64_t base = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * kScanItems;
  int64_t s = 0;
#pragma unroll 4
  for (int k = 0; k < kScanItems; ++k) {
    int64_t i = base + k;
    if (i < n) s += item_count(src, i);
  }
  int64_t tot;
  block_excl_scan(s, wt, tot);
  if (threadIdx.x == 0) partial[blockIdx.x] = tot;
}

// One CTA: exclusive scan of nparts partial sums in place; total to *total.
__global__ __launch_bounds__(1024) void k_scan_tops(int64_t* partial, int64_t nparts, int64_t* total) {
  __shared__ int64_t wt[33];
  __shared__ int64_t carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int64_t base = 0; base < nparts; base += 1024) {
    int64_t i = base + threadIdx.x;
    int64_t v = i < nparts ? partial[i] : 0;
    int64_t inc = warp_incl_scan(v);
    if (lane == 31) wt[warp] = inc;
    __syncthreads();
    if (warp == 0) {
      int64_t t = wt[lane];
      int64_t ti = warp_incl_scan(t);
      wt[lane] = ti - t;
      if (lane == 31) wt[32] = ti;
    }
    __syncthreads();
    int64_t ex = carry + wt[warp] + inc - v;
    if (i < nparts) partial[i] = ex;
    __syncthreads();
    if (threadIdx.x == 0) carry += wt[32];
    __syncthreads();
  }
  if (threadIdx.x == 0) *total = carry;
}

template <typename OutT>
__global__ __launch_bounds__(kScanThreads) void k_offsets(ScanSrc src, int64_t n, const int64_t* partial,
                                                          OutT* out) {
  __shared__ int64_t wt[kScanThreads / 32 + 1];
  const int64_t base = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * kScanItems;
  int64_t v[kScanItems];
  int64_t s = 0;
#pragma unroll
  for (int k = 0; k < kScanItems; ++k) {
    int64_t i = base + k;
    v[k] = i < n ? item_count(src, i) : 0;
    s += v[k];
  }
  int64_t tot;
  int64_t run = block_excl_scan(s, wt, tot) + partial[blockIdx.x];
#pragma unroll
  for (int k = 0; k < kScanItems; ++k) {
    int64_t i = base + k;
    if (i < n) out[i] = (OutT)run;
    run += v[k];
  }
}

ss_status scan_phase1(const ScanSrc& src, int64_t n, void* temp, int64_t* total_dev, cudaStream_t st) {
  int64_t* partial = reinterpret_cast<int64_t*>(temp);
  int64_t nparts = ceil_div(n, kScanTile);
  if (nparts > 0) k_partials<<<(unsigned)nparts, kScanThreads, 0, st>>>(src, n, partial);
  k_scan_tops<<<1, 1024, 0, st>>>(partial, nparts, total_dev);
  return cuda_status(cudaGetLastError(), "scan phase 1");
}

template <typename OutT>
ss_status scan_phase2(const ScanSrc& src, int64_t n, void* temp, OutT* out, cudaStream_t st) {
  const int64_t* partial = reinterpret_cast<const int64_t*>(temp);
  int64_t nparts = ceil_div(n, kScanTile);
  if (nparts > 0) k_offsets<OutT><<<(unsigned)nparts, kScanThreads, 0, st>>>(src, n, partial, out);
  return cuda_status(cudaGetLastError(), "scan phase 2");
}

template ss_status scan_phase2<int64_t>(const ScanSrc&, int64_t, void*, int64_t*, cudaStream_t);
template ss_status scan_phase2<uint32_t>(const ScanSrc&, int64_t, void*, uint32_t*, cudaStream_t);

}  // namespace ss
