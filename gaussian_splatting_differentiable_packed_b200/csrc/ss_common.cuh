// Shared host/device plumbing of libss: geometry derived from ss_dims, status
// and error reporting, launch helpers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>
#include <string>

#include "ss.h"

namespace ss {

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

constexpr int kBlock = SS_PMASK_BLOCK;  // pairs per popcount block
constexpr int kTile = SS_TILE;
constexpr int kRowF = SS_ROW_FLOATS;

struct Geo {
  int C, W, H, deg, K;
  int64_t N, n_pad, words_per_cam, blocks_per_cam, mask_words, mask_blocks;
  int tiles_x, tiles_y;
  int64_t tiles_per_cam, n_tiles;
  float near_plane, far_plane;
};

inline Geo geometry(const ss_dims& d) {
  Geo g;
  g.C = d.C; g.W = d.W; g.H = d.H; g.deg = d.sh_degree; g.K = (d.sh_degree + 1) * (d.sh_degree + 1);
  g.N = d.N;
  g.n_pad = (d.N + kBlock - 1) / kBlock * kBlock;
  g.words_per_cam = g.n_pad / 32;
  g.blocks_per_cam = g.n_pad / kBlock;
  g.mask_words = g.words_per_cam * d.C;
  g.mask_blocks = g.blocks_per_cam * d.C;
  g.tiles_x = (d.W + kTile - 1) / kTile;
  g.tiles_y = (d.H + kTile - 1) / kTile;
  g.tiles_per_cam = (int64_t)g.tiles_x * g.tiles_y;
  g.n_tiles = g.tiles_per_cam * d.C;
  g.near_plane = d.near_plane;
  g.far_plane = d.far_plane;
  return g;
}

// Dims accepted by every entry point.
inline bool dims_ok(const ss_dims* d) {
  if (!d) return false;
  if (d->C < 1 || d->W < 1 || d->H < 1 || d->N < 0) return false;
  if (d->sh_degree < 0 || d->sh_degree > 3) return false;
  if (!(d->near_plane > 0.0f) || !(d->far_plane > d->near_plane)) return false;
  if (d->W > 65535 * 16 || d->H > 65535 * 16) return false;
  // tile ids must fit the high word of a key
  int64_t tiles = (int64_t)((d->W + kTile - 1) / kTile) * ((d->H + kTile - 1) / kTile) * d->C;
  if (tiles >= (int64_t(1) << 32)) return false;
  return true;
}

void set_error(const std::string& msg);

// Records and maps a CUDA error; returns SS_OK when err == cudaSuccess.
inline ss_status cuda_status(cudaError_t err, const char* where) {
  if (err == cudaSuccess) return SS_OK;
  set_error(std::string(where) + ": " + cudaGetErrorString(err));
  return SS_ERR_CUDA;
}

inline ss_status invalid(const char* what) {
  set_error(std::string("invalid argument: ") + what);
  return SS_ERR_INVALID_ARG;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

constexpr int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
constexpr size_t align_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

// Asks L2 to fetch [p, p + bytes) ahead of use (bulk prefetch, no data
// returned to the SM; bytes is rounded down to the 16-byte granule).
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  bytes &= ~15u;
  if (bytes == 0 || ((uintptr_t)p & 15)) return;
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Asynchronous 4-byte copy global -> shared (no register holds the word;
// the copies of a thread complete at cp_async_wait_all).
__device__ __forceinline__ void cp_async4(float* smem_dst, const float* gsrc) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(gsrc) : "memory");
}
// Asynchronous 16-byte copy global -> shared (both 16-byte aligned), L2 only.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Waits until at most N of the thread's committed copy groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Resident CTAs of a kernel over the whole GPU (SMs x CTAs per SM): the
// distance, in blocks, between a CTA and the one that starts about a wave
// later.  0 if the query fails (then nothing is prefetched ahead).
template <typename K>
inline int64_t wave_blocks(K kernel, int threads, size_t smem) {
  int dev = 0, sms = 0, per = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kernel, threads, smem) != cudaSuccess) return 0;
  return (int64_t)sms * per;
}

// ----- generic exclusive scan (int64 totals), defined in scan.cu -----
// Items are produced by a "counter" selected by kind:
enum ScanKind { SCAN_U32 = 0, SCAN_TILES = 1 };
struct ScanSrc {
  int kind;
  const uint32_t* u32;     // SCAN_U32: counts
  const uint32_t* aabb16;  // SCAN_TILES: per-row AABB16, count = tiles covered
  int W, H, tiles_x, tiles_y;
};
constexpr int kScanItems = 16;
constexpr int kScanThreads = 256;
constexpr int64_t kScanTile = (int64_t)kScanItems * kScanThreads;
inline size_t scan_temp_bytes(int64_t n) { return align_up((size_t)(ceil_div(n, kScanTile) + 2) * 8, 256); }
// Phase 1: partial sums + exclusive scan of the partials; writes the total to
// *total_dev.  Phase 2 (after the caller has read the total): per-item offsets.
ss_status scan_phase1(const ScanSrc& src, int64_t n, void* temp, int64_t* total_dev, cudaStream_t st);
template <typename OutT>
ss_status scan_phase2(const ScanSrc& src, int64_t n, void* temp, OutT* out, cudaStream_t st);

}  // namespace ss
