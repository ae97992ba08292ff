// Stable LSD radix sort of (key, value) pairs on the (tile_id << 32 | depth)
// keys ("Spirula Studio VRAM deep-dive", buffer-cost table: double-buffered
// isect.ids_a/b; the reference's CUDA backend calls a library sort, this one is
// written here).  8-bit digits: the four bytes of the depth and the bytes the
// tile ids need.  A digit that is the same in every key (for example the top
// byte of depths whose exponents share their high bits) cannot change the
// order, so its pass is skipped: the host reads the histograms (one small
// copy) and launches only the passes whose digits vary.
//
//   k_hist_all   one read of the keys: the global digit histogram of every pass
//                (a permutation does not change them); skipped when the caller
//                passes the counts (key_hist, as the intersection writes them)
//   k_bases      the exclusive scan of each pass's 256 counts
//   k_onesweep   per pass, one kernel: each CTA takes the next 4096-key tile by
//                ticket, ranks its keys stably among equal digits (warp match +
//                per-warp counters), publishes its digit counts and looks back
//                over earlier tiles' published counts (decoupled look-back) for
//                its global offsets, then writes the keys in contiguous runs
//                from shared memory.  12 B read + 12 B written per key per pass.
//                The last pass also sets the tile offsets at tile boundaries
//                inside its runs; k_range_starts then takes the runs' first
//                keys (their places follow from the look-back status).
//
// The look-back spin is bounded: after kSpinLimit polls it records an error
// flag (reported by the call as SS_ERR_DEVICE_CHECK) and goes on.  Tiles are
// handed out by ticket, so every tile a CTA waits on belongs to a CTA that is
// already running and never waits on a later tile.
#include <algorithm>
#include <mutex>
#include <string>
#include <utility>

#include "ss_common.cuh"

namespace ss {

constexpr int kSortThreads = 256;
constexpr int kSortItems = 16;
constexpr int kSortTile = kSortThreads * kSortItems;  // 4096 keys per CTA
constexpr int kRadix = 256;
constexpr int kSortWarps = kSortThreads / 32;
constexpr int kHistItems = 8;  // keys per thread per histogram round

constexpr int kMaxPasses = 8;
constexpr uint64_t kFlagAgg = 1ull << 54;
constexpr uint64_t kFlagPre = 2ull << 54;
constexpr uint64_t kValMask = (1ull << 54) - 1;
constexpr int kSpinLimit = 1 << 20;

// Digit histograms of every pass in one read of the keys.  PASSES is a
// template argument so every digit is a constant byte of the key's low or
// high word.  Each warp counts into its own copy (dynamic shared memory,
// [warp][pass][digit]), so warps do not contend for the bins of common digits
// (the tile bytes of a region); the copies are summed at the end and added to
// the global histogram.
template <int PASSES>
__global__ __launch_bounds__(kSortThreads) void k_hist_all(const uint64_t* __restrict__ keys, int64_t n,
                                                           int lo_bytes, uint32_t* __restrict__ hist) {
  extern __shared__ uint32_t hw[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kPerWarp = PASSES * kRadix;
  for (int i = threadIdx.x; i < kSortWarps * kPerWarp; i += kSortThreads) hw[i] = 0;
  __syncthreads();
  uint32_t* mine = hw + warp * kPerWarp;
  // coalesced: a warp reads kHistItems runs of 32 consecutive keys, all in
  // flight together; neighbouring keys share digits (a row's keys share the
  // depth and neighbouring tile ids), so each run of equal digits is counted
  // by its first lane with one shared atomic
  const int64_t stride = (int64_t)gridDim.x * kSortThreads * kHistItems;
  for (int64_t base = ((int64_t)blockIdx.x * kSortWarps + warp) * 32 * kHistItems; base < n; base += stride) {
    uint64_t kr[kHistItems];
#pragma unroll
    for (int r = 0; r < kHistItems; ++r) {
      const int64_t i = base + r * 32 + lane;
      kr[r] = i < n ? keys[i] : 0ull;
    }
#pragma unroll
    for (int r = 0; r < kHistItems; ++r) {
      const bool valid = base + r * 32 + lane < n;
      const uint32_t lo = (uint32_t)kr[r], hi = (uint32_t)(kr[r] >> 32);
      const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
      const uint32_t end_all = 32u - (uint32_t)__clz(vmask);
      const uint32_t above = ~((2u << lane) - 1u);  // lanes above this one
#pragma unroll
      for (int p = 0; p < PASSES; ++p) {
        const uint32_t d = ((p < lo_bytes ? lo >> (8 * p) : hi >> (8 * (p - lo_bytes)))) & 0xFFu;
        const uint32_t prev = __shfl_up_sync(0xffffffffu, d, 1);
        const bool head = valid && (lane == 0 || d != prev);
        const uint32_t after = __ballot_sync(0xffffffffu, head) & above;
        if (head) atomicAdd(&mine[p * kRadix + d], (after ? (uint32_t)(__ffs(after) - 1) : end_all) - (uint32_t)lane);
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kPerWarp; i += kSortThreads) {
    uint32_t v = 0;
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) v += hw[w * kPerWarp + i];
    if (v) atomicAdd(&hist[i], v);
  }
}

template <int PASSES>
ss_status launch_hist(unsigned grid, cudaStream_t st, const uint64_t* keys, int64_t n, int lo_bytes, uint32_t* hist) {
  const size_t smem = sizeof(uint32_t) * kSortWarps * PASSES * kRadix;
  ss_status s = cuda_status(
      cudaFuncSetAttribute(k_hist_all<PASSES>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem), "smem attr");
  if (s) return s;
  k_hist_all<PASSES><<<grid, kSortThreads, smem, st>>>(keys, n, lo_bytes, hist);
  return cuda_status(cudaGetLastError(), "radix histogram");
}

// hist[p][d] -> exclusive scan over d, in place (one CTA of 256 threads).
__global__ __launch_bounds__(kRadix) void k_bases(uint32_t* __restrict__ hist, int passes) {
  __shared__ uint32_t wt[kRadix / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int p = 0; p < passes; ++p) {
    const uint32_t v = hist[p * kRadix + threadIdx.x];
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += x;
    }
    if (lane == 31) wt[warp] = inc;
    __syncthreads();
    uint32_t before = 0;
    for (int w = 0; w < warp; ++w) before += wt[w];
    hist[p * kRadix + threadIdx.x] = before + inc - v;
    __syncthreads();
  }
}

struct OnesweepSmem {
  uint32_t wcnt[kSortWarps][kRadix];
  uint32_t dstart[kRadix];
  int64_t gbase[kRadix];
  uint32_t wtot[kSortWarps + 1];
  uint32_t tile;
  uint64_t k[kSortTile];
  uint32_t v[kSortTile];
};

__device__ __forceinline__ uint64_t ld_status(const uint64_t* p) {
  return *reinterpret_cast<const volatile unsigned long long*>(p);
}

// Keys only: three CTAs per SM (85 registers); with values two.  RANGES (the
// last pass of the key sort): a tile-id boundary between two keys of the
// same digit run of this CTA sets the tile offsets it crosses; the runs'
// first keys are left to k_range_starts.
template <bool VALS, bool RANGES>
__global__ __launch_bounds__(kSortThreads, VALS ? 2 : 3) void k_onesweep(const uint64_t* __restrict__ kin,
                                                           const uint32_t* __restrict__ vin,
                                                           uint64_t* __restrict__ kout, uint32_t* __restrict__ vout,
                                                           int64_t n, int shift, uint64_t epoch,
                                                           const uint32_t* __restrict__ bases,
                                                           uint64_t* __restrict__ status,
                                                           uint32_t* __restrict__ ticket, uint32_t* __restrict__ err,
                                                           int64_t* __restrict__ tile_off) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  OnesweepSmem& S = *reinterpret_cast<OnesweepSmem*>(smem_raw);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) S.tile = atomicAdd(ticket, 1u);
  for (int i = threadIdx.x; i < kSortWarps * kRadix; i += kSortThreads) (&S.wcnt[0][0])[i] = 0;
  __syncthreads();
  const int64_t tile = S.tile;
  const int64_t tile0 = tile * kSortTile;
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
    if (VALS) vv[r] = valid ? vin[i] : 0u;
    const uint32_t d = valid ? (uint32_t)(kk[r] >> shift) & 0xFFu : 0x100u;
    const uint32_t peers = __match_any_sync(0xffffffffu, d);
    const uint32_t before = valid ? S.wcnt[warp][d] : 0u;
    __syncwarp();
    if (valid && lane == 31 - __clz(peers)) S.wcnt[warp][d] = before + __popc(peers);
    __syncwarp();
    pos[r] = valid ? before + __popc(peers & lt) : 0xFFFFFFFFu;
  }
  __syncthreads();
  {
    const int d = threadIdx.x;
    uint32_t run = 0;
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) {
      const uint32_t t = S.wcnt[w][d];
      S.wcnt[w][d] = run;
      run += t;
    }
    // publish this tile's count of digit d, then look back for its prefix
    uint64_t* st = status + tile * kRadix + d;
    if (tile == 0) {
      atomicExch(reinterpret_cast<unsigned long long*>(st), epoch | kFlagPre | run);
    } else {
      atomicExch(reinterpret_cast<unsigned long long*>(st), epoch | kFlagAgg | run);
    }
    uint64_t prefix = 0;
    if (tile > 0) {
      // walk back over earlier tiles' published counts, fetching a window of
      // kLook predecessors per round trip; stop at the first inclusive prefix
      constexpr int kLook = 8;
      int64_t t = tile - 1;
      int spins = 0;
      bool found = false;
      while (!found && t >= 0) {
        uint64_t w[kLook];
#pragma unroll
        for (int j = 0; j < kLook; ++j) w[j] = t - j >= 0 ? ld_status(status + (t - j) * kRadix + d) : 0ull;
        int j = 0;
        for (; j < kLook && t - j >= 0; ++j) {
          const uint64_t sv = w[j];
          const bool ready = (sv & ~(kValMask | kFlagAgg | kFlagPre)) == epoch && (sv & (kFlagAgg | kFlagPre));
          if (!ready) break;
          prefix += sv & kValMask;
          if (sv & kFlagPre) {
            found = true;
            break;
          }
        }
        if (found) break;
        if (j == kLook || t - j < 0) {
          t -= j;
          continue;
        }
        // predecessor t - j has not published yet: wait for it (bounded)
        t -= j;
        if (++spins > kSpinLimit) {
          atomicOr(err, 1u);
          break;
        }
        __nanosleep(32);
      }
      atomicExch(reinterpret_cast<unsigned long long*>(st), epoch | kFlagPre | (prefix + run));
    }
    S.gbase[d] = (int64_t)bases[d] + (int64_t)prefix;
    // exclusive scan of the tile's digit counts -> local digit starts
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
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kSortItems; ++r) {
    if (pos[r] == 0xFFFFFFFFu) continue;
    const uint32_t d = (uint32_t)(kk[r] >> shift) & 0xFFu;
    const uint32_t lp = S.dstart[d] + S.wcnt[warp][d] + pos[r];
    S.k[lp] = kk[r];
    if (VALS) S.v[lp] = vv[r];
  }
  __syncthreads();
  const int cnt = (int)min64(kSortTile, n - tile0);
  for (int i = threadIdx.x; i < cnt; i += kSortThreads) {
    const uint64_t key = S.k[i];
    const uint32_t d = (uint32_t)(key >> shift) & 0xFFu;
    const int64_t gpos = S.gbase[d] + (i - (int64_t)S.dstart[d]);
    kout[gpos] = key;
    if (VALS) vout[gpos] = S.v[i];
    if (RANGES && i != (int)S.dstart[d]) {
      // inside this CTA's run of digit d the predecessor in the output is
      // the previous key in shared memory
      const int64_t prev = (int64_t)(S.k[i - 1] >> 32), cur = (int64_t)(key >> 32);
      for (int64_t t = prev + 1; t <= cur; ++t) tile_off[t] = gpos;
    }
  }
}

// The first key of every (CTA tile, digit) run of the last pass: its place is
// the digit's base plus the run's exclusive prefix (the previous tile's
// inclusive status), its predecessor the key before it in the output; sets
// the tile offsets that boundary crosses.  Thread (0, 0) also closes the
// ranges after the last key.
__global__ __launch_bounds__(kRadix) void k_range_starts(const uint64_t* __restrict__ status,
                                                         const uint32_t* __restrict__ bases,
                                                         const uint64_t* __restrict__ keys, int64_t n,
                                                         int64_t ntiles, int64_t* __restrict__ tile_off) {
  const int64_t t = blockIdx.x;
  const int d = threadIdx.x;
  const uint64_t incl = status[t * kRadix + d] & kValMask;
  const uint64_t excl = t > 0 ? status[(t - 1) * kRadix + d] & kValMask : 0ull;
  if (incl > excl) {
    const int64_t gpos = (int64_t)bases[d] + (int64_t)excl;
    const int64_t prev = gpos == 0 ? -1 : (int64_t)(keys[gpos - 1] >> 32), cur = (int64_t)(keys[gpos] >> 32);
    for (int64_t u = prev + 1; u <= cur; ++u) tile_off[u] = gpos;
  }
  if (t == 0 && d == 0) {
    for (int64_t u = (int64_t)(keys[n - 1] >> 32) + 1; u <= ntiles; ++u) tile_off[u] = n;
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


// Scratch layout: hist [kMaxPasses][256] u32 | tickets [kMaxPasses] u32 |
// error flag u32 | look-back status [tiles][256] u64.
constexpr size_t sort_status_offset() { return align_up(kMaxPasses * kRadix * 4 + kMaxPasses * 4 + 4, 256); }

constexpr size_t sort_scratch_bytes(int64_t n) {
  return sort_status_offset() + (size_t)ceil_div(n > 1 ? n : 1, kSortTile) * kRadix * 8;
}

size_t sort_temp_bytes(int64_t n) { return sort_scratch_bytes(n); }

}  // namespace ss

using namespace ss;

namespace ss {

// Stable LSD sort of n (key, value) pairs over byte digits: the low word's
// lo_bytes bytes (4, or 0 when the keys already arrive in the order of their
// low words, ties in the order to keep), then the high word's hi_bytes bytes.
// The histograms are read back (one small copy, stream sync) and a digit
// equal in every key is skipped.  va and vb null: keys only.  *in_b: the
// result is in (kb, vb).  temp: sort_temp_bytes(n), cleared here.  The
// look-back flag is left in temp (radix_sort_flag).
ss_status radix_sort_pairs(uint64_t* ka, uint32_t* va, uint64_t* kb, uint32_t* vb, int64_t n, int lo_bytes,
                           int hi_bytes, const uint32_t* given_hist, void* temp, cudaStream_t st, bool* in_b,
                           int64_t* tile_off, int64_t ntiles, bool* ranged) {
  *in_b = false;
  if (ranged) *ranged = false;
  const bool vals = va != nullptr;
  auto pass_kernel = [&](bool ranges) {
    return vals ? (ranges ? k_onesweep<true, true> : k_onesweep<true, false>)
                : (ranges ? k_onesweep<false, true> : k_onesweep<false, false>);
  };
  ss_status s = SS_OK;
  for (int r = 0; r < 2 && !s; ++r)
    s = cuda_status(cudaFuncSetAttribute(pass_kernel(r == 1), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(OnesweepSmem)),
                    "set smem attribute");
  if (s) return s;
  const int64_t tiles = ceil_div(n, kSortTile);
  char* tb = reinterpret_cast<char*>(temp);
  uint32_t* hist = reinterpret_cast<uint32_t*>(tb);
  uint32_t* tickets = hist + kMaxPasses * kRadix;
  uint32_t* err = tickets + kMaxPasses;
  uint64_t* status = reinterpret_cast<uint64_t*>(tb + sort_status_offset());
  s = cuda_status(cudaMemsetAsync(temp, 0, sort_status_offset() + (size_t)tiles * kRadix * 8, st), "memset");
  if (s) return s;
  const int passes = lo_bytes + hi_bytes;
  if (passes < 1 || passes > kMaxPasses) return invalid("sort digit count");
  const unsigned hgrid = (unsigned)min64(tiles, 148 * 8);
  if (given_hist) {  // the digit counts come with the keys
    s = cuda_status(cudaMemcpyAsync(hist, given_hist, (size_t)passes * kRadix * 4, cudaMemcpyDeviceToDevice, st),
                    "copy histograms");
  } else switch (passes) {
    case 1: s = launch_hist<1>(hgrid, st, ka, n, lo_bytes, hist); break;
    case 2: s = launch_hist<2>(hgrid, st, ka, n, lo_bytes, hist); break;
    case 3: s = launch_hist<3>(hgrid, st, ka, n, lo_bytes, hist); break;
    case 4: s = launch_hist<4>(hgrid, st, ka, n, lo_bytes, hist); break;
    case 5: s = launch_hist<5>(hgrid, st, ka, n, lo_bytes, hist); break;
    case 6: s = launch_hist<6>(hgrid, st, ka, n, lo_bytes, hist); break;
    case 7: s = launch_hist<7>(hgrid, st, ka, n, lo_bytes, hist); break;
    default: s = launch_hist<8>(hgrid, st, ka, n, lo_bytes, hist); break;
  }
  if (s) return s;
  // which digits vary: a pass whose histogram holds all n keys in one bin
  // keeps the order as it is
  uint32_t h[kMaxPasses * kRadix];
  s = cuda_status(cudaMemcpyAsync(h, hist, (size_t)passes * kRadix * 4, cudaMemcpyDeviceToHost, st), "copy histograms");
  if (s) return s;
  s = cuda_status(cudaStreamSynchronize(st), "radix histogram");
  if (s) return s;
  k_bases<<<1, kRadix, 0, st>>>(hist, passes);
  s = cuda_status(cudaGetLastError(), "radix bases");
  if (s) return s;
  uint64_t* kin = ka;
  uint32_t* vin = va;
  uint64_t* kout = kb;
  uint32_t* vout = vb;
  bool varies[kMaxPasses];
  int last = -1;
  for (int p = 0; p < passes; ++p) {
    bool one_bin = false;
    for (int d = 0; d < kRadix; ++d) one_bin = one_bin || (int64_t)h[p * kRadix + d] == n;
    varies[p] = !one_bin;
    if (varies[p]) last = p;
  }
  int run = 0;
  for (int p = 0; p < passes; ++p) {
    if (!varies[p]) continue;
    const int shift = p < lo_bytes ? 8 * p : 32 + 8 * (p - lo_bytes);
    const uint64_t epoch = (uint64_t)(run + 1) << 56;
    const bool ranges = tile_off != nullptr && p == last;
    pass_kernel(ranges)<<<(unsigned)tiles, kSortThreads, sizeof(OnesweepSmem), st>>>(
        kin, vin, kout, vout, n, shift, epoch, hist + p * kRadix, status, tickets + run, err, tile_off);
    s = cuda_status(cudaGetLastError(), "radix pass");
    if (s) return s;
    if (ranges) {
      k_range_starts<<<(unsigned)tiles, kRadix, 0, st>>>(status, hist + p * kRadix, kout, n, ntiles, tile_off);
      s = cuda_status(cudaGetLastError(), "tile ranges");
      if (s) return s;
      *ranged = true;
    }
    std::swap(kin, kout);
    std::swap(vin, vout);
    ++run;
  }
  *in_b = run & 1;
  return SS_OK;
}

// Whether a sort's look-back wait ran out (stream sync).
ss_status radix_sort_flag(const void* temp, cudaStream_t st, bool* flagged) {
  const uint32_t* err = reinterpret_cast<const uint32_t*>(temp) + kMaxPasses * kRadix + kMaxPasses;
  uint32_t herr = 0;
  ss_status s = cuda_status(cudaMemcpyAsync(&herr, err, 4, cudaMemcpyDeviceToHost, st), "copy sort flag");
  if (s) return s;
  s = cuda_status(cudaStreamSynchronize(st), "sort");
  if (s) return s;
  *flagged = herr != 0;
  return SS_OK;
}

}  // namespace ss

extern "C" ss_status ss_sort_isects(const ss_dims* dims, uint64_t* keys_a, uint32_t* vals_a, uint64_t* keys_b,
                                    uint32_t* vals_b, int64_t n, int presorted_depth, const uint32_t* key_hist,
                                    void* temp, size_t temp_bytes, int64_t* tile_off, int* result_in_b_out,
                                    void* stream) {
  if (!dims_ok(dims)) return invalid("dims");
  if (!result_in_b_out || !tile_off) return invalid("null output");
  if (n < 0) return invalid("n < 0");
  if (n >= (int64_t(1) << 31)) {
    set_error("ss_sort_isects: n >= 2^31");
    return SS_ERR_OVERFLOW;
  }
  const Geo g = geometry(*dims);
  cudaStream_t st = as_stream(stream);
  *result_in_b_out = 0;
  if (n == 0) return cuda_status(cudaMemsetAsync(tile_off, 0, sizeof(int64_t) * (g.n_tiles + 1), st), "memset");
  if (!keys_a || !vals_a || !keys_b || !vals_b) return invalid("null keys/vals");
  if (!temp || temp_bytes < sort_temp_bytes(n)) return invalid("temp too small");
  if (key_hist && !presorted_depth) return invalid("key_hist needs presorted_depth (tile-id digits only)");
  // every byte of the depth (none when the keys arrive in depth order) and
  // the bytes of the tile ids; the plan drops the bytes that do not vary
  const int lo_bytes = presorted_depth ? 0 : 4;
  const int hi_bytes = max((tile_bits(g.n_tiles) + 7) / 8, lo_bytes ? 0 : 1);
  bool in_b = false, ranged = false;
  ss_status s = radix_sort_pairs(keys_a, vals_a, keys_b, vals_b, n, lo_bytes, hi_bytes, key_hist, temp, st, &in_b,
                                 tile_off, g.n_tiles, &ranged);
  if (s) return s;
  if (!ranged) {  // no pass ran: the keys were already in order
    const unsigned grid = (unsigned)ceil_div(n + 1, 256);
    k_tile_ranges<<<grid, 256, 0, st>>>(in_b ? keys_b : keys_a, n, g.n_tiles, tile_off);
    s = cuda_status(cudaGetLastError(), "tile ranges");
    if (s) return s;
  }
  bool flagged = false;
  s = radix_sort_flag(temp, st, &flagged);
  if (s) return s;
  *result_in_b_out = in_b ? 1 : 0;
  if (flagged) {
    set_error("ss_sort_isects: look-back wait exceeded its limit");
    return SS_ERR_DEVICE_CHECK;
  }
  return SS_OK;
}

// ---------------------------------------------------------------------------
// Allocation-free variant.  Some callers cannot call cudaMalloc at all: code
// that runs inside another runtime's allocator callbacks or memory-pool hooks
// (a nested cudaMalloc would re-enter that allocator), or a host that hands
// out only fixed, pre-sized device buffers.  This entry point keeps the
// sort's scratch in a file-scope device array instead of a caller buffer.
// The array is part of the loaded module: every GPU that loads the library
// holds it until the process exits.

namespace ss {

constexpr size_t kNoAllocScratchBytes = size_t(24) << 20;  // 24 MiB
// Largest key count whose scratch fits: whole 4096-key tiles of look-back
// status after the fixed header.
constexpr int64_t kNoAllocMaxKeys =
    (int64_t)((kNoAllocScratchBytes - sort_status_offset()) / (kRadix * 8)) * kSortTile;
static_assert(sort_scratch_bytes(kNoAllocMaxKeys) <= kNoAllocScratchBytes, "limit must fit the scratch");
static_assert(sort_scratch_bytes(kNoAllocMaxKeys + 1) > kNoAllocScratchBytes, "limit must be the largest that fits");

__device__ __align__(256) unsigned char g_sort_scratch[kNoAllocScratchBytes];

// Host code may not use g_sort_scratch as a device address: the symbol's host
// side is only a stand-in.  The device address is looked up with
// cudaGetSymbolAddress once per device and context (the module, and so the
// array, is loaded again in a new context, e.g. after cudaDeviceReset).
typedef int (*CtxGetCurrentFn)(void**);
std::mutex g_scratch_mu;
struct ScratchSlot {
  void* ctx;
  void* addr;
};
ScratchSlot g_scratch_slot[256] = {};

// The context current on this thread (NULL before the runtime has made one).
ss_status current_context(void** ctx) {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    ss_status s = cuda_status(cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q),
                              "cudaGetDriverEntryPoint");
    if (s) return s;
    if (!f || q != cudaDriverEntryPointSuccess) return invalid("cuCtxGetCurrent not found");
    fn = reinterpret_cast<CtxGetCurrentFn>(f);
  }
  *ctx = nullptr;
  if (fn(ctx) != 0) *ctx = nullptr;
  return SS_OK;
}

ss_status noalloc_scratch(void** out) {
  int dev = 0;
  ss_status s = cuda_status(cudaGetDevice(&dev), "cudaGetDevice");
  if (s) return s;
  if (dev < 0 || dev >= 256) return invalid("device ordinal out of range");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  void* ctx = nullptr;
  s = current_context(&ctx);
  if (s) return s;
  ScratchSlot& slot = g_scratch_slot[dev];
  if (!ctx || slot.ctx != ctx || !slot.addr) {
    // the lookup also makes the runtime's context current if none was
    void* p = nullptr;
    s = cuda_status(cudaGetSymbolAddress(&p, g_sort_scratch), "cudaGetSymbolAddress");
    if (s) return s;
    s = current_context(&ctx);
    if (s) return s;
    slot.ctx = ctx;
    slot.addr = p;
  }
  *out = slot.addr;
  return SS_OK;
}

}  // namespace ss

extern "C" ss_status ss_sort_isects_noalloc(const ss_dims* dims, uint64_t* keys_a, uint32_t* vals_a,
                                            uint64_t* keys_b, uint32_t* vals_b, int64_t n, int64_t* tile_off,
                                            int* result_in_b_out, void* stream) {
  if (n < 0) return invalid("n < 0");
  if (n > kNoAllocMaxKeys) {
    set_error("ss_sort_isects_noalloc: n = " + std::to_string(n) + " exceeds the " +
              std::to_string(kNoAllocScratchBytes >> 20) + " MiB static scratch (at most " +
              std::to_string(kNoAllocMaxKeys) + " keys)");
    return SS_ERR_INVALID_ARG;
  }
  void* scratch = nullptr;
  if (n > 0) {
    ss_status s = noalloc_scratch(&scratch);
    if (s) return s;
  }
  return ss_sort_isects(dims, keys_a, vals_a, keys_b, vals_b, n, 0, nullptr, scratch, kNoAllocScratchBytes,
                        tile_off, result_in_b_out, stream);
}
