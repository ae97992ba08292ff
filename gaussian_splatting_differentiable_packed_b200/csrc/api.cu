// Host-side entry points of libss that launch nothing: sizes, scratch sizes,
// status strings and the per-thread error message.
#include <algorithm>
#include <string>

#include "ss_common.cuh"

namespace ss {

thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }

size_t sort_temp_bytes(int64_t n);
size_t isect_temp_bytes(int64_t nnz);
size_t tile_order_temp_bytes();
size_t project_temp_bytes(const Geo& g);

}  // namespace ss

using namespace ss;

extern "C" int64_t ss_size(const ss_dims* dims, int what) {
  if (!dims_ok(dims)) return -1;
  const Geo g = geometry(*dims);
  switch (what) {
    case SS_SIZE_MASK_WORDS: return g.mask_words;
    case SS_SIZE_MASK_BLOCKS: return g.mask_blocks;
    case SS_SIZE_TILES_X: return g.tiles_x;
    case SS_SIZE_TILES_Y: return g.tiles_y;
    case SS_SIZE_N_TILES: return g.n_tiles;
    case SS_SIZE_N_PAD: return g.n_pad;
    default: return -1;
  }
}

extern "C" size_t ss_workspace_bytes(const ss_dims* dims, int which, int64_t count) {
  if (!dims_ok(dims)) return 0;
  const Geo g = geometry(*dims);
  switch (which) {
    case SS_WS_PROJECT: return project_temp_bytes(g);
    case SS_WS_INTERSECT: return isect_temp_bytes(max64(count, 1));
    case SS_WS_SORT: return sort_temp_bytes(max64(count, 1));
    case SS_WS_TILE_ORDER: return tile_order_temp_bytes();
    default: return 0;
  }
}

extern "C" const char* ss_status_string(ss_status s) {
  switch (s) {
    case SS_OK: return "ok";
    case SS_ERR_INVALID_ARG: return "invalid argument";
    case SS_ERR_CAPACITY: return "capacity exceeded";
    case SS_ERR_OVERFLOW: return "count overflows 32-bit indices";
    case SS_ERR_CUDA: return "CUDA error";
    case SS_ERR_DEVICE_CHECK: return "device-side check failed";
    default: return "unknown status";
  }
}

extern "C" const char* ss_last_error(void) { return g_last_error.c_str(); }
