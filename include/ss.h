/*
 * ss.h — C ABI of the packed 3D Gaussian Splatting training step (libss.so).
 *
 * One forward+backward step over C cameras x N Gaussians, as described on the
 * "Spirula Studio" pages:
 *   ss_project_packed   packed projection (visibility bitmask, block-count scan,
 *                       compaction into screen rows and 16-bit AABBs)
 *   ss_intersect_tiles  tile intersections with an exact 64-bit count
 *   ss_sort_isects      radix sort of (tile_id << 32 | depth) keys + tile ranges
 *   ss_tile_order       tiles by decreasing entry count (rasterizer scheduling)
 *   ss_rasterize_fwd    16x16-tile front-to-back alpha compositing
 *   ss_rasterize_bwd    per-pixel reverse replay -> screen-space gradients
 *   ss_project_bwd      screen-space gradients -> means, quats, scales,
 *                       opacities, SH coefficients
 *   ss_project_bwd_adam the same, fused with an Adam step on the parameters
 *   ss_project_bwd_gq   the same, accumulating into block-quantised 16-bit
 *                       gradient accumulators
 *
 * Conventions (all entry points):
 *   - Every array pointer is a DEVICE pointer owned by the caller unless the
 *     parameter name ends in _out (host scalar).  The library never allocates
 *     or frees memory and keeps no state between calls.  Calls that need
 *     scratch take (temp, temp_bytes), sized by ss_workspace_bytes().
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is the
 *     legacy default stream).  ss_project_packed and ss_intersect_tiles
 *     synchronise the stream to return the counts that size later buffers,
 *     ss_sort_isects to read its device-side check flag.
 *   - Outputs are overwritten, never accumulated into (ss_project_bwd_adam
 *     updates its parameters and optimizer state in place).
 *   - Floating point is IEEE fp32; integer outputs are deterministic.
 *   - Errors are returned as ss_status; a failing call writes no element
 *     outside the caller's stated capacities.  Device-side checks never trap.
 *   - All sizes and offsets are 64-bit; buffers may exceed 4 GiB.
 *
 * Layouts:
 *   cams      float [C][20]: world-to-camera 4x4 view matrix, row-major, OpenCV
 *             axes (x right, y down, z forward), then fx, fy, cx, cy (pixels)
 *   means     float [N][3]      quats  float [N][4] (w,x,y,z; normalised inside)
 *   scales    float [N][3] activated (exp of the log-scale)
 *   opacities float [N]    activated (sigmoid of the logit)
 *   sh        float [N][K][3], K = (sh_degree+1)^2, real SH, degree-major
 *   mask      uint32 [ss_size(SS_SIZE_MASK_WORDS)]: bit (c*n_pad + n), LSB
 *             first, n_pad = N rounded up to SS_PMASK_BLOCK; padding bits are 0
 *   block_count uint32 [ss_size(SS_SIZE_MASK_BLOCKS)]: set bits per 128-pair block
 *   block_off int64 [blocks + 1]: exclusive scan of block_count; last = nnz
 *   screen    float [cap_rows][12]: x, y, conic a, conic b, conic c, opacity,
 *             r, g, b, depth, 0, 0 (48-byte rows: three 16-byte vectors)
 *   aabb16    uint32 [cap_rows][2]: word0 = qx0 | qy0 << 16, word1 = qx1 | qy1 << 16,
 *             edges on the grid extent/65535, min floored, max ceiled
 *   row_depth float [cap_rows]: the row's camera depth (the screen row's depth,
 *             stored compactly for the intersection pass's keys)
 *   keys      uint64 [cap_isects]: (c*tiles_per_cam + ty*tiles_x + tx) << 32 | bits(depth)
 *   vals      uint32 [cap_isects]: screen row index
 *   tile_off  int64 [n_tiles + 1]: tile t owns sorted entries [tile_off[t], tile_off[t+1])
 *   img       float [C][H][W][3]   T_final float [C][H][W]   last_id int32 [C][H][W]
 *   v_screen  float [nnz][12]: d/d(x, y, a, b, c, opacity, r, g, b, depth), 0, 0
 */
#ifndef SS_H
#define SS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Pairs per visibility block: each 128-pair block of the mask gets one
 * popcount ("Spirula Studio VRAM deep-dive", section "bitmask compaction":
 * both passes must agree on this constant). */
#define SS_PMASK_BLOCK 128
/* Rasterizer tile edge in pixels. */
#define SS_TILE 16
/* Floats per screen row and per screen-gradient row. */
#define SS_ROW_FLOATS 12

typedef int ss_status;
#define SS_OK 0
#define SS_ERR_INVALID_ARG 1   /* bad dims, null pointer, short temp buffer */
#define SS_ERR_CAPACITY 2      /* output capacity too small; the exact count is still returned */
#define SS_ERR_OVERFLOW 3      /* n_isects >= 2^31 (values and last_id are 32-bit) */
#define SS_ERR_CUDA 4          /* a CUDA runtime error; see ss_last_error() */
#define SS_ERR_DEVICE_CHECK 5  /* a device-side check failed (reported, never trapped) */

typedef struct ss_dims {
  int32_t C;          /* cameras, >= 1 */
  int32_t W, H;       /* image size in pixels, >= 1 */
  int32_t sh_degree;  /* 0..3 */
  int64_t N;          /* Gaussians, >= 0 */
  float near_plane;   /* > 0 */
  float far_plane;    /* > near_plane */
} ss_dims;

/* Sizes derived from dims (element counts, not bytes). */
#define SS_SIZE_MASK_WORDS 0   /* C * n_pad / 32 */
#define SS_SIZE_MASK_BLOCKS 1  /* C * n_pad / 128 */
#define SS_SIZE_TILES_X 2
#define SS_SIZE_TILES_Y 3
#define SS_SIZE_N_TILES 4      /* C * tiles_x * tiles_y */
#define SS_SIZE_N_PAD 5
int64_t ss_size(const ss_dims* dims, int what);

/* Scratch bytes needed by a call: which = SS_WS_PROJECT (count ignored),
 * SS_WS_INTERSECT (count = nnz), SS_WS_SORT (count = number of keys),
 * SS_WS_TILE_ORDER (count ignored). */
#define SS_WS_PROJECT 0
#define SS_WS_INTERSECT 1
#define SS_WS_SORT 2
#define SS_WS_TILE_ORDER 3
size_t ss_workspace_bytes(const ss_dims* dims, int which, int64_t count);

const char* ss_status_string(ss_status status);
/* Message of the last failing call on this host thread ("" if none). */
const char* ss_last_error(void);

/*
 * Packed projection ("Spirula Studio VRAM deep-dive", sections "bitmask
 * compaction" and "16-bit packed AABB"; "Spirula Studio backward pass",
 * section 5 for the projection chain).
 *
 * Pass 1 projects every (camera, Gaussian) pair (EWA covariance from quat and
 * scale, 0.3 dilation, 3-sigma radius) and writes the visibility bitmask and
 * one popcount per 128-pair block; the block counts are scanned into block_off
 * and nnz = block_off[blocks] is copied to *nnz_out (stream sync).  If screen
 * is NULL the call stops there (count-only).  If nnz > cap_rows it returns
 * SS_ERR_CAPACITY with *nnz_out exact and writes no row.  Otherwise pass 2
 * re-projects the survivors only: row = block_off[block] + set bits before the
 * pair, writing the screen row (SH colour evaluated toward the camera centre),
 * the 16-bit AABB and the row's depth into row_depth (4 bytes a row: the
 * intersection pass reads it instead of the 48-byte screen row).  Rows are
 * ordered camera-major, Gaussian-minor.  quats and sh must be 16-byte aligned
 * (SS_ERR_INVALID_ARG otherwise).
 *
 * cap_visible ("Spirula Studio VRAM deep-dive", practical guide: --cap-max,
 * the per-image visible splat cap that holds down nnz): < 0 for no cap.
 * Otherwise, in every camera with more than cap_visible visible pairs, only
 * the cap_visible of highest opacity stay visible (opacity ordered by its
 * fp32 value, IEEE total order; ties go to the lower Gaussian index; the page
 * names the cap but no selection rule, this is this library's reading); the
 * mask, block counts, block_off and nnz describe the capped set, so every
 * later call (and the projection backward) sees only the kept pairs.  Needs
 * opacities (even in count-only mode) and N <= 2^32; when the cap binds it
 * costs one more small copy and stream sync and 8 selection passes over the
 * mask.
 */
ss_status ss_project_packed(const ss_dims* dims, const float* cams, const float* means, const float* quats,
                            const float* scales, const float* opacities, const float* sh, uint32_t* mask,
                            uint32_t* block_count, int64_t* block_off, float* screen, uint32_t* aabb16,
                            float* row_depth, int64_t cap_rows, int64_t cap_visible, void* temp, size_t temp_bytes,
                            int64_t* nnz_out, void* stream);

/*
 * Tile intersections ("Spirula Studio VRAM deep-dive", section "4 GiB rule and
 * 2^31 limit": exact 64-bit count, host check before the scan, write window
 * clamped to the allocation; key format from the buffer-cost table).
 *
 * Counts the tiles of each row from its AABB16 (integer arithmetic), sums them
 * exactly in 64 bits and returns the total in *n_isects_out (stream sync).
 * Returns SS_ERR_CAPACITY if the total exceeds cap_isects and
 * SS_ERR_OVERFLOW if it is >= 2^31, writing no key in either case.
 * Otherwise writes one (key, row) per covered tile, the rows taken in order
 * of their depth (the IEEE bits of row_depth, ties by row index), each row's
 * tiles row-major over (ty, tx), so that ss_sort_isects can sort the tile
 * ids alone (presorted_depth); isect_off[nnz+1] holds the exclusive offsets
 * of the rows in that order.  block_off, aabb16 and row_depth are the arrays
 * ss_project_packed wrote (block_off gives each camera's first row).  temp:
 * ss_workspace_bytes(SS_WS_INTERSECT, nnz) bytes (it holds the depth order
 * of the rows).  The call synchronises the stream once more after the write
 * and returns SS_ERR_DEVICE_CHECK if a bounded look-back wait (the depth
 * sort's or the write's offsets) ran out.  key_hist (device, nullable):
 * uint32 [4][256], set to the counts of each digit value of byte b of the
 * written keys' tile ids (rows b >= the tile-id bytes stay zero), for
 * ss_sort_isects' key_hist.
 */
ss_status ss_intersect_tiles(const ss_dims* dims, const float* row_depth, const uint32_t* aabb16,
                             const int64_t* block_off, int64_t nnz, int64_t* isect_off, uint64_t* keys,
                             uint32_t* vals, uint32_t* key_hist, int64_t cap_isects, void* temp, size_t temp_bytes,
                             uint64_t* n_isects_out, void* stream);

/*
 * Stable LSD radix sort of n (key, value) pairs by key, 8-bit digits over the
 * 32 depth bits and the tile-id bits only ("Spirula Studio VRAM deep-dive",
 * buffer table: double-buffered isect.ids_a/b); a digit that is equal in
 * every key is skipped (it cannot change the order).  presorted_depth != 0
 * says the keys arrive in ascending order of their low words (the depths),
 * ties in the order to keep, as ss_intersect_tiles writes them: the tile-id
 * bytes alone are then sorted, which yields the same order.  Ping-pongs
 * between (keys_a, vals_a) and (keys_b, vals_b); *result_in_b_out (host)
 * says which pair holds the result (b after an odd number of digit passes,
 * which depends on the keys).  Then writes tile_off[n_tiles+1].
 * key_hist (device, nullable; only with presorted_depth != 0): the digit
 * counts of the keys' tile-id bytes, uint32 [4][256] as ss_intersect_tiles
 * writes them; the sort then skips its own histogram read of the keys.
 * n >= 2^31 returns SS_ERR_OVERFLOW.  Equal keys keep their input order.
 * Synchronises the stream at the end (reads the look-back error flag).
 */
ss_status ss_sort_isects(const ss_dims* dims, uint64_t* keys_a, uint32_t* vals_a, uint64_t* keys_b,
                         uint32_t* vals_b, int64_t n, int presorted_depth, const uint32_t* key_hist, void* temp,
                         size_t temp_bytes, int64_t* tile_off, int* result_in_b_out, void* stream);

/*
 * Projection backward fused with an Adam step (the pages' fused projection
 * backward + optimizer, "Spirula Studio backward pass", section 6: the
 * world-space gradient sums go straight into the optimizer, so no gradient
 * arrays are written).  Same gradient chain as ss_project_bwd; then, per
 * element, Adam with bias correction on the raw parameters
 *   m = b1 m + (1 - b1) g,  v = b2 v + (1 - b2) g^2,
 *   p = p - lr * (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
 * where the raw parameters are means, quats (unnormalised), log_scales,
 * logit_opacities and sh, and g for log-scales / logit-opacities is the
 * activated gradient times s / o (1 - o).  Updates in place: means, quats,
 * log_scales, logit_opacities, sh and the moments; refreshes the activated
 * copies scales = exp(log_scales) and opacities = sigmoid(logit_opacities)
 * that the forward reads (scales and opacities are read first as the
 * activated values the forward used).  All arrays are device memory laid out
 * like the parameters; state and hp are host structs.  quats, mask, v_screen,
 * sh and the SH moments must be 16-byte aligned; hp->step >= 1.
 */
typedef struct ss_adam {
  float lr_means, lr_quats, lr_scales, lr_opacities, lr_sh_dc, lr_sh_rest;
  float beta1, beta2, eps;
  int32_t step; /* t of this update, >= 1 */
} ss_adam;

typedef struct ss_adam_state {
  float *m_means, *v_means;         /* [N][3] */
  float *m_quats, *v_quats;         /* [N][4] */
  float *m_scales, *v_scales;       /* [N][3], of the log-scales */
  float *m_opacities, *v_opacities; /* [N], of the logit-opacities */
  float *m_sh, *v_sh;               /* [N][K][3] */
} ss_adam_state;

ss_status ss_project_bwd_adam(const ss_dims* dims, const float* cams, float* means, float* quats, float* log_scales,
                              float* scales, float* logit_opacities, float* opacities, float* sh,
                              const uint32_t* mask, const int64_t* block_off, const float* v_screen,
                              const ss_adam_state* state, const ss_adam* hp, void* stream);

/*
 * Projection backward with block-quantised gradient accumulation ("Spirula
 * Studio backward pass", section 6, technique 1): instead of fp32 gradient
 * arrays, each attribute's gradient accumulator is held as 16-bit codes in
 * blocks of 256 Gaussians (index n / 256), one fp32 scale per attribute and
 * block; the call decodes the accumulator (code * scale), adds this
 * sub-batch's gradient (the same gradient ss_project_bwd computes for the
 * cameras of dims) and quantises the sums again: scale = the block's largest
 * magnitude / 32767, code = nearest-even(x * (1 / scale)) in fp32 (within
 * 0.005 of a step of the exact quotient), 0 for an all-zero block.
 * first != 0 starts from zero (the accumulator's contents are ignored), as
 * for a step's first sub-batch.  Accumulator layout (device, owned by the
 * caller, updated in place):
 *   means [N][3], quats [N][4], scales [N][3], opacities [N], sh_dc [N][3]
 *   (SH coefficient 0), sh_rest [N][K-1][3] (NULL allowed when K == 1) as
 *   int16; block_scale [6][ceil(N/256)] float in that attribute order.
 * 118 B per Gaussian at SH degree 3 against 236 for the fp32 gradients.
 * quats, mask, v_screen, sh, sh_dc and sh_rest must be 16-byte aligned
 * (SS_ERR_INVALID_ARG otherwise).  Two CTAs of 128 Gaussians form one block; they run as a
 * thread-block cluster of two and exchange their maxima through distributed
 * shared memory.
 */
typedef struct ss_gq_accum {
  int16_t* means;
  int16_t* quats;
  int16_t* scales;
  int16_t* opacities;
  int16_t* sh_dc;
  int16_t* sh_rest;
  float* block_scale;
} ss_gq_accum;

ss_status ss_project_bwd_gq(const ss_dims* dims, const float* cams, const float* means, const float* quats,
                            const float* scales, const float* opacities, const float* sh, const uint32_t* mask,
                            const int64_t* block_off, const float* v_screen, const ss_gq_accum* acc, int first,
                            void* stream);

/*
 * Allocation-free variant of ss_sort_isects (the pages have no counterpart:
 * this is an addition of this library).  For callers that cannot call
 * cudaMalloc themselves: code that runs inside another runtime's allocator
 * callbacks or memory-pool hooks, where a nested cudaMalloc would re-enter
 * that allocator, or a host that hands out only fixed, pre-sized device
 * buffers.  The sort's scratch lives in a file-scope device array of 24 MiB
 * that the library holds on every GPU that loads it, until the process exits.
 * The caller still passes the key/value buffers and tile_off; no cudaMalloc,
 * cudaFree or allocating routine is called.  n may be at most 50,311,168 keys
 * (the whole 4096-key tiles of look-back state that fit in the 24 MiB after
 * a fixed header); a larger n returns SS_ERR_INVALID_ARG before any device work.  The
 * first call on a device (and context) looks up the array's device address
 * (cudaGetSymbolAddress) with that device current and keeps it for later
 * calls in that context.  Every call shares the one array (cleared at the
 * start of each call), so calls that overlap on the GPU race with each other:
 * serialise them, e.g. on one stream.  Like ss_sort_isects, the call
 * synchronises the stream at the end to read the sort's device-side check
 * flag.  Results equal ss_sort_isects'.
 */
ss_status ss_sort_isects_noalloc(const ss_dims* dims, uint64_t* keys_a, uint32_t* vals_a, uint64_t* keys_b,
                                 uint32_t* vals_b, int64_t n, int64_t* tile_off, int* result_in_b_out,
                                 void* stream);

/*
 * Scheduling order of the rasterizers' tiles: a permutation of [0, n_tiles)
 * into tile_order[n_tiles] (device uint32), tiles with more entries first
 * (tile_off[t+1] - tile_off[t], binned four bins per power of two; empty tiles
 * last; the order inside a bin is unspecified).  The rasterizers run one CTA
 * per tile and the block scheduler starts CTAs in index order, so a heavy
 * tile late in index order would run on alone at the end; longest first
 * keeps every SM busy until the work runs out.  temp: ss_workspace_bytes
 * (SS_WS_TILE_ORDER) bytes.
 */
ss_status ss_tile_order(const ss_dims* dims, const int64_t* tile_off, uint32_t* tile_order, void* temp,
                        size_t temp_bytes, void* stream);

/*
 * Forward rasterizer ("Spirula Studio backward pass", section 4: the forward
 * keeps tile offsets, the intersection list, each pixel's last Gaussian and
 * its transmittance for the backward pass).  One CTA per 16x16 tile, front to
 * back over the tile's sorted entries: alpha = min(0.99, o*exp(-sigma)),
 * entries with alpha < 1/255 skipped, stop before the entry that would take
 * T below 1e-4.  Writes img[C][H][W][3], T_final[C][H][W] and
 * last_id[C][H][W] (the sorted index of the last composited entry, -1 if
 * none).  vals are the sorted values.
 *
 * Optional outputs (the pages' depth/T render outputs and background blend;
 * pass NULL to leave them out, which runs the plain kernel):
 *   depth  [C][H][W] device float, the expected depth sum_i alpha_i T_i d_i
 *          with d_i the row's camera depth (not normalised by 1 - T_final);
 *   bg     [C][3] device float, a background colour per camera; img becomes
 *          C + T_final * bg.
 * tile_order (may be NULL: tile index order) is the order the CTAs take the
 * tiles in, as written by ss_tile_order; it changes only the scheduling (the
 * outputs are the same).  An entry >= n_tiles is skipped.
 */
ss_status ss_rasterize_fwd(const ss_dims* dims, const float* screen, const uint32_t* vals, const int64_t* tile_off,
                           const uint32_t* tile_order, float* img, float* T_final, int32_t* last_id, float* depth,
                           const float* bg, void* stream);

/*
 * Measurement helper, not part of the step: ss_rasterize_fwd plus exact work
 * counts summed over all pixels into counts[5] (device uint64, zeroed by the
 * call): [0] entries evaluated (up to and including the one that stopped the
 * pixel), [1] entries whose exp was evaluated, [2] entries composited,
 * [3] entries the backward replays (tile start to last_id), [4] exps among
 * those.  Used to state the rasterizers' arithmetic work for a roofline.
 */
ss_status ss_rasterize_fwd_counts(const ss_dims* dims, const float* screen, const uint32_t* vals,
                                  const int64_t* tile_off, float* img, float* T_final, int32_t* last_id,
                                  uint64_t* counts, void* stream);

/*
 * Backward rasterizer ("Spirula Studio backward pass", section 4): per pixel,
 * reverse replay from last_id using the saved state (no re-intersection),
 * splitting v_img (and v_T, may be NULL) by each entry's alpha contribution.
 * Gradients are reduced over the tile's pixels and added with atomics into
 * v_screen[nnz][12], which the call zeroes first.  v_depth ([C][H][W], may be
 * NULL) is the gradient of the expected depth of ss_rasterize_fwd and fills
 * the rows' depth gradient (column 9); bg ([C][3], may be NULL) must be the
 * background the forward blended.  tile_order as for ss_rasterize_fwd (the
 * rows' float sums are then added in another order: equal up to rounding).
 */
ss_status ss_rasterize_bwd(const ss_dims* dims, const float* screen, const uint32_t* vals, const int64_t* tile_off,
                           const uint32_t* tile_order, const float* T_final, const int32_t* last_id,
                           const float* v_img, const float* v_T, const float* v_depth, const float* bg,
                           float* v_screen, int64_t nnz, void* stream);

/*
 * Projection backward ("Spirula Studio backward pass", section 5): for each
 * Gaussian, over the cameras whose mask bit is set, the screen-row gradient is
 * taken back through the conic, the EWA Jacobian, the camera transform, the
 * covariance and the SH colour.  Deterministic (one thread per Gaussian, no
 * atomics).  Writes every element of the five outputs (zero where invisible).
 * quats, mask, v_quats, v_screen, sh and v_sh must be 16-byte aligned
 * (SS_ERR_INVALID_ARG otherwise).
 */
ss_status ss_project_bwd(const ss_dims* dims, const float* cams, const float* means, const float* quats,
                         const float* scales, const float* opacities, const float* sh, const uint32_t* mask,
                         const int64_t* block_off, const float* v_screen, float* v_means, float* v_quats,
                         float* v_scales, float* v_opacities, float* v_sh, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SS_H */
