/*
 * gs.h -- C ABI of libgs: one 3D Gaussian Splatting training step on an
 * NVIDIA B200 (sm_100a), with the BoundedGS memory scheme.
 *
 * The step for one view is
 *
 *   gs_project       cull + EWA projection of the candidate Gaussians,
 *                    per-tile intersection counts and their summed-area table
 *   gs_depth_order   depth presort of the candidates (once per view)
 *   gs_leaf_partition  (host) split the tile grid into Leaves whose
 *                    estimated load fits a byte budget
 *   for each Leaf:
 *     gs_bin_tiles   one entry per (candidate, tile) in depth order
 *     gs_sort_tiles  stable radix sort on the Leaf-local tile index
 *                    -> per-tile lists (the order of the 64-bit keys
 *                    tile << 32 | depth)
 *     gs_raster_fwd  front-to-back compositing (+ fused L1 loss)
 *     gs_raster_bwd  reverse blend, accumulated into the view's compact
 *                    per-candidate 2D gradients
 *   gs_project_bwd   projection backward, fused with ONE Adam update per view
 *
 * Sources (page title, section):
 *  - "BoundedGS: memory-efficient training for high-resolution 3D Gaussian
 *    Splatting" (project page), section 01: gradients of a local region are
 *    merged before its buffers are released; Leaves are sized by a load
 *    estimate from overlaps, pixels and buffer layout; the whole view's
 *    gradient is summed before one parameter update.  Section 02: A -> B
 *    two-stage backward (raster backward first, then projection backward);
 *    B -> C load-budgeted Leaves, over-budget regions split again, load
 *    re-checked before each execution; C -> D -> E candidate-index
 *    projection and compact gradients.
 *  - "SkipGS: Post-Densification Backward Skipping for Efficient 3DGS
 *    Training" (paper notes), sections "research background" (differentiable
 *    rasterisation of anisotropic 3D Gaussians), "key design 2" (backward =
 *    gradient back-propagation, atomic accumulation, coordinate and
 *    covariance differentiation) and "loss function / training strategy"
 *    (gradients through the projected 2D covariance and the transmittance
 *    accumulation to means, quaternions, scales, opacities and SH
 *    coefficients; Adam).
 *
 * Conventions
 *  - Every call returns a gs_status.  Arguments are checked on the host;
 *    errors found by a kernel are OR-ed into the caller's device word
 *    `dev_status` (GS_DEV_* bits) and reported by gs_check().
 *  - All device buffers are owned by the caller.  The library never
 *    allocates or frees memory; scratch comes from a caller workspace whose
 *    size the gs_*_workspace_size() queries return.  Workspaces need 256-byte
 *    alignment.
 *  - Every device call is asynchronous on the given stream (a cudaStream_t;
 *    NULL = the legacy default stream) and never synchronises, except
 *    gs_check().  There is no global state: calls on different streams with
 *    different buffers may run concurrently.
 *  - Layout of the model (planar SoA, fp32): params[P][n_pad],
 *    P = 11 + 3 (D+1)^2:  0..2 mean, 3..5 log-scale, 6..9 quaternion
 *    (w,x,y,z), 10 opacity logit, 11 + 3k + ch SH coefficient k, channel ch.
 *    n_pad must be a multiple of 4 and params 16-byte aligned.
 *  - Tiles are 16 x 16 pixels; TW = ceil(W/16), TH = ceil(H/16); tile id =
 *    ty * TW + tx.  Pixel centres are at (x + 0.5, y + 0.5).
 */
#ifndef GS_H
#define GS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t gs_status;
#define GS_OK 0
#define GS_WARN_BUDGET 1       /* a 1x1 Leaf is over budget (accepted) */
#define GS_ERR_ARG (-1)        /* bad pointer, size, alignment or value */
#define GS_ERR_CAPACITY (-2)   /* buffer or workspace too small; *needed set */
#define GS_ERR_CUDA (-3)       /* a CUDA runtime call failed */
#define GS_ERR_TIMEOUT (-4)    /* a bounded device wait gave up */
#define GS_ERR_BOUNDS (-5)     /* a kernel saw an index out of range */
#define GS_ERR_UNSUPPORTED (-6)

/* bits a kernel ORs into *dev_status */
#define GS_DEV_TIMEOUT 1u
#define GS_DEV_BOUNDS 2u
#define GS_DEV_NONFINITE 4u    /* non-finite parameter met; Gaussian culled */

#define GS_TILE 16
/* tiles per side of a block of the two-level binning (section 4) */
#define GS_TILE_BLOCK 8

typedef void* gs_stream; /* cudaStream_t */

/* Pinhole camera.  x_cam = R x_world + t (R row-major), OpenCV axes. */
typedef struct gs_camera {
  float R[9];
  float t[3];
  float fx, fy, cx, cy;
  int32_t width, height;
} gs_camera;

typedef struct gs_model {
  int64_t n;          /* Gaussians */
  int64_t n_pad;      /* plane stride, multiple of 4, >= n */
  int32_t sh_degree;  /* 0..3 */
  int32_t reserved;
  float* params;      /* device [P][n_pad] */
} gs_model;

/* Per-view projected state of the candidates (Gaussians that can touch the
 * view), in ascending Gaussian index.  Written by gs_project.
 * rec: 12 floats per candidate = three float4
 *   {u_hi, v_hi, lo, box}     u = u_hi + lo.x, v = v_hi + lo.y with lo a
 *                             half2 of fp16 corrections (bits in a float);
 *                             box a half2 of the alpha box half extents
 *                             (hx, hy) rounded up
 *   {s1, beta, s2, opacity}   q = s1 (dx + beta dy)^2 + s2 dy^2 with
 *                             s1 = a/2, beta = b/a, s2 = 1/(2 Sigma'_11),
 *                             (a, b, c) the conic Sigma'^-1
 *   {R, G, B, depth}
 * rect: tiles [x0, x1) x [y0, y1): those of the 3-sigma square whose
 * pixel-centre box [16 tx + 0.5, 16 tx + 15.5] x [16 ty + 0.5, 16 ty + 15.5]
 * meets the bounding box of the region where alpha can reach 1/255 (the
 * ellipse q <= ln(255 o), inflated by 1e-4 relative + 1e-4 in q and 0.01
 * px).  Every tile left out would skip the Gaussian at every pixel, so the
 * image and gradients equal those of the plain 3-sigma square.  A Gaussian
 * with 255 o < exp(-1e-4) is never a candidate. */
typedef struct gs_proj {
  int64_t capacity;     /* candidate capacity of the arrays below (>= n) */
  int32_t* n_cand;      /* device scalar */
  int32_t* cand_idx;    /* device [capacity] Gaussian index of each slot */
  int32_t* slot;        /* device [n] slot of Gaussian i, or -1 */
  float* rec;           /* device [capacity][12], 16-byte aligned */
  int16_t* rect;        /* device [capacity][4] */
  uint32_t* depth_key;  /* device [capacity] bits of fp32 camera depth */
  /* optional device scalar (NULL = off): total tiles of the candidates'
   * plain 3-sigma squares (clamped to the grid), the conventional count of
   * Gaussian-tile intersections */
  unsigned long long* square_isect;
} gs_proj;

/* A rectangle of tiles, half-open. */
typedef struct gs_rect {
  int32_t x0, y0, x1, y1;
} gs_rect;

/* Per-pixel buffers of one Leaf.  Pixel (x, y) of the image, for x in
 * [x0, x0 + w), y in [y0, y0 + h), lives at offset (y - y0) * pitch +
 * (x - x0) of img, T_final, last and each colour plane of dL_dimg; colour
 * planes are `plane` elements apart.  The target has its own layout: pixel
 * (x, y), channel c at target[(y - ty0) * tpitch + (x - tx0) + c * tplane]
 * (e.g. the whole view resident with tx0 = ty0 = 0, tpitch = W). */
typedef struct gs_pixels {
  int32_t x0, y0, w, h;
  int64_t pitch;
  int64_t plane;
  float* img;             /* [3] planes: rendered colour (written by fwd) */
  float* T_final;         /* transmittance after the last composited entry */
  int32_t* last;          /* 1 + list position of the last composited entry */
  float* dL_dimg;         /* [3] planes: dL/dcolour */
  const float* target;    /* or NULL (the forward then skips the loss) */
  int32_t tx0, ty0;
  int64_t tpitch;
  int64_t tplane;
  float* loss_tiles;      /* per global tile: norm * sum |r - t|, or NULL */
  double norm;            /* 1 / (3 W H): whole-view normaliser */
  /* optional work counters (NULL = off): [0] += pixel-Gaussian pairs
   * evaluated, [1] += pairs composited (forward) / differentiated
   * (backward); the forward also adds [2] += the method's evaluations
   * (each pixel's list entries up to its stop, or the whole list) and
   * [3] += the sum of last (the backward's evaluations), so a forward
   * needs 4 counters, a backward 2.  Used to account the work of a
   * launch. */
  unsigned long long* counters;
} gs_pixels;

/* Byte cost model of a Leaf (the buffers this library needs per unit). */
typedef struct gs_load_model {
  int64_t bytes_per_isect;
  int64_t bytes_per_pixel;
  int64_t bytes_per_tile;
  int64_t fixed_bytes;
  int64_t align;
} gs_load_model;

/* Hyper-parameters in fp64; the kernels apply the fp32 roundings of lr,
 * beta1, beta2, (1 - beta1), (1 - beta2), eps and the bias corrections
 * 1 - beta^t, each computed in fp64 on the host. */
typedef struct gs_adam_args {
  double lr, beta1, beta2, eps;
  int32_t step;  /* 1 on the first update */
  int32_t reserved;
} gs_adam_args;

int32_t gs_version(void);
const char* gs_status_string(gs_status s);

/* Number of kernel launches this library has issued in the calling process
 * since it was loaded (all devices and streams; launches that failed to
 * start included).  Host-only, thread-safe; no counterpart in the method,
 * it serves launch accounting of the callers. */
int64_t gs_launch_counter(void);

/* Synchronises `stream`, then reads and clears *dev_status.  Returns the
 * most severe condition (GS_ERR_TIMEOUT > GS_ERR_BOUNDS > GS_OK). */
gs_status gs_check(int32_t* dev_status, gs_stream stream);

/* ---- 1. projection -------------------------------------------------------
 * Cull + EWA projection.  For every Gaussian: t = R mu + t_cam; cull if
 * t_z <= 0.2, |t_x/t_z| > 1.3 (W/2)/f_x or |t_y/t_z| > 1.3 (H/2)/f_y, the
 * 2D covariance is not positive definite, or the tile rect is empty.  For
 * candidates: Sigma = R S S^T R^T (normalised quaternion, S = exp(log-scale)),
 * Sigma' = J W Sigma W^T J^T + 0.3 I, conic = Sigma'^-1, radius =
 * ceil(3 sqrt(lambda_max)), colour = max(0, sum_k sh_k Y_k(d) + 0.5),
 * opacity = sigmoid(logit), depth = t_z.  Candidates are compacted in
 * ascending index order (slot map in proj->slot).  Also writes the
 * (TH+1) x (TW+1) int64 summed-area table of per-tile intersection counts
 * (row 0 and column 0 zero) to `tile_sat`.
 * proj->capacity may be below n: candidates beyond it are not written,
 * GS_DEV_BOUNDS is set and *n_cand still receives the full count, so the
 * caller can retry with that capacity (the dense layout needs n).
 * The projection arithmetic is fp64; records are rounded to fp32.
 * flags: 0, or GS_PROJ_DENSE: the whole-image ("Original") layout of the
 * BoundedGS page, Fig. A and the ablation's configuration A: every Gaussian
 * keeps slot i (n_cand = n, cand_idx = identity), a culled one gets an
 * empty rect, depth -1 in its record and depth key 0xffffffff; the SAT and
 * all later stages skip it. */
#define GS_PROJ_DENSE 1u
/* gs_project_region: gs_project with every tile rect clipped to `region`
 * (tile units, half-open, inside the grid); a Gaussian whose rect misses it
 * is culled, the SAT and the 3-sigma count cover the region only.  The cull
 * tests, positions and records are the full view's, so a pixel of the
 * region gets the same list as with gs_project.  It serves the grouped and
 * fixed-block schedules (BoundedGS page, section 02 "from rendering to full
 * training" (F: finer grouping) and Figs. 5-6 (fixed blocks)). */
size_t gs_project_workspace_size(int64_t n, int32_t width, int32_t height);
gs_status gs_project(const gs_model* model, const gs_camera* cam,
                     uint32_t flags, const gs_proj* out, int64_t* tile_sat,
                     void* ws, size_t ws_bytes, int32_t* dev_status,
                     gs_stream stream);
gs_status gs_project_region(const gs_model* model, const gs_camera* cam,
                            uint32_t flags, gs_rect region, const gs_proj* out,
                            int64_t* tile_sat, void* ws, size_t ws_bytes,
                            int32_t* dev_status, gs_stream stream);

/* ---- 2. radix sorts ------------------------------------------------------
 * The per-tile depth order of the tile rasteriser: its duplicated 64-bit
 * keys (tile << 32 | depth bits) sorted ascending, ties in candidate order
 * (the sort the SkipGS paper notes' differentiable tile rasteriser rests
 * on, "research background"; the BoundedGS page sorts each Leaf's entries,
 * section 02 B -> C).  This library sorts the candidates once by depth and
 * then only the tile bits, which gives the same order.
 * Stable LSD radix sort of (key, value) pairs on key bits [begin_bit,
 * end_bit), 8-bit digits, an even number of passes: a histogram of every
 * digit in one pass over the keys, then per digit either three kernels
 * (per-tile digit counts, a scan of the counts per digit, a stable scatter
 * per tile; the default) or, with GS_SORT_ONESWEEP, one kernel with
 * decoupled look-back across tiles (Adinets & Merrill's "onesweep").  The
 * result is in keys[], vals[] (in place).  For the 32-bit variant, keys_in
 * (if not NULL) is read instead of keys on the first pass, and flag
 * GS_SORT_IOTA makes the input values 0..n-1.  The onesweep look-back waits
 * are bounded: on expiry GS_DEV_TIMEOUT is set and the call returns
 * without hanging. */
#define GS_SORT_IOTA 1u
#define GS_SORT_ONESWEEP 2u
/* Test hook of the bounded wait: the first tile of the first pass does not
 * publish its counts, so every later tile's look-back runs out and reports
 * GS_DEV_TIMEOUT (the result is then unspecified).  Never set otherwise. */
#define GS_SORT_TEST_STALL 0x80000000u
size_t gs_sort_workspace_size(int64_t n, int32_t key_bytes, int32_t begin_bit,
                              int32_t end_bit);
gs_status gs_sort_keys(uint64_t* keys, int32_t* vals, int64_t n,
                       int32_t begin_bit, int32_t end_bit, void* ws,
                       size_t ws_bytes, int32_t* dev_status, gs_stream stream);
gs_status gs_sort_keys32(const uint32_t* keys_in, uint32_t* keys,
                         int32_t* vals, int64_t n, int32_t begin_bit,
                         int32_t end_bit, uint32_t flags, void* ws,
                         size_t ws_bytes, int32_t* dev_status,
                         gs_stream stream);

/* Sort of binned entries by tile: (tile_keys, vals) with tile_keys in
 * [0, n_tiles) stably by key (bits [0, ceil(log2 n_tiles))), the digit
 * histograms taken from ranges (key t occurs ranges[2t+1] - ranges[2t]
 * times, as gs_bin_tiles writes them) instead of a pass over the keys.
 * Workspace: gs_sort_workspace_size(n, 4, 0, ceil(log2 n_tiles)).  Keys
 * that disagree with the ranges give an unspecified order (a scatter out of
 * range sets GS_DEV_BOUNDS and is skipped). */
gs_status gs_sort_tiles(uint32_t* tile_keys, int32_t* vals, int64_t n,
                        const int64_t* ranges, int64_t n_tiles, void* ws,
                        size_t ws_bytes, int32_t* dev_status, gs_stream stream);

/* Allocation-free variant of gs_sort_keys32 (no counterpart on the pages;
 * an addition of this library).  For callers that cannot allocate device
 * memory when they need the sort, e.g. code inside a host application whose
 * allocator owns the whole device, or a latency-critical loop that must not
 * risk an allocation's implicit device synchronisation.  Same arguments and
 * result as gs_sort_keys32 without the workspace: the scratch is an array
 * of GS_SORT_NOALLOC_SCRATCH_BYTES (3 MiB) inside the library that every
 * GPU loading the library holds until the process exits.  n >
 * GS_SORT_NOALLOC_MAX_N returns GS_ERR_CAPACITY and launches nothing;
 * flags other than GS_SORT_IOTA and GS_SORT_ONESWEEP return GS_ERR_ARG.
 * Every call looks up the array's address in the current device's context
 * (cudaGetSymbolAddress; GS_ERR_CUDA if that fails); the first call on a
 * device may load the library's device code, so make it before any stream
 * capture.  It never calls cudaMalloc or cudaFree.  All calls share the one
 * array: calls that overlap on the GPU (e.g. on two streams) race and give
 * wrong results; serialise them.  The parts of the array that must start
 * at zero are cleared by every call, so a call does not depend on the
 * previous one. */
#define GS_SORT_NOALLOC_MAX_N (1 << 18)
#define GS_SORT_NOALLOC_SCRATCH_BYTES ((size_t)3 << 20)
gs_status gs_sort_keys32_noalloc(const uint32_t* keys_in, uint32_t* keys,
                                 int32_t* vals, int64_t n, int32_t begin_bit,
                                 int32_t end_bit, uint32_t flags,
                                 int32_t* dev_status, gs_stream stream);

/* ---- 3. Leaf partition (host) --------------------------------------------
 * Recursive split of the tile grid: a rect whose estimated load
 *   align(I * b_isect) + align(pixels * b_px) + align(tiles * b_tile) + fixed
 * (I from the host copy of the SAT, pixels clipped to the image) exceeds
 * `budget` is cut at the midpoint of its longer side (x on ties) and both
 * halves are processed, first half first; a 1x1 rect is always accepted and
 * flagged over_budget if it does not fit.  Leaves come out in that
 * depth-first order.  Returns GS_WARN_BUDGET if any Leaf is over budget,
 * GS_ERR_CAPACITY if more than max_leaves would be needed (*n_leaves is
 * then the number required). */
/* gs_leaf_load_model: the per-unit bytes of one Leaf's buffers for the
 * binning path used (GS_BIN_SORT: gs_bin_tiles + gs_sort_tiles with
 * tile_bits = bits of the grid's tile count; GS_BIN_EXPAND:
 * gs_expand_tiles, whose per-view block lists and chunk tables are not part
 * of a Leaf's load). */
#define GS_BIN_SORT 0
#define GS_BIN_EXPAND 1
/* or-ed into `binning`: the Leaf also holds gs_loss_ssim's workspace */
#define GS_LOAD_SSIM 0x100
gs_status gs_leaf_load_model(int32_t binning, int32_t tile_bits,
                             gs_load_model* out);
gs_status gs_leaf_partition(const int64_t* sat_host, int32_t TW, int32_t TH,
                            int32_t width, int32_t height,
                            const gs_load_model* lm, int64_t budget,
                            gs_rect* leaves, int64_t* leaf_isect,
                            int64_t* leaf_bytes, uint8_t* over_budget,
                            int32_t max_leaves, int32_t* n_leaves);

/* ---- 4. depth order and binning -----------------------------------------
 * gs_depth_order (once per view): depth_order[0..n_cand) = candidate slots
 * sorted by the fp32 bits of their depth (stable: equal depths keep the
 * ascending Gaussian index), and depth_rect[j] = rect[depth_order[j]].
 * n_cand = GS_COUNT_ON_DEVICE reads the count from proj->n_cand on the
 * device (at most proj->capacity; buffers and workspace sized for the
 * capacity), so the call can be issued before the host has read it. */
#define GS_COUNT_ON_DEVICE (-1)
/* gs_bin_tiles (per Leaf): for the candidates in depth order, one entry per
 * tile of rect ∩ leaf, written in depth order: vals = candidate slot,
 * tile_keys = Leaf-local tile index (ly * leaf width + lx), and, if keys64
 * is not NULL, the duplicated 64-bit key (tile id << 32) | depth_key.  A
 * stable sort of (tile_keys, vals) on the low ceil(log2(Leaf tiles)) bits
 * (gs_sort_keys32) then gives the order of the 64-bit keys, i.e. each tile's
 * list front to back with ties by Gaussian index.  Also writes the Leaf's
 * per-tile ranges (ranges[2 t] = begin, [2 t + 1] = end, t = local tile
 * index) from the device SAT.  n_isect: the Leaf's intersection count (from
 * the host SAT); must be <= capacity, else GS_ERR_CAPACITY with *needed. */
size_t gs_depth_order_workspace_size(int64_t n_cand);
gs_status gs_depth_order(const gs_proj* proj, int64_t n_cand,
                         int32_t* depth_order, int16_t* depth_rect, void* ws,
                         size_t ws_bytes, int32_t* dev_status,
                         gs_stream stream);
size_t gs_bin_workspace_size(int64_t n_cand);
gs_status gs_bin_tiles(const gs_proj* proj, int64_t n_cand,
                       const int32_t* depth_order, const int16_t* depth_rect,
                       gs_rect leaf, int32_t TW, int32_t TH,
                       const int64_t* tile_sat, int64_t n_isect,
                       uint32_t* tile_keys, int32_t* vals, uint64_t* keys64,
                       int64_t capacity, int64_t* ranges, int64_t* needed,
                       void* ws, size_t ws_bytes, int32_t* dev_status,
                       gs_stream stream);

/* Two-level binning: the same per-Leaf lists as gs_bin_tiles followed by the
 * tile sort (bit-identical vals and ranges), without per-entry keys or a
 * sort of the Leaf's entries.  An implementation choice of this library for
 * the binning step (per-tile lists in depth order) of the tile rasteriser
 * that the SkipGS paper notes ("loss function / training strategy") leave
 * unchanged; the pages do not describe it.
 *
 * gs_block_sat (once per view, may run before the host learns n_cand):
 * block_sat = (BH + 1) x (BW + 1) summed-area table (zero first row and
 * column), BW = ceil(TW / GS_TILE_BLOCK), BH likewise, of the number of
 * candidates whose tile rect meets each block of GS_TILE_BLOCK^2 tiles.
 * Reads the candidate count *proj->n_cand on the device.
 *
 * gs_bin_blocks (once per view): per block, in row-major block order, the
 * slots of the candidates meeting it in depth order (block_vals), with
 * block_ranges[2 b], [2 b + 1] = begin, end of block b.  n_entries = the
 * total (block_sat[BH][BW] from a host copy); must be <= capacity, else
 * GS_ERR_CAPACITY with *needed.  The workspace also holds the block keys and
 * their sort.
 *
 * gs_expand_tiles (per Leaf): vals/ranges exactly as gs_bin_tiles +
 * gs_sort_tiles give them (ranges from the tile SAT, n_isect the Leaf's
 * count from the host SAT).  block_entries: the summed lengths of the block
 * lists of the blocks meeting the Leaf (from a host copy of block_sat); it
 * sizes the workspace.  A plan or a per-tile count that does not match the
 * SAT sets GS_DEV_BOUNDS in *dev_status. */
size_t gs_block_sat_workspace_size(int32_t TW, int32_t TH);
gs_status gs_block_sat(const gs_proj* proj, int32_t TW, int32_t TH,
                       int64_t* block_sat, void* ws, size_t ws_bytes,
                       int32_t* dev_status, gs_stream stream);
size_t gs_bin_blocks_workspace_size(int64_t n_cand, int64_t n_entries,
                                    int32_t TW, int32_t TH);
gs_status gs_bin_blocks(const gs_proj* proj, int64_t n_cand,
                        const int32_t* depth_order, const int16_t* depth_rect,
                        int32_t TW, int32_t TH, const int64_t* block_sat,
                        int64_t n_entries, int32_t* block_vals,
                        int64_t capacity, int64_t* block_ranges,
                        int64_t* needed, void* ws, size_t ws_bytes,
                        int32_t* dev_status, gs_stream stream);
size_t gs_expand_workspace_size(gs_rect leaf, int64_t block_entries);
gs_status gs_expand_tiles(const gs_proj* proj, const int32_t* block_vals,
                          const int64_t* block_ranges, int64_t block_entries,
                          gs_rect leaf, int32_t TW, int32_t TH,
                          const int64_t* tile_sat, int64_t n_isect,
                          int32_t* vals, int64_t capacity, int64_t* ranges,
                          int64_t* needed, void* ws, size_t ws_bytes,
                          int32_t* dev_status, gs_stream stream);

/* ---- 5. raster forward ---------------------------------------------------
 * Front-to-back alpha compositing of the projected Gaussians (SkipGS paper
 * notes, "research background" and "loss function / training strategy":
 * differentiable rasterisation through the transmittance accumulation;
 * BoundedGS page, section 02 B -> C: one Leaf's pixels at a time).
 * Per pixel p of the Leaf, over its tile's list in order: d = (u, v) - p;
 * q = (a d_x^2 + c d_y^2)/2 + b d_x d_y; alpha = min(0.99, o exp(-q)); skip
 * if alpha < 1/255; T' = T (1 - alpha); stop (without compositing) if
 * T' < 1e-4; else C += rgb alpha T, T = T'.  Background 0.  Writes img,
 * T_final, last; if px->target is set, also the L1 loss terms (as
 * gs_loss_l1).  fp32 arithmetic.
 * flags & 7 selects the pixels per thread (1, 2 or 4; 0 = the default, 2
 * here and 4 in gs_raster_bwd, the faster shapes on B200); img, T_final,
 * last and dL_dimg do not depend on it, the fp32 summation order of a
 * tile's loss partial (over the tile's warps) does.  The same flag applies
 * to gs_raster_bwd. */
gs_status gs_raster_fwd(const gs_proj* proj, const int32_t* vals,
                        const int64_t* ranges, gs_rect leaf,
                        const gs_camera* cam, const gs_pixels* px,
                        uint32_t flags, int32_t* dev_status, gs_stream stream);

/* gs_tile_ranges: the Leaf's per-tile list segments from the tile SAT
 * (ranges[2 t] = begin, [2 t + 1] = end, t = local tile index), as
 * gs_bin_tiles writes them.
 *
 * gs_raster_fwd_blocks: gs_raster_fwd with the tile lists built on the fly
 * from the per-block lists of gs_bin_blocks (an implementation choice of
 * this library, not on the pages): each tile filters its block's
 * depth-ordered list by "tile inside the candidate's rect", which is the
 * tile's list, and composites it; it stops reading once its pixels are
 * done.  ranges: in, the segments of gs_tile_ranges; out, end = begin + the
 * number of list entries consumed, and vals[begin .. end) = that prefix of
 * the tile's list (everything gs_raster_bwd reads: positions < last).
 * Image, T_final, last and loss are identical to gs_raster_fwd on the full
 * lists.  n_isect: the Leaf's count (host SAT), must be <= capacity.
 * By default all threads of a tile build its list, stage the records and
 * composite them in turn, meeting at CTA barriers; flags & GS_RASTER_WS
 * selects a warp-specialised form in which one warp per tile builds the list
 * and stages the records through an mbarrier ring while the others
 * composite (pixels per thread 2, or 4 with flags & 7 == 4).  Both give
 * identical results; on B200 the default is faster (the forward is bound by
 * its instruction issue, and the producer warp lowers the resident
 * compositing warps). */
#define GS_RASTER_WS 0x20u
gs_status gs_tile_ranges(const int64_t* tile_sat, int32_t TW, int32_t TH,
                         gs_rect leaf, int64_t* ranges, gs_stream stream);
gs_status gs_raster_fwd_blocks(const gs_proj* proj, const int32_t* block_vals,
                               const int64_t* block_ranges, gs_rect leaf,
                               const gs_camera* cam, const gs_pixels* px,
                               int32_t* vals, int64_t capacity,
                               int64_t n_isect, int64_t* ranges,
                               int64_t* needed, uint32_t flags,
                               int32_t* dev_status, gs_stream stream);

/* gs_upload_crop: the Leaf's crop [x0, x0 + w) x [y0, y0 + h) of a planar
 * host image (channels planes of host_plane floats, rows of host_pitch) into
 * a device buffer (rows of dev_pitch, planes of dev_plane), one 2D copy per
 * channel on `stream` (asynchronous when the host memory is pinned).  The
 * bounded supply of the supervision image, one Leaf at a time (BoundedGS
 * page, section 02 B -> C: the Leaf's forward, loss and backward). */
gs_status gs_upload_crop(const float* host, int64_t host_pitch,
                         int64_t host_plane, int32_t x0, int32_t y0, int32_t w,
                         int32_t h, int32_t channels, float* dev,
                         int64_t dev_pitch, int64_t dev_plane,
                         gs_stream stream);

/* ---- 6. L1 loss ----------------------------------------------------------
 * For the Leaf's pixels: dL/dimg = sign(img - target) * norm (sign(0) = 0)
 * and, per global tile, loss_tiles[tile] = norm * sum |img - target| in a
 * fixed order.  gs_loss_total sums loss_tiles[0..n) in a fixed order in
 * fp64 into *loss (device), so the loss is independent of the Leaves. */
gs_status gs_loss_l1(const gs_pixels* px, gs_rect leaf, const gs_camera* cam,
                     gs_stream stream);
gs_status gs_loss_total(const float* loss_tiles, int64_t n, double* loss,
                        gs_stream stream);

/* ---- 6b. SSIM term of the composite loss ---------------------------------
 * The composite photometric loss (1 - lambda) L1 + lambda (1 - SSIM),
 * lambda = 0.2 (SkipGS paper notes, "loss function / training strategy"),
 * with SSIM windows local to the Leaf (BoundedGS page, section 02: local
 * SSIM windows differ from full-image SSIM at their boundary).  SSIM is the
 * structural similarity of Wang et al. (IEEE TIP 2004): over the Leaf's
 * pixel rectangle R (its tiles clipped to the image), per channel, window
 * sums W[.] with the 11 x 11 Gaussian window (sigma 1.5, normalised; zero
 * outside R) of the render x = px->img and the target y = px->target give
 * mu_x = W[x], mu_y = W[y], sigma_x^2 = W[x^2] - mu_x^2, sigma_y^2,
 * sigma_xy = W[x y] - mu_x mu_y, and
 *   S = (2 mu_x mu_y + C1)(2 sigma_xy + C2) /
 *       ((mu_x^2 + mu_y^2 + C1)(sigma_x^2 + sigma_y^2 + C2)),
 * C1 = 0.01^2, C2 = 0.03^2 (data range 1).
 *
 * gs_loss_ssim adds weight * sum over each tile's pixels and channels of
 * (1 - S) to px->loss_tiles[tile] (global tile index, fixed summation
 * order) and, when ws is not NULL, weight * d sum(1 - S) / dx to
 * px->dL_dimg.  The L1 part comes first: gs_raster_fwd (or gs_loss_l1) with
 * px->norm = (1 - lambda) / (3 W H) writes dL_dimg and loss_tiles; then
 * weight = lambda / (3 W H).  ws (device, 16-byte aligned, at least
 * gs_ssim_workspace_size(leaf, cam) bytes) holds the partials of S in
 * (W[x], W[x^2], W[x y]) per pixel and channel between the two launches;
 * ws = NULL computes the loss only (one launch).  px->img and px->target
 * must cover R; px->loss_tiles must not be NULL.  fp32 arithmetic. */
size_t gs_ssim_workspace_size(gs_rect leaf, const gs_camera* cam);
gs_status gs_loss_ssim(const gs_pixels* px, gs_rect leaf, const gs_camera* cam,
                       double weight, void* ws, size_t ws_bytes,
                       gs_stream stream);

/* ---- 7. raster backward --------------------------------------------------
 * Reverse blend over list positions last-1 .. 0 with the forward's skip
 * tests, transmittance recovered as T_i = T_{i+1} / (1 - alpha_i) (with the
 * hardware reciprocal: T only scales gradient values, no decision).
 * Accumulates (adds) per candidate slot into g2d[slot][12] the gradients
 * {du, dv, da, db, dc, dopacity, dR, dG, dB, 0, 0, 0} ((a, b, c) = conic)
 * with per-tile reduction before the global atomics. */
gs_status gs_raster_bwd(const gs_proj* proj, const int32_t* vals,
                        const int64_t* ranges, gs_rect leaf,
                        const gs_camera* cam, const gs_pixels* px, float* g2d,
                        uint32_t flags, int32_t* dev_status, gs_stream stream);

/* ---- 8. projection backward ----------------------------------------------
 * Stage 2 of the two-stage backward: the exact derivative of gs_project's
 * candidate formulas, from g2d[slot][12] to every parameter (mean including
 * the SH view-direction term, log-scale, quaternion through the
 * normalisation, opacity logit, SH).  If `fused` is NULL, writes compact
 * gradients g3d[P][g3d_stride] (column = candidate slot).  Otherwise applies
 * one Adam update (as gs_adam with a zero gradient for non-candidates) to
 * model->params, adam_m and adam_v over all n Gaussians in one streaming pass
 * over every Gaussian's planes that forms the SH gradients on the fly.  The
 * candidates' geometric gradients (fp32 chain) are computed inside that pass
 * when g3d is NULL; with g3d given they come from a first pass into g3d used
 * as scratch (>= 14 * n_cand floats, 8-byte aligned, g3d_stride = its size in
 * floats).  Both forms give the same update up to fp32 rounding. */
gs_status gs_project_bwd(const gs_model* model, const gs_camera* cam,
                         const gs_proj* proj, int64_t n_cand,
                         const float* g2d, float* g3d, int64_t g3d_stride,
                         float* adam_m, float* adam_v,
                         const gs_adam_args* fused, int32_t* dev_status,
                         gs_stream stream);

/* gs_grad_accumulate: adds compact gradients g3d[P][g3d_stride] (column j =
 * candidate j) into a dense gradient G[P][n_pad] at column cand_idx[j].  A
 * Gaussian is at most one candidate of a projection, so this is a plain
 * add.  It sums the groups of a grouped schedule into the view's gradient
 * before its one Adam update (BoundedGS page, section 01: the whole view's
 * gradient is summed, then one update). */
gs_status gs_grad_accumulate(const float* g3d, int64_t g3d_stride,
                             const int32_t* cand_idx, int64_t n_cand, int32_t P,
                             float* G, int64_t n_pad, gs_stream stream);

/* ---- 9. Adam -------------------------------------------------------------
 * One Adam update per view on the view's summed gradient (BoundedGS page,
 * section 01: every region's gradient is summed over the whole view, then
 * the parameters are updated once; Kingma & Ba's Adam with bias
 * correction, the optimiser of 3DGS training):
 * m = b1 m + (1-b1) g; v = b2 v + (1-b2) g^2;
 * p -= lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps), for i < n, all P
 * planes.  If slot is NULL, g is dense [P][n_pad]; else g is compact
 * [P][g_stride] and Gaussian i reads column slot[i] (zero if -1). */
gs_status gs_adam(float* params, float* m, float* v, const float* g,
                  int64_t g_stride, const int32_t* slot, int64_t n,
                  int64_t n_pad, int32_t P, const gs_adam_args* args,
                  gs_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* GS_H */
