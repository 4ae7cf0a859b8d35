// Host-side parts of libgs: the Leaf planner, the Leaf byte model, status
// handling.
//
// BoundedGS project page, section 01: the load of a region is estimated from
// its number of Gaussian-tile overlaps, its pixels and the buffer layout, so
// dense regions get smaller Leaves and sparse ones larger; section 02
// (B -> C): a region over the budget is subdivided again, and the current
// load is re-checked before each execution (here: the plan is rebuilt from
// the current view's counts every step).
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <vector>

#include "gs.h"

namespace {

constexpr int kTile = GS_TILE;

struct Plan {
  const int64_t* sat;
  int64_t stride;
  int32_t W, H;
  gs_load_model lm;
  int64_t budget;
  gs_rect* leaves;
  int64_t* leaf_isect;
  int64_t* leaf_bytes;
  uint8_t* over;
  int32_t cap;
  int32_t count;
  bool any_over;
};

int64_t up(int64_t x, int64_t a) { return a > 1 ? (x + a - 1) / a * a : x; }

int64_t rect_isect(const Plan& p, const gs_rect& r) {
  auto at = [&](int32_t x, int32_t y) { return p.sat[(int64_t)y * p.stride + x]; };
  return at(r.x1, r.y1) - at(r.x0, r.y1) - at(r.x1, r.y0) + at(r.x0, r.y0);
}

int64_t rect_bytes(const Plan& p, const gs_rect& r, int64_t isect) {
  const int64_t pw = std::min<int64_t>((int64_t)r.x1 * kTile, p.W) - (int64_t)r.x0 * kTile;
  const int64_t ph = std::min<int64_t>((int64_t)r.y1 * kTile, p.H) - (int64_t)r.y0 * kTile;
  const int64_t tiles = (int64_t)(r.x1 - r.x0) * (r.y1 - r.y0);
  return up(isect * p.lm.bytes_per_isect, p.lm.align) + up(pw * ph * p.lm.bytes_per_pixel, p.lm.align) +
         up(tiles * p.lm.bytes_per_tile, p.lm.align) + p.lm.fixed_bytes;
}

// Iterative depth-first split (explicit stack, first half processed first).
void plan_leaves(Plan& p, gs_rect root) {
  std::vector<gs_rect> stack{root};
  while (!stack.empty()) {
    const gs_rect r = stack.back();
    stack.pop_back();
    const int64_t isect = rect_isect(p, r);
    const int64_t bytes = rect_bytes(p, r, isect);
    const int32_t w = r.x1 - r.x0, h = r.y1 - r.y0;
    if (bytes <= p.budget || (w == 1 && h == 1)) {
      if (p.count < p.cap) {
        p.leaves[p.count] = r;
        if (p.leaf_isect) p.leaf_isect[p.count] = isect;
        if (p.leaf_bytes) p.leaf_bytes[p.count] = bytes;
        if (p.over) p.over[p.count] = bytes > p.budget ? 1 : 0;
      }
      p.any_over |= bytes > p.budget;
      p.count++;
      continue;
    }
    gs_rect a = r, b = r;
    if (w >= h) {
      a.x1 = b.x0 = r.x0 + w / 2;
    } else {
      a.y1 = b.y0 = r.y0 + h / 2;
    }
    stack.push_back(b);  // processed after a
    stack.push_back(a);
  }
}

std::atomic<int64_t> g_launches{0};

}  // namespace

namespace gs {
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace gs

extern "C" int32_t gs_version(void) { return 1; }

extern "C" int64_t gs_launch_counter(void) { return g_launches.load(std::memory_order_relaxed); }

extern "C" const char* gs_status_string(gs_status s) {
  switch (s) {
    case GS_OK: return "ok";
    case GS_WARN_BUDGET: return "a single-tile Leaf exceeds the load budget";
    case GS_ERR_ARG: return "invalid argument";
    case GS_ERR_CAPACITY: return "buffer or workspace too small";
    case GS_ERR_CUDA: return "CUDA runtime error";
    case GS_ERR_TIMEOUT: return "bounded device wait expired";
    case GS_ERR_BOUNDS: return "device index out of range";
    case GS_ERR_UNSUPPORTED: return "unsupported";
    default: return "unknown status";
  }
}

extern "C" gs_status gs_check(int32_t* dev_status, gs_stream stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return GS_ERR_CUDA;
  if (!dev_status) return GS_OK;
  int32_t v = 0;
  if (cudaMemcpy(&v, dev_status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return GS_ERR_CUDA;
  if (v != 0 && cudaMemset(dev_status, 0, sizeof v) != cudaSuccess) return GS_ERR_CUDA;
  if (v & GS_DEV_TIMEOUT) return GS_ERR_TIMEOUT;
  if (v & GS_DEV_BOUNDS) return GS_ERR_BOUNDS;
  return GS_OK;
}

// Per-unit bytes of the buffers one Leaf needs.
// GS_BIN_SORT (gs_bin_tiles + gs_sort_tiles): intersections take 32-bit tile
// keys + 32-bit values + their sort double buffers (16 B) plus the counts of
// the tile sort (256 x 4 B per 4096 items per pass); tile_bits, the bits of
// the whole grid's tile count, bounds any Leaf's local bits.  Fixed: sort
// histograms, tickets and alignment.
// GS_BIN_EXPAND (gs_expand_tiles): intersections take their 32-bit value
// only; fixed: the alignment of the Leaf's buffers.
// Both: pixels take colour (12), T_final (4), last (4), target crop (12) and
// dL/dcolour (12), with the SSIM term 36 more; tiles the int64 range pair.
extern "C" gs_status gs_leaf_load_model(int32_t binning, int32_t tile_bits, gs_load_model* out) {
  if (!out || tile_bits < 0 || tile_bits > 32) return GS_ERR_ARG;
  const bool ssim = (binning & GS_LOAD_SSIM) != 0;
  binning &= ~GS_LOAD_SSIM;
  // the SSIM term's workspace: three partials per pixel and channel
  out->bytes_per_pixel = 44 + (ssim ? 36 : 0);
  out->bytes_per_tile = 16;
  out->align = 512;
  if (binning == GS_BIN_EXPAND) {
    out->bytes_per_isect = 4;
    out->fixed_bytes = 8 * 256;
    return GS_OK;
  }
  if (binning != GS_BIN_SORT) return GS_ERR_ARG;
  const int passes = tile_bits == 0 ? 0 : 2 * ((tile_bits + 15) / 16);
  out->bytes_per_isect = 16 + (passes + 1) / 2;
  out->fixed_bytes = 2 * 8 * 256 * 8 + 64 * 4 + (int64_t)passes * 256 * 8 + 16 * 256;
  return GS_OK;
}

extern "C" gs_status gs_leaf_partition(const int64_t* sat_host, int32_t TW, int32_t TH,
                                       int32_t width, int32_t height, const gs_load_model* lm,
                                       int64_t budget, gs_rect* leaves, int64_t* leaf_isect,
                                       int64_t* leaf_bytes, uint8_t* over_budget,
                                       int32_t max_leaves, int32_t* n_leaves) {
  if (!sat_host || !lm || !leaves || !n_leaves || TW <= 0 || TH <= 0 || max_leaves < 0 ||
      budget < 0 || width <= 0 || height <= 0)
    return GS_ERR_ARG;
  if ((int64_t)(width + kTile - 1) / kTile != TW || (int64_t)(height + kTile - 1) / kTile != TH)
    return GS_ERR_ARG;
  if (lm->bytes_per_isect < 0 || lm->bytes_per_pixel < 0 || lm->bytes_per_tile < 0 ||
      lm->fixed_bytes < 0 || lm->align < 1)
    return GS_ERR_ARG;
  Plan p{sat_host, (int64_t)TW + 1, width, height, *lm, budget, leaves, leaf_isect, leaf_bytes,
         over_budget, max_leaves, 0, false};
  plan_leaves(p, gs_rect{0, 0, TW, TH});
  *n_leaves = p.count;
  if (p.count > max_leaves) return GS_ERR_CAPACITY;
  return p.any_over ? GS_WARN_BUDGET : GS_OK;
}

// Leaf crop of a planar host image ([channels][height][host_pitch] floats,
// plane stride host_plane) into a device buffer, one 2D copy per channel.
// Asynchronous when the host memory is pinned.
extern "C" gs_status gs_upload_crop(const float* host, int64_t host_pitch, int64_t host_plane,
                                    int32_t x0, int32_t y0, int32_t w, int32_t h,
                                    int32_t channels, float* dev, int64_t dev_pitch,
                                    int64_t dev_plane, gs_stream stream) {
  if (!host || !dev || x0 < 0 || y0 < 0 || w < 0 || h < 0 || channels < 1) return GS_ERR_ARG;
  if (w == 0 || h == 0) return GS_OK;
  if (host_pitch < (int64_t)x0 + w || host_plane < host_pitch * ((int64_t)y0 + h) ||
      dev_pitch < w || dev_plane < dev_pitch * (int64_t)h)
    return GS_ERR_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (int32_t c = 0; c < channels; ++c) {
    const float* src = host + c * host_plane + (int64_t)y0 * host_pitch + x0;
    float* dst = dev + c * dev_plane;
    if (cudaMemcpy2DAsync(dst, (size_t)dev_pitch * sizeof(float), src,
                          (size_t)host_pitch * sizeof(float), (size_t)w * sizeof(float),
                          (size_t)h, cudaMemcpyHostToDevice, s) != cudaSuccess)
      return GS_ERR_CUDA;
  }
  return GS_OK;
}
