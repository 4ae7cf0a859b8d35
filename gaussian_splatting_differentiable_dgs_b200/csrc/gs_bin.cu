// gs_bin_tiles: per Leaf, the duplicated keys (tile id << 32 | depth bits)
// and candidate-slot values of every (candidate, tile) pair with the tile
// inside the Leaf, emitted in the candidates' depth order; plus the Leaf's
// per-tile ranges, read from the summed-area table of per-tile counts.
//
// BoundedGS project page, section 02 (B -> C): the image is split into
// Leaves and each Leaf is rasterised on its own; the per-Leaf key buffers
// are what the load budget bounds.
#include "gs_internal.cuh"

namespace gs {
namespace {

constexpr int kBinThreads = 256;

__global__ void __launch_bounds__(kBinThreads)
k_bin(const short4* __restrict__ rect, const uint32_t* __restrict__ depth_key,
      const int32_t* __restrict__ order, int64_t n_cand, gs_rect leaf, int TW,
      uint64_t* __restrict__ keys, int32_t* __restrict__ vals, int64_t capacity,
      unsigned long long* __restrict__ lb, unsigned int* __restrict__ ticket, int32_t* dev_status) {
  __shared__ unsigned int s_b;
  __shared__ long long s_scan[kBinThreads / 32 + 1];
  __shared__ long long s_prefix;
  if (threadIdx.x == 0) s_b = atomicAdd(ticket, 1u);
  __syncthreads();
  const int64_t b = s_b;
  const int64_t j = b * kBinThreads + threadIdx.x;
  int32_t slot = -1;
  int x0 = 0, x1 = 0, y0 = 0, y1 = 0;
  long long cnt = 0;
  if (j < n_cand) {
    slot = order[j];
    const short4 r = rect[slot];
    x0 = max((int)r.x, leaf.x0);
    x1 = min((int)r.z, leaf.x1);
    y0 = max((int)r.y, leaf.y0);
    y1 = min((int)r.w, leaf.y1);
    if (x1 > x0 && y1 > y0) cnt = (long long)(x1 - x0) * (y1 - y0);
  }
  long long total;
  const long long rank = block_exclusive_scan<long long, kBinThreads / 32>(cnt, s_scan, &total);
  if (threadIdx.x < 32) {
    const int64_t ex = lookback_warp(lb, b, total, dev_status);
    if (threadIdx.x == 0) s_prefix = ex;
  }
  __syncthreads();
  if (cnt == 0) return;
  int64_t off = s_prefix + rank;
  if (off + cnt > capacity) {
    dev_flag(dev_status, GS_DEV_BOUNDS);
    return;
  }
  const uint64_t dk = depth_key[slot];
  for (int ty = y0; ty < y1; ++ty)
    for (int tx = x0; tx < x1; ++tx) {
      keys[off] = ((uint64_t)((int64_t)ty * TW + tx) << 32) | dk;
      vals[off] = slot;
      ++off;
    }
}

__device__ __forceinline__ long long sat_rect(const int64_t* __restrict__ sat, int64_t s, int x0,
                                              int y0, int x1, int y1) {
  return sat[(int64_t)y1 * s + x1] - sat[(int64_t)y0 * s + x1] - sat[(int64_t)y1 * s + x0] +
         sat[(int64_t)y0 * s + x0];
}

__global__ void k_ranges(const int64_t* __restrict__ sat, gs_rect leaf, int TW,
                         int64_t* __restrict__ ranges) {
  const int lw = leaf.x1 - leaf.x0, lh = leaf.y1 - leaf.y0;
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (int64_t)lw * lh) return;
  const int tx = leaf.x0 + (int)(t % lw), ty = leaf.y0 + (int)(t / lw);
  const int64_t s = TW + 1;
  const long long begin = sat_rect(sat, s, leaf.x0, leaf.y0, leaf.x1, ty) +
                          sat_rect(sat, s, leaf.x0, ty, tx, ty + 1);
  const long long cnt = sat_rect(sat, s, tx, ty, tx + 1, ty + 1);
  ranges[2 * t] = begin;
  ranges[2 * t + 1] = begin + cnt;
}

struct BinWs {
  unsigned int* ticket;
  unsigned long long* lb;
  size_t bytes;
};

BinWs carve_bin(void* ws, size_t cap, int64_t n_cand) {
  Carver cv(ws, cap);
  BinWs w;
  w.ticket = cv.take<unsigned int>(64);
  const int64_t nb = (n_cand + kBinThreads - 1) / kBinThreads;
  w.lb = cv.take<unsigned long long>(nb > 0 ? nb : 1);
  w.bytes = cv.off;
  return w;
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" size_t gs_bin_workspace_size(int64_t n_cand) {
  if (n_cand < 0) return 0;
  return carve_bin(nullptr, 0, n_cand).bytes;
}

extern "C" gs_status gs_bin_tiles(const gs_proj* proj, int64_t n_cand, const int32_t* depth_order,
                                  gs_rect leaf, int32_t TW, int32_t TH,
                                  const int64_t* tile_sat,
                                  int64_t n_isect, uint64_t* keys, int32_t* vals, int64_t capacity,
                                  int64_t* ranges, int64_t* needed, void* ws, size_t ws_bytes,
                                  int32_t* dev_status, gs_stream stream) {
  if (!proj || n_cand < 0 || n_cand > proj->capacity || TW <= 0 || TH <= 0 || !tile_sat ||
      !ranges)
    return GS_ERR_ARG;
  if (leaf.x0 < 0 || leaf.y0 < 0 || leaf.x1 <= leaf.x0 || leaf.y1 <= leaf.y0 || leaf.x1 > TW ||
      leaf.y1 > TH)
    return GS_ERR_ARG;
  if (n_isect < 0) return GS_ERR_ARG;
  if (n_isect > capacity) {
    if (needed) *needed = n_isect;
    return GS_ERR_CAPACITY;
  }
  if (n_cand > 0 && (!depth_order || !proj->rect || !proj->depth_key)) return GS_ERR_ARG;
  if (n_isect > 0 && (!keys || !vals)) return GS_ERR_ARG;
  BinWs w = carve_bin(ws, ws_bytes, n_cand);
  if (!ws || w.bytes > ws_bytes) {
    if (needed) *needed = (int64_t)w.bytes;
    return GS_ERR_CAPACITY;
  }
  if (!aligned(ws, 256)) return GS_ERR_ARG;
  cudaStream_t s = to_stream(stream);
  const int64_t ntiles = (int64_t)(leaf.x1 - leaf.x0) * (leaf.y1 - leaf.y0);
  k_ranges<<<(unsigned)((ntiles + 255) / 256), 256, 0, s>>>(tile_sat, leaf, TW, ranges);
  GS_LAUNCH_CHECK();
  if (n_cand == 0 || n_isect == 0) return GS_OK;
  GS_TRY(cudaMemsetAsync(ws, 0, w.bytes, s));
  const int64_t nb = (n_cand + kBinThreads - 1) / kBinThreads;
  k_bin<<<(unsigned)nb, kBinThreads, 0, s>>>(reinterpret_cast<const short4*>(proj->rect),
                                              proj->depth_key, depth_order, n_cand, leaf, TW, keys,
                                              vals, capacity, w.lb, w.ticket, dev_status);
  GS_LAUNCH_CHECK();
  return GS_OK;
}
