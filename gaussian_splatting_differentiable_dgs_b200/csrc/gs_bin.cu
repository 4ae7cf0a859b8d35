// Depth order of the candidates (once per view) and per-Leaf binning.
//
// gs_depth_order sorts the candidates by the fp32 bits of their camera
// depth (stable, so equal depths keep the ascending Gaussian index) and
// gathers their tile rects into that order, so the per-Leaf scans below read
// a contiguous stream.
//
// gs_bin_tiles: per Leaf, one entry per (candidate, tile) pair with the tile
// inside the Leaf, emitted in the candidates' depth order: value = candidate
// slot, key = Leaf-local tile index (row-major within the Leaf), and, on
// request, the duplicated 64-bit key (global tile id << 32 | depth bits).
// A stable sort of the entries on the local tile index then yields exactly
// the order of the 64-bit keys; the Leaf's per-tile ranges come from the
// summed-area table of per-tile counts.
//
// BoundedGS project page, section 02 (B -> C): the image is split into
// Leaves and each Leaf is rasterised on its own; the per-Leaf key buffers
// are what the load budget bounds.
#include "gs_internal.cuh"

namespace gs {
namespace {

constexpr int kBinThreads = 256;
constexpr int kBinItems = 4;                       // candidates per thread
constexpr int kBinChunk = kBinThreads * kBinItems; // candidates per block

__global__ void __launch_bounds__(256)
k_gather_rects(const short4* __restrict__ rect, const int32_t* __restrict__ order, int64_t n,
               short4* __restrict__ out) {
  const int64_t j = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (j < n) out[j] = rect[order[j]];
}

__global__ void __launch_bounds__(kBinThreads)
k_bin(const short4* __restrict__ drect, const int32_t* __restrict__ order,
      const uint32_t* __restrict__ depth_key, int64_t n_cand, gs_rect leaf, int TW,
      uint32_t* __restrict__ tile_keys, int32_t* __restrict__ vals, uint64_t* __restrict__ keys64,
      int64_t capacity, unsigned long long* __restrict__ lb, unsigned int* __restrict__ ticket,
      int32_t* dev_status) {
  __shared__ unsigned int s_b;
  __shared__ long long s_scan[kBinThreads / 32 + 1];
  __shared__ long long s_prefix;
  __shared__ long long s_ex[kBinChunk + 1];
  __shared__ short s_x0[kBinChunk], s_y0[kBinChunk], s_w[kBinChunk];
  const int t = threadIdx.x;
  if (t == 0) s_b = atomicAdd(ticket, 1u);
  __syncthreads();
  const int64_t b = s_b;
  const int64_t j0 = b * kBinChunk + (int64_t)t * kBinItems;
  long long cnt[kBinItems];
  long long mine = 0;
#pragma unroll
  for (int k = 0; k < kBinItems; ++k) {
    const int64_t j = j0 + k;
    cnt[k] = 0;
    int x0 = 0, y0 = 0, w = 1;
    if (j < n_cand) {
      const short4 r = drect[j];
      x0 = max((int)r.x, leaf.x0);
      const int x1 = min((int)r.z, leaf.x1);
      y0 = max((int)r.y, leaf.y0);
      const int y1 = min((int)r.w, leaf.y1);
      if (x1 > x0 && y1 > y0) {
        w = x1 - x0;
        cnt[k] = (long long)w * (y1 - y0);
      }
    }
    s_x0[t * kBinItems + k] = (short)x0;
    s_y0[t * kBinItems + k] = (short)y0;
    s_w[t * kBinItems + k] = (short)w;
    mine += cnt[k];
  }
  long long total;
  long long run = block_exclusive_scan<long long, kBinThreads / 32>(mine, s_scan, &total);
#pragma unroll
  for (int k = 0; k < kBinItems; ++k) {
    s_ex[t * kBinItems + k] = run;
    run += cnt[k];
  }
  if (t == 0) s_ex[kBinChunk] = total;
  if (t < 32) {
    const int64_t ex = lookback_warp(lb, b, total, dev_status);
    if (t == 0) s_prefix = ex;
  }
  __syncthreads();
  if (total == 0) return;
  const int64_t base = s_prefix;
  if (base + total > capacity) {
    if (t == 0) dev_flag(dev_status, GS_DEV_BOUNDS);
    return;
  }
  const int lw = leaf.x1 - leaf.x0;
  // cooperative emission: entry e of the block belongs to the last candidate
  // whose exclusive offset is <= e; consecutive e are consecutive addresses
  for (long long e = t; e < total; e += kBinThreads) {
    int lo = 0, hi = kBinChunk - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_ex[mid] <= e) lo = mid;
      else hi = mid - 1;
    }
    const int c = lo;
    const long long q = e - s_ex[c];
    const int w = s_w[c];
    const int ty = s_y0[c] + (int)(q / w);
    const int tx = s_x0[c] + (int)(q % w);
    const int64_t pos = base + e;
    const int64_t j = b * kBinChunk + c;
    const int32_t slot = order[j];
    tile_keys[pos] = (uint32_t)((ty - leaf.y0) * lw + (tx - leaf.x0));
    vals[pos] = slot;
    if (keys64) keys64[pos] = ((uint64_t)((int64_t)ty * TW + tx) << 32) | depth_key[slot];
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
  const int64_t nb = (n_cand + kBinChunk - 1) / kBinChunk;
  w.lb = cv.take<unsigned long long>(nb > 0 ? nb : 1);
  w.bytes = cv.off;
  return w;
}

struct OrderWs {
  uint32_t* keys;
  void* sort_ws;
  size_t sort_bytes;
  size_t bytes;
};

OrderWs carve_order(void* ws, size_t cap, int64_t n_cand) {
  Carver cv(ws, cap);
  OrderWs w;
  w.keys = cv.take<uint32_t>(n_cand > 0 ? n_cand : 1);
  w.sort_bytes = gs_sort_workspace_size(n_cand, 4, 0, 32);
  w.sort_ws = cv.take<unsigned char>(w.sort_bytes);
  w.bytes = cv.off;
  return w;
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" size_t gs_depth_order_workspace_size(int64_t n_cand) {
  if (n_cand < 0) return 0;
  return carve_order(nullptr, 0, n_cand).bytes;
}

extern "C" gs_status gs_depth_order(const gs_proj* proj, int64_t n_cand, int32_t* depth_order,
                                    int16_t* depth_rect, void* ws, size_t ws_bytes,
                                    int32_t* dev_status, gs_stream stream) {
  if (!proj || n_cand < 0 || n_cand > proj->capacity) return GS_ERR_ARG;
  if (n_cand == 0) return GS_OK;
  if (!depth_order || !depth_rect || !proj->depth_key || !proj->rect) return GS_ERR_ARG;
  if (!aligned(depth_rect, 8) || !aligned(ws, 256)) return GS_ERR_ARG;
  OrderWs w = carve_order(ws, ws_bytes, n_cand);
  if (!ws || w.bytes > ws_bytes) return GS_ERR_CAPACITY;
  const gs_status st = gs_sort_keys32(proj->depth_key, w.keys, depth_order, n_cand, 0, 32,
                                      GS_SORT_IOTA, w.sort_ws, w.sort_bytes, dev_status, stream);
  if (st != GS_OK) return st;
  k_gather_rects<<<(unsigned)((n_cand + 255) / 256), 256, 0, to_stream(stream)>>>(
      reinterpret_cast<const short4*>(proj->rect), depth_order, n_cand,
      reinterpret_cast<short4*>(depth_rect));
  GS_LAUNCH_CHECK();
  return GS_OK;
}

extern "C" size_t gs_bin_workspace_size(int64_t n_cand) {
  if (n_cand < 0) return 0;
  return carve_bin(nullptr, 0, n_cand).bytes;
}

extern "C" gs_status gs_bin_tiles(const gs_proj* proj, int64_t n_cand, const int32_t* depth_order,
                                  const int16_t* depth_rect, gs_rect leaf, int32_t TW, int32_t TH,
                                  const int64_t* tile_sat, int64_t n_isect, uint32_t* tile_keys,
                                  int32_t* vals, uint64_t* keys64, int64_t capacity,
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
  if (n_cand > 0 && (!depth_order || !depth_rect || (keys64 && !proj->depth_key)))
    return GS_ERR_ARG;
  if (n_isect > 0 && (!tile_keys || !vals)) return GS_ERR_ARG;
  BinWs w = carve_bin(ws, ws_bytes, n_cand);
  if (!ws || w.bytes > ws_bytes) {
    if (needed) *needed = (int64_t)w.bytes;
    return GS_ERR_CAPACITY;
  }
  if (!aligned(ws, 256) || !aligned(depth_rect, 8)) return GS_ERR_ARG;
  cudaStream_t s = to_stream(stream);
  const int64_t ntiles = (int64_t)(leaf.x1 - leaf.x0) * (leaf.y1 - leaf.y0);
  k_ranges<<<(unsigned)((ntiles + 255) / 256), 256, 0, s>>>(tile_sat, leaf, TW, ranges);
  GS_LAUNCH_CHECK();
  if (n_cand == 0 || n_isect == 0) return GS_OK;
  GS_TRY(cudaMemsetAsync(ws, 0, w.bytes, s));
  const int64_t nb = (n_cand + kBinChunk - 1) / kBinChunk;
  k_bin<<<(unsigned)nb, kBinThreads, 0, s>>>(
      reinterpret_cast<const short4*>(depth_rect), depth_order, proj->depth_key, n_cand, leaf, TW,
      tile_keys, vals, keys64, capacity, w.lb, w.ticket, dev_status);
  GS_LAUNCH_CHECK();
  return GS_OK;
}
