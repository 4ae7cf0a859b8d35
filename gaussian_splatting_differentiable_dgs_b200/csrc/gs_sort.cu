// Stable LSD radix sort of (key, int32 value) pairs: one histogram pass over
// all digits, then one "onesweep" pass per digit (Adinets & Merrill,
// "Onesweep: a faster least significant digit radix sort for GPUs", 2022):
// each block ranks its tile of 4096 items in shared memory, obtains the
// global offset of each digit by decoupled look-back across tiles, and
// scatters through a shared-memory staging buffer so runs of equal digits
// leave as coalesced stores.
//
// Used twice per view: the depth presort of the candidates (32-bit keys),
// and per Leaf a sort of the duplicated (tile << 32 | depth) keys on the
// tile bits only.  Because the keys are emitted in depth order, the stable
// tile-bit sort yields the same order as a full 64-bit sort.

#include "gs_internal.cuh"

namespace gs {
namespace {

// Launch shape (overridable at build time for tuning sweeps).
#ifndef GS_SORT_THREADS
#define GS_SORT_THREADS 512
#endif
#ifndef GS_SORT_IPT
#define GS_SORT_IPT 8
#endif
#ifndef GS_SORT_WIN
#define GS_SORT_WIN 4
#endif
#ifndef GS_SORT_MINB
#define GS_SORT_MINB 2
#endif

constexpr int kSortThreads = GS_SORT_THREADS;
constexpr int kIPT = GS_SORT_IPT;
constexpr int kSortTile = kSortThreads * kIPT;
constexpr int kWarps = kSortThreads / 32;
constexpr int kRadix = 256;
constexpr int kLookWin = GS_SORT_WIN;  // predecessors read per look-back round trip
static_assert(kSortThreads >= kRadix, "one thread per digit");

struct SortPlan {
  int passes;
  int shift[8];
  int bits[8];
};

SortPlan plan_sort(int begin_bit, int end_bit) {
  SortPlan p{};
  const int nb = end_bit - begin_bit;
  if (nb <= 0) return p;
  // an even number of passes keeps the result in the caller's buffers
  p.passes = 2 * ((nb + 15) / 16);
  const int per = (nb + p.passes - 1) / p.passes;
  int b = begin_bit;
  for (int k = 0; k < p.passes; ++k) {
    p.shift[k] = b;
    p.bits[k] = b + per <= end_bit ? per : end_bit - b;
    if (p.bits[k] < 0) p.bits[k] = 0;
    b += p.bits[k];
  }
  return p;
}

template <class K>
__device__ __forceinline__ unsigned digit_of(K key, int shift, unsigned mask) {
  return (unsigned)(key >> shift) & mask;
}

template <class K>
__global__ void __launch_bounds__(kSortThreads)
k_hist(const K* __restrict__ keys, int64_t n, SortPlan plan, unsigned long long* __restrict__ hist,
       const int32_t* __restrict__ n_dev) {
  if (n_dev) n = min(n, (int64_t)*n_dev);  // the count on the device, at most n
  __shared__ unsigned int sh[8][kRadix];
  for (int e = threadIdx.x; e < 8 * kRadix; e += kSortThreads) (&sh[0][0])[e] = 0;
  __syncthreads();
  const int64_t stride = (int64_t)gridDim.x * kSortThreads;
  for (int64_t i = (int64_t)blockIdx.x * kSortThreads + threadIdx.x; i < n; i += stride) {
    const K k = keys[i];
    for (int p = 0; p < plan.passes; ++p)
      atomicAdd(&sh[p][digit_of(k, plan.shift[p], (1u << plan.bits[p]) - 1)], 1u);
  }
  __syncthreads();
  for (int p = 0; p < plan.passes; ++p)
    for (int d = threadIdx.x; d < kRadix; d += kSortThreads)
      if (sh[p][d]) atomicAdd(&hist[p * kRadix + d], (unsigned long long)sh[p][d]);
}

// Digit histograms of keys 0..n_tiles-1 whose multiplicities are the range
// lengths (ranges[2t+1] - ranges[2t]): the keys need not be read.
__global__ void __launch_bounds__(256)
k_hist_from_ranges(const int64_t* __restrict__ ranges, int64_t n_tiles, SortPlan plan,
                   unsigned long long* __restrict__ hist) {
  __shared__ unsigned long long sh[8][kRadix];
  for (int e = threadIdx.x; e < 8 * kRadix; e += 256) (&sh[0][0])[e] = 0;
  __syncthreads();
  for (int64_t t = (int64_t)blockIdx.x * 256 + threadIdx.x; t < n_tiles; t += (int64_t)gridDim.x * 256) {
    const unsigned long long c = (unsigned long long)(ranges[2 * t + 1] - ranges[2 * t]);
    if (!c) continue;
    for (int p = 0; p < plan.passes; ++p)
      atomicAdd(&sh[p][((uint64_t)t >> plan.shift[p]) & ((1u << plan.bits[p]) - 1)], c);
  }
  __syncthreads();
  for (int p = 0; p < plan.passes; ++p)
    for (int d = threadIdx.x; d < kRadix; d += 256)
      if (sh[p][d]) atomicAdd(&hist[p * kRadix + d], sh[p][d]);
}

// Exclusive scan of each pass's digit histogram (one block per pass):
// start[p][d] = number of keys with a smaller digit in pass p.
__global__ void __launch_bounds__(kRadix)
k_hist_scan(const unsigned long long* __restrict__ hist, unsigned long long* __restrict__ start) {
  __shared__ unsigned long long s_scan[kRadix / 32 + 1];
  const int p = blockIdx.x, d = threadIdx.x;
  unsigned long long tot;
  start[p * kRadix + d] =
      block_exclusive_scan<unsigned long long, kRadix / 32>(hist[p * kRadix + d], s_scan, &tot);
}

template <class K>
struct SortSmem {
  K keys[kSortTile];
  int32_t vals[kSortTile];
  unsigned int wh[kWarps][kRadix];   // per-warp digit counts -> exclusive offsets
  long long gbase[kRadix];           // global position of the tile's first item of digit d
  unsigned int tex[kRadix];          // tile-local exclusive offset of digit d
  unsigned int scan[kWarps + 1];
  unsigned int tile;
};

template <class K>
__global__ void __launch_bounds__(kSortThreads, GS_SORT_MINB)
k_onesweep(const K* __restrict__ src_k, const int32_t* __restrict__ src_v, bool iota,
           K* __restrict__ dst_k, int32_t* __restrict__ dst_v, int64_t n, int shift, int bits,
           const unsigned long long* __restrict__ hist, unsigned long long* __restrict__ status,
           unsigned int* __restrict__ ticket, bool stall, int32_t* dev_status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SortSmem<K>& S = *reinterpret_cast<SortSmem<K>*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const unsigned mask = (1u << bits) - 1u;
  if (tid == 0) S.tile = atomicAdd(ticket, 1u);
  for (int e = tid; e < kWarps * kRadix; e += kSortThreads) (&S.wh[0][0])[e] = 0;
  __syncthreads();
  const int64_t tile = S.tile;
  const int64_t base = tile * kSortTile;

  // load in warp-striped order: warp w owns items [w*256, w*256+256) of the tile
  K key[kIPT];
  int32_t val[kIPT];
  unsigned dig[kIPT];
  unsigned rank[kIPT];
#pragma unroll
  for (int k = 0; k < kIPT; ++k) {
    const int64_t idx = base + w * (32 * kIPT) + k * 32 + lane;
    if (idx < n) {
      key[k] = src_k[idx];
      val[k] = iota ? (int32_t)idx : src_v[idx];
      dig[k] = digit_of(key[k], shift, mask);
    } else {
      key[k] = 0;
      val[k] = 0;
      dig[k] = kRadix;  // sentinel: not ranked, not written
    }
  }
  // stable rank within the warp: items in (k, lane) order
  const unsigned lt_mask = (1u << lane) - 1u;
#pragma unroll
  for (int k = 0; k < kIPT; ++k) {
    const unsigned peers = __match_any_sync(0xffffffffu, dig[k]);
    unsigned cnt = 0;
    if (dig[k] < kRadix) cnt = S.wh[w][dig[k]];
    __syncwarp();
    if (dig[k] < kRadix && lane == __ffs(peers) - 1) S.wh[w][dig[k]] = cnt + __popc(peers);
    rank[k] = cnt + __popc(peers & lt_mask);
    __syncwarp();
  }
  __syncthreads();

  // per digit: tile count, exclusive offsets across warps
  unsigned tcount = 0;
  if (tid < kRadix) {
#pragma unroll
    for (int ww = 0; ww < kWarps; ++ww) {
      const unsigned c = S.wh[ww][tid];
      S.wh[ww][tid] = tcount;
      tcount += c;
    }
    // publish this tile's aggregate as early as possible
    unsigned long long* st = status + tile * kRadix + tid;
    if (tile == 0) {
      if (!stall) st_relaxed(st, kFlagInc | tcount);
    } else {
      st_relaxed(st, kFlagAgg | tcount);
    }
  }
  // global start of each digit (precomputed per pass)
  const unsigned long long hstart = tid < kRadix ? hist[tid] : 0ull;
  unsigned tstart = 0, ttot;
  tstart = block_exclusive_scan<unsigned, kWarps>(tid < kRadix ? tcount : 0u, S.scan, &ttot);
  if (tid < kRadix) {
    S.tex[tid] = tstart;
    // look back over earlier tiles for this digit, kLookWin predecessors per
    // round trip (their status words are loaded together)
    long long excl = 0;
    if (tile > 0) {
      int64_t j = tile - 1;
      int spins = 0;
      bool found = false, timed_out = false;
      {
        // the nearest predecessor alone first: usually it is already final
        unsigned long long w = ld_relaxed(status + j * kRadix + tid);
        while ((w >> 62) == 0) {
          if (++spins > kSpinCap) {
            dev_flag(dev_status, GS_DEV_TIMEOUT);
            timed_out = true;
            break;
          }
          __nanosleep(32);
          w = ld_relaxed(status + j * kRadix + tid);
        }
        if (!timed_out) {
          excl += (long long)(w & kValMask);
          found = (w >> 62) == 2;
        }
        --j;
      }
      while (j >= 0 && !found && !timed_out) {
        unsigned long long wv[kLookWin];
#pragma unroll
        for (int i = 0; i < kLookWin; ++i)
          wv[i] = (j - i >= 0) ? ld_relaxed(status + (j - i) * kRadix + tid) : kFlagInc;
#pragma unroll
        for (int i = 0; i < kLookWin; ++i) {
          if (found || timed_out) break;
          unsigned long long w = wv[i];
          while ((w >> 62) == 0) {  // not yet published: wait for this one
            if (++spins > kSpinCap) {
              dev_flag(dev_status, GS_DEV_TIMEOUT);
              timed_out = true;
              break;
            }
            __nanosleep(64);
            w = ld_relaxed(status + (j - i) * kRadix + tid);
          }
          if (timed_out) break;
          excl += (long long)(w & kValMask);
          if ((w >> 62) == 2) found = true;
        }
        j -= kLookWin;
      }
      st_relaxed(status + tile * kRadix + tid, kFlagInc | (unsigned long long)(excl + tcount));
    }
    S.gbase[tid] = (long long)hstart + excl;
  }
  __syncthreads();

  // stage in shared memory in digit order (stable)
#pragma unroll
  for (int k = 0; k < kIPT; ++k) {
    if (dig[k] < kRadix) {
      const unsigned pos = S.tex[dig[k]] + S.wh[w][dig[k]] + rank[k];
      S.keys[pos] = key[k];
      S.vals[pos] = val[k];
    }
  }
  __syncthreads();
  const int64_t rem = n - base;
  const int count = rem < kSortTile ? (int)rem : kSortTile;
  for (int e = tid; e < count; e += kSortThreads) {
    const K kk = S.keys[e];
    const unsigned d = digit_of(kk, shift, mask);
    const int64_t gpos = S.gbase[d] + (e - (int64_t)S.tex[d]);
    if (gpos < 0 || gpos >= n) {
      dev_flag(dev_status, GS_DEV_BOUNDS);
      continue;
    }
    dst_k[gpos] = kk;
    dst_v[gpos] = S.vals[e];
  }
}

// ---------------------------------------------------------------------------
// Chain-free digit pass (upsweep / scan / downsweep): per-tile digit counts
// are stored digit-major, scanned per digit across tiles, and each tile then
// scatters to its precomputed offsets.  No tile waits on another.
// ---------------------------------------------------------------------------
template <class K>
__global__ void __launch_bounds__(kSortThreads)
k_upsweep(const K* __restrict__ keys, int64_t n, int shift, int bits, int64_t tiles,
          unsigned int* __restrict__ counts, const int32_t* __restrict__ n_dev) {
  if (n_dev) n = min(n, (int64_t)*n_dev);  // tiles past the count write zero counts
  __shared__ unsigned int sh[kRadix];
  const unsigned mask = (1u << bits) - 1u;
  for (int d = threadIdx.x; d < kRadix; d += kSortThreads) sh[d] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kSortTile;
  if constexpr (sizeof(K) == 4 && kIPT % 4 == 0) {
    // four keys per 128-bit load where the whole quad is in range
#pragma unroll
    for (int k = 0; k < kIPT / 4; ++k) {
      const int64_t q = base + 4 * ((int64_t)k * kSortThreads + threadIdx.x);
      if (q + 3 < n) {
        const uint4 v4 = *reinterpret_cast<const uint4*>(keys + q);
        atomicAdd(&sh[(v4.x >> shift) & mask], 1u);
        atomicAdd(&sh[(v4.y >> shift) & mask], 1u);
        atomicAdd(&sh[(v4.z >> shift) & mask], 1u);
        atomicAdd(&sh[(v4.w >> shift) & mask], 1u);
      } else {
        for (int64_t i = q; i < n && i < q + 4; ++i) atomicAdd(&sh[digit_of(keys[i], shift, mask)], 1u);
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < kIPT; ++k) {
      const int64_t idx = base + (int64_t)k * kSortThreads + threadIdx.x;
      if (idx < n) atomicAdd(&sh[digit_of(keys[idx], shift, mask)], 1u);
    }
  }
  __syncthreads();
  for (int d = threadIdx.x; d < kRadix; d += kSortThreads)
    counts[(int64_t)d * tiles + blockIdx.x] = sh[d];
}

// Block d: counts[d][0..tiles) -> exclusive prefix + global start of digit d.
__global__ void __launch_bounds__(1024)
k_scan_tiles(unsigned int* __restrict__ counts, int64_t tiles,
             const unsigned long long* __restrict__ start) {
  __shared__ unsigned long long s_scan[1024 / 32 + 1];
  const int d = blockIdx.x;
  unsigned int* row = counts + (int64_t)d * tiles;
  unsigned long long carry = start[d];
  for (int64_t t0 = 0; t0 < tiles; t0 += 1024) {
    const int64_t t = t0 + threadIdx.x;
    const unsigned long long c = t < tiles ? row[t] : 0ull;
    unsigned long long tot;
    const unsigned long long ex = block_exclusive_scan<unsigned long long, 32>(c, s_scan, &tot);
    if (t < tiles) row[t] = (unsigned int)(carry + ex);
    carry += tot;
  }
}

template <class K>
__global__ void __launch_bounds__(kSortThreads, GS_SORT_MINB)
k_downsweep(const K* __restrict__ src_k, const int32_t* __restrict__ src_v, bool iota,
            K* __restrict__ dst_k, int32_t* __restrict__ dst_v, int64_t n, int shift, int bits,
            const unsigned int* __restrict__ offsets, int64_t tiles, int32_t* dev_status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SortSmem<K>& S = *reinterpret_cast<SortSmem<K>*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const unsigned mask = (1u << bits) - 1u;
  const int64_t tile = blockIdx.x;
  for (int e = tid; e < kWarps * kRadix; e += kSortThreads) (&S.wh[0][0])[e] = 0;
  // global base of each digit for this tile (stored 32-bit: n < 2^32)
  if (tid < kRadix) S.gbase[tid] = offsets[(int64_t)tid * tiles + tile];
  __syncthreads();
  const int64_t base = tile * kSortTile;
  K key[kIPT];
  int32_t val[kIPT];
  unsigned dig[kIPT];
  unsigned rank[kIPT];
#pragma unroll
  for (int k = 0; k < kIPT; ++k) {
    const int64_t idx = base + w * (32 * kIPT) + k * 32 + lane;
    if (idx < n) {
      key[k] = src_k[idx];
      val[k] = iota ? (int32_t)idx : src_v[idx];
      dig[k] = digit_of(key[k], shift, mask);
    } else {
      key[k] = 0;
      val[k] = 0;
      dig[k] = kRadix;
    }
  }
  const unsigned lt_mask = (1u << lane) - 1u;
#pragma unroll
  for (int k = 0; k < kIPT; ++k) {
    const unsigned peers = __match_any_sync(0xffffffffu, dig[k]);
    unsigned cnt = 0;
    if (dig[k] < kRadix) cnt = S.wh[w][dig[k]];
    __syncwarp();
    if (dig[k] < kRadix && lane == __ffs(peers) - 1) S.wh[w][dig[k]] = cnt + __popc(peers);
    rank[k] = cnt + __popc(peers & lt_mask);
    __syncwarp();
  }
  __syncthreads();
  unsigned tcount = 0;
  if (tid < kRadix) {
#pragma unroll
    for (int ww = 0; ww < kWarps; ++ww) {
      const unsigned c = S.wh[ww][tid];
      S.wh[ww][tid] = tcount;
      tcount += c;
    }
  }
  unsigned ttot;
  const unsigned tstart = block_exclusive_scan<unsigned, kWarps>(tid < kRadix ? tcount : 0u, S.scan, &ttot);
  if (tid < kRadix) S.tex[tid] = tstart;
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kIPT; ++k) {
    if (dig[k] < kRadix) {
      const unsigned pos = S.tex[dig[k]] + S.wh[w][dig[k]] + rank[k];
      S.keys[pos] = key[k];
      S.vals[pos] = val[k];
    }
  }
  __syncthreads();
  const int64_t rem = n - base;
  const int count = rem < kSortTile ? (int)rem : kSortTile;
  for (int e = tid; e < count; e += kSortThreads) {
    const K kk = S.keys[e];
    const unsigned d = digit_of(kk, shift, mask);
    const int64_t gpos = S.gbase[d] + (e - (int64_t)S.tex[d]);
    if (gpos < 0 || gpos >= n) {
      dev_flag(dev_status, GS_DEV_BOUNDS);
      continue;
    }
    dst_k[gpos] = kk;
    dst_v[gpos] = S.vals[e];
  }
}

// Leaner downsweep for 32-bit keys: (key, value) staged as one 64-bit word,
// one per-digit delta (global start - tile-local start), loops sized to the
// pass's active digits.
struct DownSmem32 {
  unsigned long long kv[kSortTile];
  unsigned int wh[kWarps][kRadix];
  int gdelta[kRadix];
  unsigned int scan[kWarps + 1];
};

__global__ void __launch_bounds__(kSortThreads, GS_SORT_MINB)
k_downsweep32(const uint32_t* __restrict__ src_k, const int32_t* __restrict__ src_v, bool iota,
              uint32_t* __restrict__ dst_k, int32_t* __restrict__ dst_v, int n, int shift,
              int bits, const unsigned int* __restrict__ offsets, int tiles, int32_t* dev_status,
              const int32_t* __restrict__ n_dev) {
  if (n_dev) n = min(n, *n_dev);  // tiles past the count write nothing
  extern __shared__ __align__(16) unsigned char smem_raw[];
  DownSmem32& S = *reinterpret_cast<DownSmem32*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const unsigned mask = (1u << bits) - 1u;
  const int nd = 1 << bits;  // active digits
  const int tile = blockIdx.x;
  if (nd >= 4) {
    const int q = nd / 4;  // uint4 words per warp row
    for (int e = tid; e < kWarps * q; e += kSortThreads)
      reinterpret_cast<uint4*>(&S.wh[e / q][0])[e % q] = make_uint4(0u, 0u, 0u, 0u);
  } else {
    for (int e = tid; e < kWarps * nd; e += kSortThreads) S.wh[e / nd][e % nd] = 0u;
  }
  int gb = 0;
  if (tid < nd) gb = (int)offsets[(int64_t)tid * tiles + tile];
  __syncthreads();
  const int base = tile * kSortTile;
  const bool full = base + kSortTile <= n;
  uint32_t key[kIPT];
  int32_t val[kIPT];
  unsigned dig[kIPT];
  unsigned rank[kIPT];
#pragma unroll
  for (int k = 0; k < kIPT; ++k) {
    const int idx = base + w * (32 * kIPT) + k * 32 + lane;
    if (full || idx < n) {
      key[k] = src_k[idx];
      val[k] = iota ? idx : src_v[idx];
      dig[k] = (key[k] >> shift) & mask;
    } else {
      key[k] = 0u;
      val[k] = 0;
      dig[k] = kRadix;
    }
  }
  const unsigned lt_mask = (1u << lane) - 1u;
#pragma unroll
  for (int k = 0; k < kIPT; ++k) {
    const unsigned peers = __match_any_sync(0xffffffffu, dig[k]);
    const bool ok = dig[k] < kRadix;
    const unsigned cnt = ok ? S.wh[w][dig[k]] : 0u;
    __syncwarp();
    if (ok && lane == __ffs(peers) - 1) S.wh[w][dig[k]] = cnt + __popc(peers);
    rank[k] = cnt + __popc(peers & lt_mask);
    __syncwarp();
  }
  __syncthreads();
  unsigned tcount = 0;
  if (tid < nd) {
#pragma unroll
    for (int ww = 0; ww < kWarps; ++ww) {
      const unsigned c = S.wh[ww][tid];
      S.wh[ww][tid] = tcount;
      tcount += c;
    }
  }
  unsigned ttot;
  const unsigned tstart = block_exclusive_scan<unsigned, kWarps>(tid < nd ? tcount : 0u, S.scan, &ttot);
  if (tid < nd) {
    S.gdelta[tid] = gb - (int)tstart;
    // fold the tile-local digit start into the per-warp offsets
#pragma unroll
    for (int ww = 0; ww < kWarps; ++ww) S.wh[ww][tid] += tstart;
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kIPT; ++k)
    if (dig[k] < kRadix)
      S.kv[S.wh[w][dig[k]] + rank[k]] =
          (unsigned long long)key[k] | ((unsigned long long)(uint32_t)val[k] << 32);
  __syncthreads();
  const int count = full ? kSortTile : n - base;
#pragma unroll
  for (int k = 0; k < kIPT; ++k) {
    const int e = k * kSortThreads + tid;
    if (full || e < count) {
      const unsigned long long kv = S.kv[e];
      const uint32_t kk = (uint32_t)kv;
      const int gpos = S.gdelta[(kk >> shift) & mask] + e;
      if ((unsigned)gpos >= (unsigned)n) {
        dev_flag(dev_status, GS_DEV_BOUNDS);
        continue;
      }
      dst_k[gpos] = kk;
      dst_v[gpos] = (int32_t)(kv >> 32);
    }
  }
}

template <class K>
__global__ void k_copy_pairs(const K* __restrict__ sk, K* __restrict__ dk, int32_t* __restrict__ dv,
                             const int32_t* __restrict__ sv, bool iota, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  dk[i] = sk[i];
  dv[i] = iota ? (int32_t)i : sv[i];
}

template <class K>
struct SortWs {
  K* alt_k;
  int32_t* alt_v;
  unsigned long long* hist;
  unsigned long long* hstart;
  unsigned int* tickets;
  unsigned long long* status;
  unsigned int* counts;
  size_t zero_begin, zero_small, zero_bytes, bytes;
};

template <class K>
SortWs<K> carve_sort(void* ws, size_t cap, int64_t n, const SortPlan& p) {
  Carver cv(ws, cap);
  SortWs<K> s;
  s.alt_k = cv.take<K>(n > 0 ? n : 1);
  s.alt_v = cv.take<int32_t>(n > 0 ? n : 1);
  const int64_t tiles = (n + kSortTile - 1) / kSortTile;
  s.hstart = cv.take<unsigned long long>((size_t)8 * kRadix);
  s.hist = cv.take<unsigned long long>((size_t)8 * kRadix);
  s.zero_begin = (size_t)((char*)s.hist - (char*)ws);
  s.tickets = cv.take<unsigned int>(64);
  // the onesweep look-back words, or (same region) the per-tile digit
  // counts of the upsweep/downsweep passes
  s.zero_small = cv.off - s.zero_begin;   // histograms and tickets
  s.status = cv.take<unsigned long long>((size_t)(p.passes > 0 ? p.passes : 1) * (tiles > 0 ? tiles : 1) * kRadix);
  s.counts = reinterpret_cast<unsigned int*>(s.status);
  s.bytes = cv.off;
  s.zero_bytes = s.bytes - s.zero_begin;
  return s;
}

template <class K>
gs_status sort_impl(const K* keys_in, K* keys, int32_t* vals, bool iota, bool stall, int64_t n,
                    int begin_bit, int end_bit, void* ws, size_t ws_bytes, int32_t* dev_status,
                    cudaStream_t s, const int64_t* ranges = nullptr, int64_t n_tiles = 0,
                    bool chained = false, const int32_t* n_dev = nullptr) {
  // n_dev: the number of pairs is read on the device (at most n); only the
  // lean 32-bit passes take it
  chained = chained || stall;
  if (n_dev && (chained || sizeof(K) != 4 || ranges)) return GS_ERR_UNSUPPORTED;
  const int kbits = (int)(8 * sizeof(K));
  if (n < 0 || begin_bit < 0 || end_bit > kbits || begin_bit > end_bit) return GS_ERR_ARG;
  if (n == 0) return GS_OK;
  if (!keys || !vals || (!keys_in && !keys)) return GS_ERR_ARG;
  if (n > (int64_t)INT32_MAX) return GS_ERR_UNSUPPORTED;  // values are int32 positions
  const SortPlan plan = plan_sort(begin_bit, end_bit);
  SortWs<K> w = carve_sort<K>(ws, ws_bytes, n, plan);
  if (!ws || w.bytes > ws_bytes) return GS_ERR_CAPACITY;
  if (!aligned(ws, 256)) return GS_ERR_ARG;
  const K* first_k = keys_in ? keys_in : keys;
  if (plan.passes == 0) {
    if (keys_in || iota)
      k_copy_pairs<K><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(first_k, keys, vals, vals, iota, n);
    GS_LAUNCH_CHECK();
    return GS_OK;
  }
  GS_TRY(cudaMemsetAsync((char*)ws + w.zero_begin, 0, chained ? w.zero_bytes : w.zero_small, s));
  const int64_t tiles = (n + kSortTile - 1) / kSortTile;
  if (ranges) {
    const int64_t hb = (n_tiles + 255) / 256;
    k_hist_from_ranges<<<(unsigned)(hb < 296 ? (hb > 0 ? hb : 1) : 296), 256, 0, s>>>(
        ranges, n_tiles, plan, w.hist);
  } else {
    const int hist_blocks = (int)(tiles < 1184 ? tiles : 1184);
    k_hist<K><<<hist_blocks, kSortThreads, 0, s>>>(first_k, n, plan, w.hist, n_dev);
  }
  GS_LAUNCH_CHECK();
  k_hist_scan<<<plan.passes, kRadix, 0, s>>>(w.hist, w.hstart);
  GS_LAUNCH_CHECK();
  const size_t smem = sizeof(SortSmem<K>);
  // the lean 32-bit downsweep indexes with int
  const bool use32 = sizeof(K) == 4 && n <= (int64_t)INT32_MAX - kSortTile;
  // a shared-memory carveout large enough for several blocks per SM
  if (chained) {
    static std::atomic<unsigned long long> done{0};
    GS_TRY(smem_attrs_once((const void*)k_onesweep<K>, (int)smem, &done));
  } else if (use32) {
    static std::atomic<unsigned long long> done{0};
    GS_TRY(smem_attrs_once((const void*)k_downsweep32, (int)sizeof(DownSmem32), &done));
  } else {
    static std::atomic<unsigned long long> done{0};
    GS_TRY(smem_attrs_once((const void*)k_downsweep<K>, (int)smem, &done));
  }
  const K* sk = first_k;
  const int32_t* sv = vals;
  bool siota = iota;
  for (int p = 0; p < plan.passes; ++p) {
    K* dk = (p & 1) ? keys : w.alt_k;
    int32_t* dv = (p & 1) ? vals : w.alt_v;
    if (chained) {
      k_onesweep<K><<<(unsigned)tiles, kSortThreads, smem, s>>>(
          sk, sv, siota, dk, dv, n, plan.shift[p], plan.bits[p], w.hstart + (size_t)p * kRadix,
          w.status + (size_t)p * tiles * kRadix, w.tickets + p, stall && p == 0, dev_status);
      GS_LAUNCH_CHECK();
      sk = dk;
      sv = dv;
      siota = false;
      continue;
    }
    k_upsweep<K><<<(unsigned)tiles, kSortThreads, 0, s>>>(sk, n, plan.shift[p], plan.bits[p], tiles,
                                                            w.counts, n_dev);
    GS_LAUNCH_CHECK();
    k_scan_tiles<<<kRadix, 1024, 0, s>>>(w.counts, tiles, w.hstart + (size_t)p * kRadix);
    GS_LAUNCH_CHECK();
    if (use32) {
      k_downsweep32<<<(unsigned)tiles, kSortThreads, sizeof(DownSmem32), s>>>(
          reinterpret_cast<const uint32_t*>(sk), sv, siota, reinterpret_cast<uint32_t*>(dk), dv,
          (int)n, plan.shift[p], plan.bits[p], w.counts, (int)tiles, dev_status, n_dev);
    } else {
      k_downsweep<K><<<(unsigned)tiles, kSortThreads, smem, s>>>(
          sk, sv, siota, dk, dv, n, plan.shift[p], plan.bits[p], w.counts, tiles, dev_status);
    }
    GS_LAUNCH_CHECK();
    sk = dk;
    sv = dv;
    siota = false;
  }
  return GS_OK;
}

}  // namespace

// The depth order's sort: 32-bit keys, values 0..count-1, the count read on
// the device (at most n).  Library-internal (hidden), used by gs_depth_order.
__attribute__((visibility("hidden")))
gs_status sort32_iota_devcount(const uint32_t* keys_in, uint32_t* keys, int32_t* vals, int64_t n,
                               const int32_t* n_dev, void* ws, size_t ws_bytes,
                               int32_t* dev_status, cudaStream_t s) {
  return sort_impl<uint32_t>(keys_in, keys, vals, true, false, n, 0, 32, ws, ws_bytes, dev_status,
                             s, nullptr, 0, false, n_dev);
}

}  // namespace gs

using namespace gs;

extern "C" size_t gs_sort_workspace_size(int64_t n, int32_t key_bytes, int32_t begin_bit,
                                         int32_t end_bit) {
  if (n < 0 || begin_bit < 0 || end_bit < begin_bit) return 0;
  const SortPlan p = plan_sort(begin_bit, end_bit);
  if (key_bytes == 8) return carve_sort<uint64_t>(nullptr, 0, n, p).bytes;
  if (key_bytes == 4) return carve_sort<uint32_t>(nullptr, 0, n, p).bytes;
  return 0;
}

extern "C" gs_status gs_sort_keys(uint64_t* keys, int32_t* vals, int64_t n, int32_t begin_bit,
                                  int32_t end_bit, void* ws, size_t ws_bytes, int32_t* dev_status,
                                  gs_stream stream) {
  return sort_impl<uint64_t>(nullptr, keys, vals, false, false, n, begin_bit, end_bit, ws,
                             ws_bytes, dev_status, to_stream(stream));
}

extern "C" gs_status gs_sort_tiles(uint32_t* tile_keys, int32_t* vals, int64_t n,
                                   const int64_t* ranges, int64_t n_tiles, void* ws,
                                   size_t ws_bytes, int32_t* dev_status, gs_stream stream) {
  if (n < 0 || n_tiles < 0 || (n_tiles > 0 && !ranges)) return GS_ERR_ARG;
  if (n_tiles > ((int64_t)1 << 32)) return GS_ERR_UNSUPPORTED;
  const int bits = n_tiles > 1 ? 64 - __builtin_clzll((unsigned long long)(n_tiles - 1)) : 0;
  return sort_impl<uint32_t>(nullptr, tile_keys, vals, false, false, n, 0, bits, ws, ws_bytes,
                             dev_status, to_stream(stream), ranges, n_tiles);
}

extern "C" gs_status gs_sort_keys32(const uint32_t* keys_in, uint32_t* keys, int32_t* vals,
                                    int64_t n, int32_t begin_bit, int32_t end_bit, uint32_t flags,
                                    void* ws, size_t ws_bytes, int32_t* dev_status,
                                    gs_stream stream) {
  if (flags & ~(GS_SORT_IOTA | GS_SORT_ONESWEEP | GS_SORT_TEST_STALL)) return GS_ERR_ARG;
  return sort_impl<uint32_t>(keys_in, keys, vals, (flags & GS_SORT_IOTA) != 0,
                             (flags & GS_SORT_TEST_STALL) != 0, n, begin_bit, end_bit, ws,
                             ws_bytes, dev_status, to_stream(stream), nullptr, 0,
                             (flags & GS_SORT_ONESWEEP) != 0);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of gs_sort_keys32.
//
// Some callers cannot allocate device memory at the moment they need a sort:
// for example a plugin inside a host application whose allocator has already
// reserved the whole device, or a latency-critical loop where an allocation
// (which may synchronise the device) is not acceptable.  For them the scratch
// of the sort lives in this file-scope device array instead of a caller
// workspace.  Every GPU that loads the library holds the array until exit.
// ---------------------------------------------------------------------------
namespace gs {
namespace {

constexpr size_t kNoAllocScratchBytes = GS_SORT_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_sort_scratch[kNoAllocScratchBytes];

// Upper bound of carve_sort<uint32_t>'s layout (each region rounded up to
// 256 bytes, the look-back / per-tile count region at its largest, 4 passes
// of 8-bit digits for 32-bit keys), so that a build with other tile sizes
// cannot make a call with n <= the maximum run out of scratch.
constexpr size_t ru256(size_t x) { return (x + 255) / 256 * 256; }
constexpr size_t noalloc_plan_bound(size_t n) {
  return ru256(n * 4) + ru256(n * 4) + ru256(8 * kRadix * 8) + ru256(8 * kRadix * 8) +
         ru256(64 * 4) + 4 * ((n + kSortTile - 1) / kSortTile) * kRadix * 8;
}
static_assert(noalloc_plan_bound(GS_SORT_NOALLOC_MAX_N) <= kNoAllocScratchBytes,
              "the allocation-free sort's array must hold the plan of its largest size");

// Device address of g_sort_scratch in the current device's context.  It is
// looked up on every call (a cheap host-side lookup once the module is
// loaded) rather than cached, because a cached address would go stale if
// the context were destroyed and recreated (cudaDeviceReset).  The first
// call on a device may load the module; make it before any stream capture.
gs_status scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_sort_scratch) != cudaSuccess || !p) {
    (void)cudaGetLastError();  // leave no sticky error for the next call
    return GS_ERR_CUDA;
  }
  *out = p;
  return GS_OK;
}

}  // namespace
}  // namespace gs

extern "C" gs_status gs_sort_keys32_noalloc(const uint32_t* keys_in, uint32_t* keys,
                                            int32_t* vals, int64_t n, int32_t begin_bit,
                                            int32_t end_bit, uint32_t flags, int32_t* dev_status,
                                            gs_stream stream) {
  // the stall hook of the bounded-wait test is not accepted here: a stalled
  // call would leave the shared array mid look-back
  if (flags & ~(GS_SORT_IOTA | GS_SORT_ONESWEEP)) return GS_ERR_ARG;
  if (n < 0) return GS_ERR_ARG;
  if (n > GS_SORT_NOALLOC_MAX_N) return GS_ERR_CAPACITY;
  if (n == 0) return GS_OK;
  void* scratch = nullptr;
  const gs_status st = scratch_address(&scratch);
  if (st != GS_OK) return st;
  // the whole plan must fit the array (it does for every n <= the maximum)
  if (gs_sort_workspace_size(n, 4, begin_bit, end_bit) > kNoAllocScratchBytes)
    return GS_ERR_CAPACITY;
  return sort_impl<uint32_t>(keys_in, keys, vals, (flags & GS_SORT_IOTA) != 0, false, n,
                             begin_bit, end_bit, scratch, kNoAllocScratchBytes, dev_status,
                             to_stream(stream), nullptr, 0, (flags & GS_SORT_ONESWEEP) != 0);
}
