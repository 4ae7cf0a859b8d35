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
               short4* __restrict__ out, const int32_t* __restrict__ n_dev) {
  if (n_dev) n = min(n, (int64_t)*n_dev);
  const int64_t j = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (j < n) out[j] = rect[order[j]];
}

// BLK = 1: entries per tile; BLK = GS_TILE_BLOCK: entries per block of
// BLK x BLK tiles (the candidate's tile rect widened to whole blocks).
template <int BLK>
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
      int rx0 = r.x, ry0 = r.y, rx1 = r.z, ry1 = r.w;
      if (rx1 <= rx0 || ry1 <= ry0) rx1 = rx0 = ry1 = ry0 = 0;  // culled (dense layout)
      if (BLK > 1 && rx1 > rx0) {  // a non-empty rect has r.z, r.w >= 1
        rx0 /= BLK;
        ry0 /= BLK;
        rx1 = (rx1 - 1) / BLK + 1;
        ry1 = (ry1 - 1) / BLK + 1;
      }
      x0 = max(rx0, leaf.x0);
      const int x1 = min(rx1, leaf.x1);
      y0 = max(ry0, leaf.y0);
      const int y1 = min(ry1, leaf.y1);
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

// ---------------------------------------------------------------------------
// Two-level binning.  Per view, every candidate is listed once per block of
// GS_TILE_BLOCK x GS_TILE_BLOCK tiles that its rect meets, in depth order
// (k_bin<GS_TILE_BLOCK> + a stable sort on the block id).  Per Leaf, each
// block list is cut into chunks of kExpChunk entries; a chunk turns each
// candidate's rect into a 64-bit mask over the block's tiles (clipped to the
// Leaf) and ranks the candidates per tile with warp ballots, so the entry of
// (candidate, tile) goes straight to its place in the tile's segment, whose
// begin the tile SAT gives.  Two passes: per-(chunk, tile) counts, an
// exclusive scan over the chunks of each block, then the writes.  The order
// within a tile is the block list's order, i.e. the depth order.
// ---------------------------------------------------------------------------
constexpr int kBlk = GS_TILE_BLOCK;
static_assert(kBlk == 8, "tile masks are 64-bit");
constexpr int kExpThreads = 256;
constexpr int kExpRounds = 4;
constexpr int kExpChunk = kExpThreads * kExpRounds;
constexpr int kExpWarps = kExpThreads / 32;

struct LeafBlocks {
  int bx0, by0, bw, bh;  // the blocks that meet the Leaf
};

__host__ __device__ inline LeafBlocks leaf_blocks(gs_rect leaf) {
  LeafBlocks b;
  b.bx0 = leaf.x0 / kBlk;
  b.by0 = leaf.y0 / kBlk;
  b.bw = (leaf.x1 - 1) / kBlk + 1 - b.bx0;
  b.bh = (leaf.y1 - 1) / kBlk + 1 - b.by0;
  return b;
}

// rect ∩ leaf ∩ block (bx, by) in block-local tile coordinates; empty when
// x1 <= x0 (then x0 = x1 = y0 = y1 = 0).
struct LocalRect {
  int x0, x1, y0, y1;
};

__device__ __forceinline__ LocalRect local_rect(short4 r, gs_rect leaf, int bx, int by) {
  const int ox = bx * kBlk, oy = by * kBlk;
  LocalRect q;
  q.x0 = max(max((int)r.x, leaf.x0), ox) - ox;
  q.x1 = min(min((int)r.z, leaf.x1), ox + kBlk) - ox;
  q.y0 = max(max((int)r.y, leaf.y0), oy) - oy;
  q.y1 = min(min((int)r.w, leaf.y1), oy + kBlk) - oy;
  if (q.x1 <= q.x0 || q.y1 <= q.y0) q.x0 = q.x1 = q.y0 = q.y1 = 0;
  return q;
}

// byte x set to 1 for x in [x0, x1) (0 <= x0 <= x1 <= 8)
__device__ __forceinline__ uint64_t row_bytes(int x0, int x1) {
  const uint64_t hi = x1 >= kBlk ? ~0ull : ((1ull << (8 * x1)) - 1ull);
  const uint64_t lo = x0 >= kBlk ? ~0ull : ((1ull << (8 * x0)) - 1ull);
  return (hi & ~lo) & 0x0101010101010101ull;
}

// bit (ly * 8 + lx) set for the tiles of the local rect
__device__ __forceinline__ uint64_t tile_mask(const LocalRect& q) {
  const uint64_t row = (uint64_t)(((1u << q.x1) - 1u) & ~((1u << q.x0) - 1u));
  return row_bytes(q.y0, q.y1) * row;
}

// This warp's count of tile (lane & 7, row) for rows lane >> 3 (lo) and
// 4 + (lane >> 3) (hi), i.e. tiles lane and 32 + lane: per row, the lanes'
// byte-packed rows are summed with one reduction per 4 tiles (counts <= 32
// fit a byte).
__device__ __forceinline__ void warp_tile_counts(const LocalRect& q, int lane, unsigned& c_lo,
                                                 unsigned& c_hi) {
  const uint64_t rb = row_bytes(q.x0, q.x1);
  const int ymin = __reduce_min_sync(0xffffffffu, q.x1 > q.x0 ? q.y0 : kBlk);
  const int ymax = __reduce_max_sync(0xffffffffu, q.y1);
  const int my_row = lane >> 3, my_x = lane & 7;
  c_lo = c_hi = 0;
  for (int y = ymin; y < ymax; ++y) {
    const bool in = q.y0 <= y && y < q.y1;
    const unsigned wl = __reduce_add_sync(0xffffffffu, in ? (unsigned)rb : 0u);
    const unsigned wh = __reduce_add_sync(0xffffffffu, in ? (unsigned)(rb >> 32) : 0u);
    const unsigned v = ((my_x < 4 ? wl : wh) >> (8 * (my_x & 3))) & 0xffu;
    if (my_row == y) c_lo = v;
    if (my_row + 4 == y) c_hi = v;
  }
}

// chunk_start[i] = first chunk of the i-th block of the Leaf (row-major over
// LeafBlocks), chunk_start[nbl] = total; one block of 1024 threads.
__global__ void __launch_bounds__(1024)
k_expand_plan(const int64_t* __restrict__ block_ranges, int BW, LeafBlocks lb,
              int64_t* __restrict__ chunk_start, int64_t max_chunks, int32_t* dev_status) {
  __shared__ long long s_scan[33];
  const int nbl = lb.bw * lb.bh;
  long long carry = 0;
  for (int base = 0; base < nbl; base += 1024) {
    const int i = base + threadIdx.x;
    long long c = 0;
    if (i < nbl) {
      const int64_t b = (int64_t)(lb.by0 + i / lb.bw) * BW + lb.bx0 + i % lb.bw;
      const long long len = block_ranges[2 * b + 1] - block_ranges[2 * b];
      c = (len + kExpChunk - 1) / kExpChunk;
    }
    long long tot;
    const long long ex = block_exclusive_scan<long long, 32>(c, s_scan, &tot);
    if (i < nbl) chunk_start[i] = carry + ex;
    carry += tot;
  }
  if (threadIdx.x == 0) {
    chunk_start[nbl] = carry;
    if (carry > max_chunks) dev_flag(dev_status, GS_DEV_BOUNDS);
  }
}

struct ChunkPos {
  int i, bx, by;
  int64_t begin, end;
};

// the block and entry range of chunk g (g < total)
__device__ __forceinline__ ChunkPos chunk_pos(int64_t g, const int64_t* __restrict__ chunk_start,
                                              int nbl, LeafBlocks lb, int BW,
                                              const int64_t* __restrict__ block_ranges) {
  int lo = 0, hi = nbl - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (chunk_start[mid] <= g) lo = mid;
    else hi = mid - 1;
  }
  ChunkPos c;
  c.i = lo;
  c.bx = lb.bx0 + lo % lb.bw;
  c.by = lb.by0 + lo / lb.bw;
  const int64_t b = (int64_t)c.by * BW + c.bx;
  c.begin = block_ranges[2 * b] + (g - chunk_start[lo]) * kExpChunk;
  const int64_t e = block_ranges[2 * b + 1];
  c.end = c.begin + kExpChunk < e ? c.begin + kExpChunk : e;
  return c;
}

__global__ void __launch_bounds__(kExpThreads)
k_expand_count(const short4* __restrict__ rect, const int32_t* __restrict__ block_vals,
               const int64_t* __restrict__ block_ranges, int BW, LeafBlocks lb, gs_rect leaf,
               const int64_t* __restrict__ chunk_start, int32_t* __restrict__ cnt) {
  __shared__ unsigned int s_wc[kExpWarps][64];
  const int nbl = lb.bw * lb.bh;
  const int64_t g = blockIdx.x;
  if (g >= chunk_start[nbl]) return;
  const ChunkPos c = chunk_pos(g, chunk_start, nbl, lb, BW, block_ranges);
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  unsigned acc_lo = 0, acc_hi = 0;  // lane j: tiles j and 32 + j
#pragma unroll 1
  for (int k = 0; k < kExpRounds; ++k) {
    const int64_t p = c.begin + k * kExpThreads + t;
    LocalRect q{0, 0, 0, 0};
    if (p < c.end) q = local_rect(rect[block_vals[p]], leaf, c.bx, c.by);
    unsigned n_lo, n_hi;
    warp_tile_counts(q, lane, n_lo, n_hi);
    acc_lo += n_lo;
    acc_hi += n_hi;
  }
  s_wc[w][lane] = acc_lo;
  s_wc[w][32 + lane] = acc_hi;
  __syncthreads();
  if (t < 64) {
    unsigned sum = 0;
#pragma unroll
    for (int ww = 0; ww < kExpWarps; ++ww) sum += s_wc[ww][t];
    cnt[g * 64 + t] = (int32_t)sum;
  }
}

// one thread per (block of the Leaf, tile of the block): the exclusive scan
// of the tile's chunk counts, started at the tile's begin in the Leaf list;
// the counts must add up to the tile's SAT count.
__global__ void __launch_bounds__(256)
k_expand_scan(const int32_t* __restrict__ cnt, const int64_t* __restrict__ chunk_start,
              LeafBlocks lb, gs_rect leaf, const int64_t* __restrict__ ranges,
              int64_t* __restrict__ base, int64_t max_chunks, int32_t* dev_status) {
  const int nbl = lb.bw * lb.bh;
  const int64_t idx = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (idx >= (int64_t)nbl * 64) return;
  const int i = (int)(idx >> 6), j = (int)(idx & 63);
  const int tx = (lb.bx0 + i % lb.bw) * kBlk + (j & 7);
  const int ty = (lb.by0 + i / lb.bw) * kBlk + (j >> 3);
  // (a plan over max_chunks has already been flagged by k_expand_plan)
  const int64_t g0 = min(chunk_start[i], max_chunks), g1 = min(chunk_start[i + 1], max_chunks);
  if (tx < leaf.x0 || tx >= leaf.x1 || ty < leaf.y0 || ty >= leaf.y1) {
    for (int64_t g = g0; g < g1; ++g) base[g * 64 + j] = 0;
    return;
  }
  const int64_t lt = (int64_t)(ty - leaf.y0) * (leaf.x1 - leaf.x0) + (tx - leaf.x0);
  long long run = ranges[2 * lt];
  for (int64_t g = g0; g < g1; ++g) {
    base[g * 64 + j] = run;
    run += cnt[g * 64 + j];
  }
  if (run != ranges[2 * lt + 1]) dev_flag(dev_status, GS_DEV_BOUNDS);
}

__global__ void __launch_bounds__(kExpThreads)
k_expand_write(const short4* __restrict__ rect, const int32_t* __restrict__ block_vals,
               const int64_t* __restrict__ block_ranges, int BW, LeafBlocks lb, gs_rect leaf,
               const int64_t* __restrict__ chunk_start, const int64_t* __restrict__ base,
               int32_t* __restrict__ vals, int32_t capacity, int32_t* dev_status) {
  __shared__ int s_cur[64];
  __shared__ int s_off[kExpWarps][64];
  __shared__ unsigned int s_wc[kExpWarps][64];
  const int nbl = lb.bw * lb.bh;
  const int64_t g = blockIdx.x;
  if (g >= chunk_start[nbl]) return;
  const ChunkPos c = chunk_pos(g, chunk_start, nbl, lb, BW, block_ranges);
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;
  // positions fit 32 bits: the host limits a Leaf list to INT32_MAX entries
  if (t < 64) s_cur[t] = (int)base[g * 64 + t];
  bool bad = false;
#pragma unroll 1
  for (int k = 0; k < kExpRounds; ++k) {
    const int64_t p = c.begin + k * kExpThreads + t;
    LocalRect q{0, 0, 0, 0};
    int32_t slot = 0;
    if (p < c.end) {
      slot = block_vals[p];
      q = local_rect(rect[slot], leaf, c.bx, c.by);
    }
    unsigned n_lo, n_hi;
    warp_tile_counts(q, lane, n_lo, n_hi);
    s_wc[w][lane] = n_lo;
    s_wc[w][32 + lane] = n_hi;
    const uint64_t m = tile_mask(q);
    const unsigned mlo = (unsigned)m, mhi = (unsigned)(m >> 32);
    const unsigned olo = __reduce_or_sync(0xffffffffu, mlo);
    const unsigned ohi = __reduce_or_sync(0xffffffffu, mhi);
    __syncthreads();
    if (t < 64) {
      int run = s_cur[t];
#pragma unroll
      for (int ww = 0; ww < kExpWarps; ++ww) {
        s_off[ww][t] = run;
        run += (int)s_wc[ww][t];
      }
      s_cur[t] = run;
    }
    __syncthreads();
    // one coalesced store per tile: the warp's entries of tile j are
    // consecutive in the tile's segment, in lane (= list) order
    for (unsigned r = olo; r; r &= r - 1) {
      const int j = __ffs(r) - 1;
      const bool mine = (mlo >> j) & 1u;
      const unsigned bal = __ballot_sync(0xffffffffu, mine);
      if (mine) {
        const int pos = s_off[w][j] + __popc(bal & lt_mask);
        if ((unsigned)pos < (unsigned)capacity) vals[pos] = slot;
        else bad = true;
      }
    }
    for (unsigned r = ohi; r; r &= r - 1) {
      const int j = __ffs(r) - 1;
      const bool mine = (mhi >> j) & 1u;
      const unsigned bal = __ballot_sync(0xffffffffu, mine);
      if (mine) {
        const int pos = s_off[w][32 + j] + __popc(bal & lt_mask);
        if ((unsigned)pos < (unsigned)capacity) vals[pos] = slot;
        else bad = true;
      }
    }
    __syncthreads();  // s_wc / s_off are rewritten by the next round
  }
  if (bad) dev_flag(dev_status, GS_DEV_BOUNDS);
}

// ---------------------------------------------------------------------------
// Block lists by a counting scatter (no sort), for grids of up to
// kScatMaxBlocks blocks.  The candidates in depth order are cut into chunks
// of `chunk` candidates.  (A) k_blk_count: per chunk, its entries per block
// (a candidate has one entry in each block its tile rect meets).  (S)
// k_blk_scan: per block, the exclusive scan of those counts over the chunks,
// offset by the block's start in the block lists (from the block SAT), so
// offs[c][b] is where chunk c's first entry of block b goes.  (B)
// k_blk_scatter: one warp per chunk walks its candidates in depth order and
// writes each entry to offs[c][b] + the entries of block b it has written
// so far (a cursor per block in shared memory, advanced by match_any
// groups), so every block list is in depth order with ties by candidate
// position: the order of a stable sort of (block, depth) keys.
// ---------------------------------------------------------------------------
#ifndef GS_SCAT_MAX_BLOCKS
#define GS_SCAT_MAX_BLOCKS 4096
#endif
constexpr int kScatMaxBlocks = GS_SCAT_MAX_BLOCKS;
constexpr size_t kScatMaxSmem = 160 << 10;  // the scatter's per-warp count grids
constexpr int64_t kScatCountBudget = 4 << 20;  // counts per view (16 MB)

int64_t scat_chunk(int64_t n_cand, int64_t nblocks) {
  int64_t c = (n_cand * nblocks + kScatCountBudget - 1) / kScatCountBudget;
  c = c < 1024 ? 1024 : c;
  return (c + 31) / 32 * 32;
}

struct BlockRect {
  int bx0, by0, bw, n;  // first block, width in blocks, number of blocks (0 = none)
};

__device__ __forceinline__ BlockRect block_rect(short4 r, int BW, int BH) {
  BlockRect b{0, 0, 1, 0};
  if (r.z <= r.x || r.w <= r.y) return b;  // empty (a culled Gaussian of the dense layout)
  const int bx0 = r.x / GS_TILE_BLOCK, by0 = r.y / GS_TILE_BLOCK;
  const int bx1 = min((r.z - 1) / GS_TILE_BLOCK + 1, BW), by1 = min((r.w - 1) / GS_TILE_BLOCK + 1, BH);
  if (bx1 <= bx0 || by1 <= by0) return b;
  b.bx0 = bx0;
  b.by0 = by0;
  b.bw = bx1 - bx0;
  b.n = b.bw * (by1 - by0);
  return b;
}

constexpr int kScatSeg = 64;  // chunk segments of the offsets' scan

// Per chunk, its entries per block through a 2D difference grid in shared
// memory: 4 atomics per candidate at its block rect's corners, then a 2D
// prefix sum (rows, then columns), so a candidate costs the same whatever
// its size.
__global__ void __launch_bounds__(256)
k_blk_count(const short4* __restrict__ drect, int64_t n_cand, int64_t chunk, int BW, int BH,
            uint32_t* __restrict__ counts) {
  extern __shared__ int32_t s_d[];  // [(BH + 1) * (BW + 1)]
  const int sw = BW + 1, cells = (BH + 1) * sw;
  for (int b = threadIdx.x; b < cells; b += 256) s_d[b] = 0;
  __syncthreads();
  const int64_t c = blockIdx.x;
  const int64_t j1 = min(n_cand, (c + 1) * chunk);
  for (int64_t base = c * chunk; base < j1; base += 4 * 256) {
    short4 r[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {  // four loads in flight per thread
      const int64_t j = base + k * 256 + threadIdx.x;
      r[k] = j < j1 ? drect[j] : make_short4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const BlockRect br = block_rect(r[k], BW, BH);
      if (br.n == 0) continue;
      const int bx1 = br.bx0 + br.bw, by1 = br.by0 + br.n / br.bw;
      atomicAdd(&s_d[br.by0 * sw + br.bx0], 1);
      atomicAdd(&s_d[br.by0 * sw + bx1], -1);
      atomicAdd(&s_d[by1 * sw + br.bx0], -1);
      atomicAdd(&s_d[by1 * sw + bx1], 1);
    }
  }
  __syncthreads();
  for (int y = threadIdx.x; y < BH; y += 256) {  // prefix along each row
    int run = 0;
    for (int x = 0; x < BW; ++x) {
      run += s_d[y * sw + x];
      s_d[y * sw + x] = run;
    }
  }
  __syncthreads();
  for (int x = threadIdx.x; x < BW; x += 256) {  // then down each column
    int run = 0;
    for (int y = 0; y < BH; ++y) {
      run += s_d[y * sw + x];
      s_d[y * sw + x] = run;
    }
  }
  __syncthreads();
  const int nbk = BW * BH;
  for (int b = threadIdx.x; b < nbk; b += 256) counts[c * nbk + b] = (uint32_t)s_d[(b / BW) * sw + b % BW];
}

// Offsets in two levels over kScatSeg segments of chunks.  One CTA per
// (32 blocks, segment): lane = block, the 8 warps split the segment.
// k_blk_segsum: the segment's total per block.
__global__ void __launch_bounds__(256)
k_blk_segsum(const uint32_t* __restrict__ counts, int64_t n_chunks, int nbk,
             uint32_t* __restrict__ segtot) {
  __shared__ uint32_t s_tot[8][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int b = blockIdx.x * 32 + lane;
  const int64_t L = (n_chunks + kScatSeg - 1) / kScatSeg;
  const int64_t c0 = min(n_chunks, blockIdx.y * L), c1 = min(n_chunks, c0 + L);
  const int64_t l = (c1 - c0 + 7) / 8;
  const int64_t a0 = min(c1, c0 + w * l), a1 = min(c1, a0 + l);
  uint32_t tot = 0;
  if (b < nbk) {
#pragma unroll 4
    for (int64_t c = a0; c < a1; ++c) tot += counts[c * nbk + b];
  }
  s_tot[w][lane] = tot;
  __syncthreads();
  if (w == 0 && b < nbk) {
    uint32_t t = 0;
#pragma unroll
    for (int ww = 0; ww < 8; ++ww) t += s_tot[ww][lane];
    segtot[(int64_t)blockIdx.y * nbk + b] = t;
  }
}

// k_blk_offs: counts[c][b] <- the block list position of chunk c's first
// entry of block b (exclusive scan over the chunks, from the block's start).
__global__ void __launch_bounds__(256)
k_blk_offs(uint32_t* __restrict__ counts, int64_t n_chunks, int nbk,
           const uint32_t* __restrict__ segtot, const int64_t* __restrict__ block_ranges,
           int32_t* dev_status) {
  __shared__ uint32_t s_tot[8][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int b = blockIdx.x * 32 + lane;
  const int64_t L = (n_chunks + kScatSeg - 1) / kScatSeg;
  const int64_t c0 = min(n_chunks, blockIdx.y * L), c1 = min(n_chunks, c0 + L);
  const int64_t l = (c1 - c0 + 7) / 8;
  const int64_t a0 = min(c1, c0 + w * l), a1 = min(c1, a0 + l);
  uint32_t tot = 0;
  if (b < nbk) {
#pragma unroll 4
    for (int64_t c = a0; c < a1; ++c) tot += counts[c * nbk + b];
  }
  s_tot[w][lane] = tot;
  __syncthreads();
  if (b >= nbk) return;
  int64_t run = block_ranges[2 * b];
  for (int s = 0; s < (int)blockIdx.y; ++s) run += segtot[(int64_t)s * nbk + b];
  for (int ww = 0; ww < w; ++ww) run += s_tot[ww][lane];
  for (int64_t c = a0; c < a1; ++c) {
    const uint32_t v = counts[c * nbk + b];
    counts[c * nbk + b] = (uint32_t)run;
    run += v;
  }
  // the last chunk of the last segment ends at the block's end
  if (blockIdx.y == gridDim.y - 1 && w == 7 && run != block_ranges[2 * b + 1])
    dev_flag(dev_status, GS_DEV_BOUNDS);
}

// One CTA of kScatWarps warps per chunk; warp w takes the w-th contiguous
// part of the chunk.  Each warp counts its part per block in its own 2D
// difference grid in shared memory; the prefix sums turn the grids into
// counts, and the CTA turns those into each warp's start per block (the
// chunk's offset plus the counts of the warps before it).  Each warp then
// emits its part in rounds of 32 candidates, entries in (candidate, block
// row-major) order, 32 at a time, advancing its cursors by match_any groups.
// The row of entry q of a w-block-wide rect is floor((q + 0.5) / w) in
// fp32: exact, since q + w < 2^21 keeps the product's error below 0.5 / w.
constexpr int kScatWarps = 8;

__global__ void __launch_bounds__(kScatWarps * 32)
k_blk_scatter(const short4* __restrict__ drect, const int32_t* __restrict__ order,
              int64_t n_cand, int64_t chunk, int BW, int BH, const uint32_t* __restrict__ offs,
              int32_t* __restrict__ block_vals, int64_t capacity, int32_t* dev_status) {
  extern __shared__ int32_t s_g[];  // [kScatWarps][(BH + 1) * (BW + 1)]
  __shared__ int s_ex[kScatWarps][32], s_bx[kScatWarps][32], s_by[kScatWarps][32],
      s_bw[kScatWarps][32], s_slot[kScatWarps][32];
  __shared__ float s_rw[kScatWarps][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int sw = BW + 1, cells = (BH + 1) * sw, nbk = BW * BH;
  int32_t* g = s_g + w * cells;
  const int64_t c = blockIdx.x;
  const int64_t cj0 = c * chunk, cj1 = min(n_cand, cj0 + chunk);
  const int64_t part = (cj1 - cj0 + kScatWarps - 1) / kScatWarps;
  const int64_t j0 = min(cj1, cj0 + w * part), j1 = min(cj1, j0 + part);
  for (int b = threadIdx.x; b < kScatWarps * cells; b += kScatWarps * 32) s_g[b] = 0;
  __syncthreads();
  // (1) this warp's counts per block
  for (int64_t j = j0 + lane; j < j1; j += 32) {
    const BlockRect br = block_rect(drect[j], BW, BH);
    if (br.n == 0) continue;
    const int bx1 = br.bx0 + br.bw, by1 = br.by0 + br.n / br.bw;
    atomicAdd(&g[br.by0 * sw + br.bx0], 1);
    atomicAdd(&g[br.by0 * sw + bx1], -1);
    atomicAdd(&g[by1 * sw + br.bx0], -1);
    atomicAdd(&g[by1 * sw + bx1], 1);
  }
  __syncwarp();
  for (int y = lane; y < BH; y += 32) {
    int run = 0;
    for (int x = 0; x < BW; ++x) run = (g[y * sw + x] += run);
  }
  __syncwarp();
  for (int x = lane; x < BW; x += 32) {
    int run = 0;
    for (int y = 0; y < BH; ++y) run = (g[y * sw + x] += run);
  }
  __syncthreads();
  // (2) counts -> each warp's first position per block
  for (int b = threadIdx.x; b < nbk; b += kScatWarps * 32) {
    const int cell = (b / BW) * sw + b % BW;
    int32_t run = (int32_t)offs[c * nbk + b];
#pragma unroll
    for (int ww = 0; ww < kScatWarps; ++ww) {
      const int32_t v = s_g[ww * cells + cell];
      s_g[ww * cells + cell] = run;
      run += v;
    }
  }
  __syncthreads();
  // (3) emission
  const unsigned lt = (1u << lane) - 1u;
  bool bad = false;
  for (int64_t base = j0; base < j1; base += 32) {
    const int64_t j = base + lane;
    BlockRect br{0, 0, 1, 0};
    int32_t slot = 0;
    if (j < j1) {
      br = block_rect(drect[j], BW, BH);
      slot = order[j];
    }
    int incl = br.n;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    __syncwarp();
    s_ex[w][lane] = incl - br.n;
    s_bx[w][lane] = br.bx0;
    s_by[w][lane] = br.by0;
    s_bw[w][lane] = br.bw;
    s_rw[w][lane] = 1.0f / (float)br.bw;
    s_slot[w][lane] = slot;
    __syncwarp();
    for (int e0 = 0; e0 < total; e0 += 32) {
      const int e = e0 + lane;
      int cell = -1, sl = 0;
      if (e < total) {
        int lo = 0;  // the last candidate whose first entry is <= e
#pragma unroll
        for (int step = 16; step > 0; step >>= 1)
          if (s_ex[w][lo + step] <= e) lo += step;
        const int q = e - s_ex[w][lo], bw = s_bw[w][lo];
        const int row = (int)(((float)q + 0.5f) * s_rw[w][lo]);
        cell = (s_by[w][lo] + row) * sw + s_bx[w][lo] + (q - row * bw);
        sl = s_slot[w][lo];
      }
      const unsigned peers = __match_any_sync(0xffffffffu, cell);
      if (cell >= 0) {
        const int32_t cur = g[cell];
        const int64_t pos = (int64_t)cur + __popc(peers & lt);
        if (pos < capacity) block_vals[pos] = sl;
        else bad = true;
        __syncwarp(peers);
        if (lane == __ffs(peers) - 1) g[cell] = cur + __popc(peers);
      }
      __syncwarp();
    }
  }
  if (bad) dev_flag(dev_status, GS_DEV_BOUNDS);
}

size_t scat_smem(int64_t BW, int64_t BH) {
  return (size_t)kScatWarps * (BW + 1) * (BH + 1) * sizeof(int32_t);
}

struct BlockBinWs {
  unsigned int* ticket;
  unsigned long long* lb;
  uint32_t* keys;
  void* sort_ws;
  size_t sort_bytes;
  uint32_t* counts;   // counting scatter: [n_chunks][nblocks]
  uint32_t* segtot;   // [kScatSeg][nblocks]
  int64_t chunk, n_chunks;
  bool scatter;
  size_t bytes;
};

BlockBinWs carve_block_bin(void* ws, size_t cap, int64_t n_cand, int64_t n_entries, int64_t TWB,
                           int64_t THB) {
  const int64_t nblocks = TWB * THB;
  Carver cv(ws, cap);
  BlockBinWs w{};
  w.scatter = nblocks <= kScatMaxBlocks && scat_smem(TWB, THB) <= kScatMaxSmem;
  if (w.scatter) {
    w.chunk = scat_chunk(n_cand, nblocks);
    w.n_chunks = (n_cand + w.chunk - 1) / w.chunk;
    w.counts = cv.take<uint32_t>(w.n_chunks > 0 ? w.n_chunks * nblocks : 1);
    w.segtot = cv.take<uint32_t>(kScatSeg * nblocks);
    w.bytes = cv.off;
    return w;
  }
  w.ticket = cv.take<unsigned int>(64);
  const int64_t nb = (n_cand + kBinChunk - 1) / kBinChunk;
  w.lb = cv.take<unsigned long long>(nb > 0 ? nb : 1);
  w.keys = cv.take<uint32_t>(n_entries > 0 ? n_entries : 1);
  const int bits = nblocks > 1 ? 64 - __builtin_clzll((unsigned long long)(nblocks - 1)) : 0;
  w.sort_bytes = gs_sort_workspace_size(n_entries, 4, 0, bits);
  w.sort_ws = cv.take<unsigned char>(w.sort_bytes);
  w.bytes = cv.off;
  return w;
}

struct ExpandWs {
  int64_t* chunk_start;
  int32_t* cnt;
  int64_t* base;
  int64_t max_chunks;
  size_t bytes;
};

ExpandWs carve_expand(void* ws, size_t cap, gs_rect leaf, int64_t block_entries) {
  Carver cv(ws, cap);
  ExpandWs w;
  const LeafBlocks lb = leaf_blocks(leaf);
  const int64_t nbl = (int64_t)lb.bw * lb.bh;
  w.max_chunks = (block_entries + kExpChunk - 1) / kExpChunk + nbl;
  w.chunk_start = cv.take<int64_t>(nbl + 1);
  w.cnt = cv.take<int32_t>(w.max_chunks * 64);
  w.base = cv.take<int64_t>(w.max_chunks * 64);
  w.bytes = cv.off;
  return w;
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
  if (!proj || n_cand < GS_COUNT_ON_DEVICE || n_cand > proj->capacity) return GS_ERR_ARG;
  // the count on the device (proj->n_cand, at most the capacity): the call
  // can be issued before the host has read the projection's count
  const bool dev = n_cand == GS_COUNT_ON_DEVICE;
  const int64_t n = dev ? proj->capacity : n_cand;
  if (dev && !proj->n_cand) return GS_ERR_ARG;
  if (n == 0) return GS_OK;
  if (!depth_order || !depth_rect || !proj->depth_key || !proj->rect) return GS_ERR_ARG;
  if (!aligned(depth_rect, 8) || !aligned(ws, 256)) return GS_ERR_ARG;
  OrderWs w = carve_order(ws, ws_bytes, n);
  if (!ws || w.bytes > ws_bytes) return GS_ERR_CAPACITY;
  const int32_t* n_dev = dev ? proj->n_cand : nullptr;
  const gs_status st = sort32_iota_devcount(proj->depth_key, w.keys, depth_order, n, n_dev,
                                            w.sort_ws, w.sort_bytes, dev_status,
                                            to_stream(stream));
  if (st != GS_OK) return st;
  k_gather_rects<<<(unsigned)((n + 255) / 256), 256, 0, to_stream(stream)>>>(
      reinterpret_cast<const short4*>(proj->rect), depth_order, n,
      reinterpret_cast<short4*>(depth_rect), n_dev);
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
  k_bin<1><<<(unsigned)nb, kBinThreads, 0, s>>>(
      reinterpret_cast<const short4*>(depth_rect), depth_order, proj->depth_key, n_cand, leaf, TW,
      tile_keys, vals, keys64, capacity, w.lb, w.ticket, dev_status);
  GS_LAUNCH_CHECK();
  return GS_OK;
}

extern "C" size_t gs_bin_blocks_workspace_size(int64_t n_cand, int64_t n_entries, int32_t TW,
                                               int32_t TH) {
  if (n_cand < 0 || n_entries < 0 || TW <= 0 || TH <= 0) return 0;
  return carve_block_bin(nullptr, 0, n_cand, n_entries, (TW + kBlk - 1) / kBlk,
                         (TH + kBlk - 1) / kBlk).bytes;
}

extern "C" gs_status gs_bin_blocks(const gs_proj* proj, int64_t n_cand, const int32_t* depth_order,
                                   const int16_t* depth_rect, int32_t TW, int32_t TH,
                                   const int64_t* block_sat, int64_t n_entries,
                                   int32_t* block_vals, int64_t capacity, int64_t* block_ranges,
                                   int64_t* needed, void* ws, size_t ws_bytes,
                                   int32_t* dev_status, gs_stream stream) {
  if (!proj || n_cand < 0 || n_cand > proj->capacity || TW <= 0 || TH <= 0 || TW > 32767 ||
      TH > 32767 || !block_sat || !block_ranges || n_entries < 0)
    return GS_ERR_ARG;
  if (n_entries > capacity) {
    if (needed) *needed = n_entries;
    return GS_ERR_CAPACITY;
  }
  if (n_cand > 0 && (!depth_order || !depth_rect)) return GS_ERR_ARG;
  if (n_entries > 0 && !block_vals) return GS_ERR_ARG;
  const int32_t BW = (TW + kBlk - 1) / kBlk, BH = (TH + kBlk - 1) / kBlk;
  const int64_t nblocks = (int64_t)BW * BH;
  BlockBinWs w = carve_block_bin(ws, ws_bytes, n_cand, n_entries, BW, BH);
  if (!ws || w.bytes > ws_bytes) {
    if (needed) *needed = (int64_t)w.bytes;
    return GS_ERR_CAPACITY;
  }
  if (!aligned(ws, 256) || !aligned(depth_rect, 8)) return GS_ERR_ARG;
  cudaStream_t s = to_stream(stream);
  const gs_rect grid{0, 0, BW, BH};
  k_ranges<<<(unsigned)((nblocks + 255) / 256), 256, 0, s>>>(block_sat, grid, BW, block_ranges);
  GS_LAUNCH_CHECK();
  if (n_cand == 0 || n_entries == 0) return GS_OK;
  if (w.scatter) {
    const int nbk = (int)nblocks;
    const size_t smem_d = (size_t)(BW + 1) * (BH + 1) * sizeof(int32_t);
    k_blk_count<<<(unsigned)w.n_chunks, 256, smem_d, s>>>(
        reinterpret_cast<const short4*>(depth_rect), n_cand, w.chunk, BW, BH, w.counts);
    GS_LAUNCH_CHECK();
    const dim3 sg((unsigned)((nbk + 31) / 32), kScatSeg);
    k_blk_segsum<<<sg, 256, 0, s>>>(w.counts, w.n_chunks, nbk, w.segtot);
    GS_LAUNCH_CHECK();
    k_blk_offs<<<sg, 256, 0, s>>>(w.counts, w.n_chunks, nbk, w.segtot, block_ranges, dev_status);
    GS_LAUNCH_CHECK();
    const size_t smem_sc = scat_smem(BW, BH);  // <= kScatMaxSmem
    {
      static std::atomic<unsigned long long> done{0};
      GS_TRY(smem_attrs_once((const void*)k_blk_scatter, (int)kScatMaxSmem, &done));
    }
    k_blk_scatter<<<(unsigned)w.n_chunks, kScatWarps * 32, smem_sc, s>>>(
        reinterpret_cast<const short4*>(depth_rect), depth_order, n_cand, w.chunk, BW, BH,
        w.counts, block_vals, capacity, dev_status);
    GS_LAUNCH_CHECK();
    return GS_OK;
  }
  GS_TRY(cudaMemsetAsync(ws, 0, (size_t)((char*)w.keys - (char*)ws), s));
  const int64_t nb = (n_cand + kBinChunk - 1) / kBinChunk;
  k_bin<kBlk><<<(unsigned)nb, kBinThreads, 0, s>>>(
      reinterpret_cast<const short4*>(depth_rect), depth_order, nullptr, n_cand, grid, BW, w.keys,
      block_vals, nullptr, capacity, w.lb, w.ticket, dev_status);
  GS_LAUNCH_CHECK();
  return gs_sort_tiles(w.keys, block_vals, n_entries, block_ranges, nblocks, w.sort_ws,
                       w.sort_bytes, dev_status, stream);
}

extern "C" size_t gs_expand_workspace_size(gs_rect leaf, int64_t block_entries) {
  if (leaf.x0 < 0 || leaf.y0 < 0 || leaf.x1 <= leaf.x0 || leaf.y1 <= leaf.y0 || block_entries < 0)
    return 0;
  return carve_expand(nullptr, 0, leaf, block_entries).bytes;
}

extern "C" gs_status gs_expand_tiles(const gs_proj* proj, const int32_t* block_vals,
                                     const int64_t* block_ranges, int64_t block_entries,
                                     gs_rect leaf, int32_t TW, int32_t TH,
                                     const int64_t* tile_sat, int64_t n_isect, int32_t* vals,
                                     int64_t capacity, int64_t* ranges, int64_t* needed, void* ws,
                                     size_t ws_bytes, int32_t* dev_status, gs_stream stream) {
  if (!proj || TW <= 0 || TH <= 0 || TW > 32767 || TH > 32767 || !tile_sat || !ranges ||
      !block_ranges || block_entries < 0 || n_isect < 0)
    return GS_ERR_ARG;
  if (leaf.x0 < 0 || leaf.y0 < 0 || leaf.x1 <= leaf.x0 || leaf.y1 <= leaf.y0 || leaf.x1 > TW ||
      leaf.y1 > TH)
    return GS_ERR_ARG;
  if (n_isect > capacity) {
    if (needed) *needed = n_isect;
    return GS_ERR_CAPACITY;
  }
  if (capacity > (int64_t)INT32_MAX) return GS_ERR_UNSUPPORTED;  // 32-bit list positions
  if (n_isect > 0 && (!vals || !block_vals || !proj->rect)) return GS_ERR_ARG;
  ExpandWs w = carve_expand(ws, ws_bytes, leaf, block_entries);
  if (!ws || w.bytes > ws_bytes) {
    if (needed) *needed = (int64_t)w.bytes;
    return GS_ERR_CAPACITY;
  }
  if (!aligned(ws, 256) || !aligned(proj->rect, 8)) return GS_ERR_ARG;
  cudaStream_t s = to_stream(stream);
  const int64_t ntiles = (int64_t)(leaf.x1 - leaf.x0) * (leaf.y1 - leaf.y0);
  k_ranges<<<(unsigned)((ntiles + 255) / 256), 256, 0, s>>>(tile_sat, leaf, TW, ranges);
  GS_LAUNCH_CHECK();
  if (n_isect == 0 || block_entries == 0) return GS_OK;
  const int32_t BW = (TW + kBlk - 1) / kBlk;
  const LeafBlocks lb = leaf_blocks(leaf);
  const int64_t nbl = (int64_t)lb.bw * lb.bh;
  const short4* r4 = reinterpret_cast<const short4*>(proj->rect);
  k_expand_plan<<<1, 1024, 0, s>>>(block_ranges, BW, lb, w.chunk_start, w.max_chunks, dev_status);
  GS_LAUNCH_CHECK();
  k_expand_count<<<(unsigned)w.max_chunks, kExpThreads, 0, s>>>(r4, block_vals, block_ranges, BW,
                                                                lb, leaf, w.chunk_start, w.cnt);
  GS_LAUNCH_CHECK();
  k_expand_scan<<<(unsigned)((nbl * 64 + 255) / 256), 256, 0, s>>>(
      w.cnt, w.chunk_start, lb, leaf, ranges, w.base, w.max_chunks, dev_status);
  GS_LAUNCH_CHECK();
  k_expand_write<<<(unsigned)w.max_chunks, kExpThreads, 0, s>>>(
      r4, block_vals, block_ranges, BW, lb, leaf, w.chunk_start, w.base, vals, (int32_t)capacity,
      dev_status);
  GS_LAUNCH_CHECK();
  return GS_OK;
}

extern "C" gs_status gs_tile_ranges(const int64_t* tile_sat, int32_t TW, int32_t TH, gs_rect leaf,
                                    int64_t* ranges, gs_stream stream) {
  if (!tile_sat || !ranges || TW <= 0 || TH <= 0) return GS_ERR_ARG;
  if (leaf.x0 < 0 || leaf.y0 < 0 || leaf.x1 <= leaf.x0 || leaf.y1 <= leaf.y0 || leaf.x1 > TW ||
      leaf.y1 > TH)
    return GS_ERR_ARG;
  const int64_t ntiles = (int64_t)(leaf.x1 - leaf.x0) * (leaf.y1 - leaf.y0);
  k_ranges<<<(unsigned)((ntiles + 255) / 256), 256, 0, to_stream(stream)>>>(tile_sat, leaf, TW,
                                                                             ranges);
  GS_LAUNCH_CHECK();
  return GS_OK;
}
