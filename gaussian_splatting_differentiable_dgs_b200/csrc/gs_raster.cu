// Tile rasteriser: front-to-back compositing (+ fused L1 loss) and the
// reverse blend with per-tile reduction of the per-Gaussian gradients.
//
// SkipGS paper notes, "loss function / training strategy": the image is the
// transmittance-weighted blend of the sorted Gaussians and the gradients
// flow back through the transmittance accumulation; "key design 2": the
// backward accumulates per-Gaussian gradients atomically.  BoundedGS project
// page, section 01: a Leaf's gradient contribution is merged into the view's
// gradient before its buffers are released (here: atomics into the compact
// per-candidate g2d that lives for the whole view).
//
// One CTA per 16x16 tile of the Leaf; each thread owns PPT pixels of one
// column.  The tile's list is staged through shared memory in batches of
// one record per thread; within a batch every thread reads each record by
// broadcast.  fp32 arithmetic with explicitly rounded operations in the
// alpha path, so the backward retakes exactly the forward's skip decisions.
#include <cuda_fp16.h>

#include <algorithm>
#include <type_traits>

#include "gs_internal.cuh"

namespace gs {
namespace {

// the forward's walk over a warp's list, two entries per iteration: the
// second entry's alpha chain (independent of T) overlaps the first's
// update (1.55 -> 1.53 ms per step on the 6M view; 4 gained nothing more,
// and the backward, with its per-entry reduction, lost time at 2)
#ifndef GS_FWD_UNROLL
#define GS_FWD_UNROLL 2
#endif
constexpr int kFwdUnroll = GS_FWD_UNROLL;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kAlphaMin = 1.0f / 255.0f;
constexpr float kAlphaMax = 0.99f;
constexpr float kTMin = 1e-4f;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Staged record: position relative to the tile origin, the exponent
// coefficients pre-scaled by -log2(e) and the opacity as its log2, which
// joins the exponent (o 2^x = 2^(x + log2 o)).
struct Staged {
  float gx, gy, beta, ns1;   // float4
  float ns2, lo2, r, g;      // float4
  float opac;
  float b, s1, s2;           // natural-log coefficients (backward)
  float hx, hy;              // alpha box half extents
  int32_t slot;
};

__device__ __forceinline__ Staged stage_record(const float4* __restrict__ rec, int32_t slot,
                                               int tx, int ty) {
  const float4 r0 = rec[3 * (int64_t)slot];
  const float4 r1 = rec[3 * (int64_t)slot + 1];
  const float4 r2 = rec[3 * (int64_t)slot + 2];
  Staged s;
  const unsigned lo_bits = __float_as_uint(r0.z), box_bits = __float_as_uint(r0.w);
  const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&lo_bits));
  const float2 box = __half22float2(*reinterpret_cast<const __half2*>(&box_bits));
  s.gx = __fadd_rn(__fsub_rn(r0.x, (float)(tx * kTile)), lo.x);
  s.gy = __fadd_rn(__fsub_rn(r0.y, (float)(ty * kTile)), lo.y);
  s.hx = box.x;
  s.hy = box.y;
  s.beta = r1.y;
  s.ns1 = __fmul_rn(r1.x, -kLog2e);
  s.ns2 = __fmul_rn(r1.z, -kLog2e);
  s.opac = r1.w;
  s.lo2 = log2f(r1.w);
  s.r = r2.x;
  s.g = r2.y;
  s.b = r2.z;
  s.s1 = r1.x;
  s.s2 = r1.z;
  s.slot = slot;
  return s;
}

// A staged record as the forward's pixel pairs read it: every field twice,
// so that one packed fp32x2 operation applies it to both pixels; the
// colours negated (they multiply the negated weight).
struct __align__(16) Packed {
  float2 gy, beta;
  float2 ns1, ns2;
  float2 lo2, nr;
  float2 ng, nb;
  float2 gx;
};

__device__ __forceinline__ Packed pack_record(const Staged& st) {
  Packed q;
  q.gx = make_float2(st.gx, st.gx);
  q.gy = make_float2(st.gy, st.gy);
  q.beta = make_float2(st.beta, st.beta);
  q.ns1 = make_float2(st.ns1, st.ns1);
  q.ns2 = make_float2(st.ns2, st.ns2);
  q.lo2 = make_float2(st.lo2, st.lo2);
  q.nr = make_float2(-st.r, -st.r);
  q.ng = make_float2(-st.g, -st.g);
  q.nb = make_float2(-st.b, -st.b);
  return q;
}

// The backward's form: colours as they are.
struct __align__(16) PackedB {
  float2 gy, beta;
  float2 ns1, ns2;
  float2 lo2, r;
  float2 g, b;
  float2 gx;
};

__device__ __forceinline__ PackedB pack_record_bwd(const Staged& st) {
  PackedB q;
  q.gx = make_float2(st.gx, st.gx);
  q.gy = make_float2(st.gy, st.gy);
  q.beta = make_float2(st.beta, st.beta);
  q.ns1 = make_float2(st.ns1, st.ns1);
  q.ns2 = make_float2(st.ns2, st.ns2);
  q.lo2 = make_float2(st.lo2, st.lo2);
  q.r = make_float2(st.r, st.r);
  q.g = make_float2(st.g, st.g);
  q.b = make_float2(st.b, st.b);
  return q;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


struct PixArgs {
  int32_t x0, y0, w, h;
  int64_t pitch, plane;
  float* img;
  float* T_final;
  int32_t* last;
  float* dL;
  const float* target;
  int32_t tx0, ty0;
  int64_t tpitch, tplane;
  float* loss_tiles;
  float norm;
  unsigned long long* counters;
};

// Pixel layout: each warp owns a compact BW x BH block of the tile (8x4,
// 8x8 or 16x8 pixels for PPT = 1, 2, 4); lane l of warp w holds pixels
// (bx0 + l % BW, by0 + l / BW + k * LROWS), k < PPT.
template <int PPT>
struct TileGeom {
  static constexpr int NT = 256 / PPT;
  static constexpr int NW = NT / 32;
  static constexpr int BW = PPT == 4 ? 16 : 8;
  static constexpr int BH = 32 * PPT / BW;
  static constexpr int LROWS = 32 / BW;
  static constexpr int BX = 16 / BW;
};

struct WarpPix {
  int lx, ly0;  // first pixel of the lane (tile-relative)
};

template <int PPT>
__device__ __forceinline__ WarpPix warp_pixels(int t) {
  using G = TileGeom<PPT>;
  const int w = t >> 5, l = t & 31;
  const int bx0 = (w % G::BX) * G::BW, by0 = (w / G::BX) * G::BH;
  WarpPix p;
  p.lx = bx0 + l % G::BW;
  p.ly0 = by0 + l / G::BW;
  return p;
}

// Tile-relative bounding box of the region where alpha >= 1/255 can hold
// (o exp(-q) >= 1/255 <=> q <= ln(255 o)), from the half extents the
// projection stores (inflated far beyond the fp32 error of the per-pixel
// alpha and rounded up): a warp whose pixel box misses it would have
// skipped the Gaussian at every pixel anyway, so culling by it leaves every
// result bit-identical.  The staging thread turns the box into one bit per
// warp; each warp then walks only its own compacted list of records.
__device__ __forceinline__ float4 alpha_box(const Staged& st) {
  return make_float4(st.gx - st.hx, st.gx + st.hx, st.gy - st.hy, st.gy + st.hy);
}

// q(e) = s1 (ex + beta ey)^2 + s2 ey^2 at an offset e from the mean.
__device__ __forceinline__ float q_at(float ex, float ey, float s1, float beta, float s2) {
  const float t = fmaf(beta, ey, ex);
  return fmaf(s1 * t, t, s2 * ey * ey);
}

// Bit w set if the record can reach alpha >= 1/255 at a pixel centre of warp
// w: its alpha box meets the warp's pixel-centre rectangle, and the smallest
// q over that rectangle stays below ln(255 o) plus a margin (1e-3 + 1e-4
// |ln(255 o)|, about a thousand times the fp32 error of the per-pixel q).
// q is convex, so its minimum over the rectangle is 0 when the mean lies
// inside, else on an edge, where it has a closed form.  A cleared bit means
// every pixel of the warp would skip the record, so culling by it changes
// no result.
template <int PPT>
__device__ __forceinline__ unsigned warp_mask(const Staged& st) {
  using G = TileGeom<PPT>;
  const float4 b = alpha_box(st);
  const float lq = __logf(255.0f * st.opac);
  const float qthr = lq + 1e-3f + 1e-4f * fabsf(lq);
  const float s1 = st.s1, beta = st.beta, s2 = st.s2;
  // on an edge ex = const, the best ey is k ex
  const float k = -s1 * beta / fmaf(s1 * beta, beta, s2);
  unsigned m = 0;
#pragma unroll
  for (int w = 0; w < G::NW; ++w) {
    const float x0 = (float)((w % G::BX) * G::BW) + 0.5f, x1 = x0 + (float)(G::BW - 1);
    const float y0 = (float)((w / G::BX) * G::BH) + 0.5f, y1 = y0 + (float)(G::BH - 1);
    const bool miss = (b.x > x1) | (b.y < x0) | (b.z > y1) | (b.w < y0);
    // the rectangle relative to the mean (pixel - mean; q is even)
    const float ex0 = x0 - st.gx, ex1 = x1 - st.gx, ey0 = y0 - st.gy, ey1 = y1 - st.gy;
    const bool inside = (ex0 <= 0.f) & (ex1 >= 0.f) & (ey0 <= 0.f) & (ey1 >= 0.f);
    float qmin = 0.f;
    if (!inside) {
      const float qa = q_at(ex0, fminf(fmaxf(k * ex0, ey0), ey1), s1, beta, s2);
      const float qb = q_at(ex1, fminf(fmaxf(k * ex1, ey0), ey1), s1, beta, s2);
      const float qc = q_at(fminf(fmaxf(-beta * ey0, ex0), ex1), ey0, s1, beta, s2);
      const float qd = q_at(fminf(fmaxf(-beta * ey1, ex0), ex1), ey1, s1, beta, s2);
      qmin = fminf(fminf(qa, qb), fminf(qc, qd));
    }
    m |= (miss || qmin > qthr) ? 0u : (1u << w);
  }
  return m;
}

// One staged entry composited into a lane's pixel pairs, front to back.
// alpha = min(0.99, o e^-q) = min(0.99, 2^(log2 o - q log2 e)) with
// q = s1 (dx + beta dy)^2 + s2 dy^2, dx = gx - px, dy = gy - py, each step
// one rounded operation: dx and dy, t = fma(beta, dy, dx), and the exponent
// fma(ns1 t, t, fma(ns2 dy, dy, log2 o)) with ns = -s log2 e.
// Branch-free: every pixel evaluates.  A pixel that is done, skips the
// entry or stops at it composites with a zero alpha, which leaves T and the
// colour sums exactly as they were.  A packed fp32x2 operation rounds each
// of its two pixels as the scalar operation would; T (1 - alpha) is one
// fma, and the negated alpha and colours make every product exact to negate.
template <int NP, bool COUNT>
__device__ __forceinline__ void composite_entry(const Packed& R, int posn, float2 nfpx2,
                                                const float2 (&npy2)[NP], float2 (&T2)[NP],
                                                float2 (&Cr2)[NP], float2 (&Cg2)[NP],
                                                float2 (&Cb2)[NP], bool (&done)[2 * NP],
                                                int (&lastp)[2 * NP], int (&stopn)[2 * NP],
                                                unsigned& n_vis, unsigned& n_kept) {
  const float2 dx2 = __fadd2_rn(R.gx, nfpx2);  // gx - px
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const float2 dy = __fadd2_rn(R.gy, npy2[p]);
    const float2 t1 = __ffma2_rn(R.beta, dy, dx2);
    const float2 qa = __fmul2_rn(R.ns1, t1);
    const float2 qb = __ffma2_rn(__fmul2_rn(R.ns2, dy), dy, R.lo2);
    const float2 e = __ffma2_rn(qa, t1, qb);
    float na[2] = {fmaxf(-ex2_approx(e.x), -kAlphaMax), fmaxf(-ex2_approx(e.y), -kAlphaMax)};
    const float2 Tn = __ffma2_rn(make_float2(na[0], na[1]), T2[p], T2[p]);
    const float tn[2] = {Tn.x, Tn.y};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int k = 2 * p + h;
      if (COUNT) n_vis += done[k] ? 0u : 1u;
      const bool use = !done[k] && na[h] <= -kAlphaMin;
      const bool stop = use && tn[h] < kTMin;
      const bool comp = use && !stop;
      if (COUNT) {
        stopn[k] = stop ? posn : stopn[k];
        n_kept += comp ? 1u : 0u;
      }
      done[k] = done[k] || stop;
      na[h] = comp ? na[h] : 0.0f;
      lastp[k] = comp ? posn : lastp[k];
    }
    const float2 na2 = make_float2(na[0], na[1]);
    const float2 nw = __fmul2_rn(na2, T2[p]);  // -alpha T
    T2[p] = __ffma2_rn(na2, T2[p], T2[p]);
    Cr2[p] = __ffma2_rn(R.nr, nw, Cr2[p]);
    Cg2[p] = __ffma2_rn(R.ng, nw, Cg2[p]);
    Cb2[p] = __ffma2_rn(R.nb, nw, Cb2[p]);
  }
}

// The batch positions j in [j0, cnt) whose record meets warp w's pixels, in
// ascending order, into list[0..n); returns n (warp-uniform).
template <class LT>
__device__ __forceinline__ int warp_list(const uint8_t* __restrict__ s_mask, int j0, int cnt, int w,
                                         int lane, LT* __restrict__ list) {
  int n = 0;
  const unsigned lt = (1u << lane) - 1u;
  for (int c = j0; c < cnt; c += 32) {
    const int j = c + lane;
    const bool m = j < cnt && ((s_mask[j] >> w) & 1u);
    const unsigned b = __ballot_sync(0xffffffffu, m);
    if (m) list[n + __popc(b & lt)] = (LT)j;
    n += __popc(b);
  }
  __syncwarp();
  return n;
}

// Source of a tile's list for the forward when it is built on the fly: the
// depth-ordered candidate list of the tile's block of GS_TILE_BLOCK^2 tiles,
// filtered by "tile inside the candidate's rect" (which keeps the order, so
// the result is the tile's list), written to vals_out as it is consumed.
struct BlockSrc {
  const short4* rect;
  const int32_t* block_vals;
  const int64_t* block_ranges;
  int BW;
  int32_t* vals_out;
  int64_t* ranges_io;  // in: the tile's segment [begin, end); out: end = begin + written
};

// ---------------------------------------------------------------------------
// forward
// ---------------------------------------------------------------------------
// BLK = false: the tile's list is vals[ranges]; BLK = true: it is built
// from the block list (BlockSrc) and only as far as the tile's pixels need
// it.  A fill reads kFillU x NT block-list entries at once (kFillU loads in
// flight per thread), keeps the hits in list order in s_hits and in the
// Leaf's vals; the hits are then staged and composited NT at a time.
constexpr int kFillU = 2;

template <int PPT, bool COUNT, bool BLK>
__global__ void __launch_bounds__(256 / PPT, PPT == 2 ? 8 : 1)
k_raster_fwd(const float4* __restrict__ rec, const int32_t* __restrict__ vals,
             const int64_t* ranges, gs_rect leaf, int W, int H, int TW, PixArgs px,
             BlockSrc bsrc, int32_t* dev_status) {
  using G = TileGeom<PPT>;
  constexpr int NT = G::NT;
  constexpr int CAP = NT;
  using LT = std::conditional_t<(CAP <= 256), uint8_t, uint16_t>;
  constexpr int HCAP = BLK ? kFillU * NT : 1;
  __shared__ Packed sPk[CAP];
  __shared__ uint8_t s_mask[CAP];
  __shared__ LT s_list[G::NW][CAP];
  __shared__ float s_red[G::NW];
  __shared__ int s_wcnt[kFillU][G::NW];
  __shared__ int32_t s_hits[HCAP];
  const int lw = leaf.x1 - leaf.x0;
  const int ltile = blockIdx.x;
  const int tx = leaf.x0 + ltile % lw, ty = leaf.y0 + ltile / lw;
  const int64_t begin = ranges[2 * ltile], end = ranges[2 * ltile + 1];
  // block-list cursor / end, list entries written, staged; hit-list cursor / length
  int64_t bp = 0, be = 0, n_filled = 0, n_staged = 0;
  int hp = 0, nh = 0;
  if (BLK) {
    const int64_t b = (int64_t)(ty / GS_TILE_BLOCK) * bsrc.BW + tx / GS_TILE_BLOCK;
    bp = bsrc.block_ranges[2 * b];
    be = bsrc.block_ranges[2 * b + 1];
  }
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const WarpPix wp = warp_pixels<PPT>(t);
  // the lane's pixels in pairs (NP of them; with an odd PPT the last pair's
  // second pixel is a placeholder that starts done): the per-pixel state of
  // a pair lives in float2s that packed fp32x2 operations update together
  constexpr int NP = (PPT + 1) / 2;
  const float fpx = (float)wp.lx + 0.5f;
  const float2 nfpx2 = make_float2(-fpx, -fpx);
  float2 npy2[NP], T2[NP], Cr2[NP], Cg2[NP], Cb2[NP];
  int lastp[2 * NP];
  int stopn[2 * NP];  // COUNT: 1-based list position of the stopping entry, 0 = none
  bool done[2 * NP], inside[2 * NP];
  unsigned n_vis = 0, n_kept = 0;
#pragma unroll
  for (int k = 0; k < 2 * NP; ++k) {
    const int ly = wp.ly0 + k * G::LROWS;
    const float npy = -((float)ly + 0.5f);
    if (k & 1) npy2[k >> 1].y = npy; else npy2[k >> 1].x = npy;
    inside[k] = k < PPT && (tx * kTile + wp.lx < W) && (ty * kTile + ly < H);
    done[k] = !inside[k];
    lastp[k] = 0;
    stopn[k] = 0;
  }
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    T2[p] = make_float2(1.0f, 1.0f);
    Cr2[p] = Cg2[p] = Cb2[p] = make_float2(0.0f, 0.0f);
  }
  bool bad = false;
  for (int64_t base = begin;; base += NT) {
    if (!BLK && base >= end) break;
    bool mine_done = true;
#pragma unroll
    for (int k = 0; k < 2 * NP; ++k) mine_done = mine_done && done[k];
    if (__syncthreads_count(mine_done) == NT) break;
    int cnt, pos1;
    if (BLK) {
      if (hp >= nh) {
        // fill: kFillU x NT block-list entries, hits kept in list order
        if (bp >= be) break;
        int32_t sl[kFillU];
        short4 rc[kFillU];
#pragma unroll
        for (int u = 0; u < kFillU; ++u) {
          const int64_t q = bp + (int64_t)u * NT + t;
          sl[u] = q < be ? bsrc.block_vals[q] : -1;
        }
#pragma unroll
        for (int u = 0; u < kFillU; ++u)
          if (sl[u] >= 0) rc[u] = bsrc.rect[sl[u]];
        const unsigned ltm = (1u << lane) - 1u;
        unsigned bal[kFillU];
#pragma unroll
        for (int u = 0; u < kFillU; ++u) {
          const bool hit = sl[u] >= 0 && (rc[u].x <= tx) & (tx < rc[u].z) & (rc[u].y <= ty) &
                                             (ty < rc[u].w);
          bal[u] = __ballot_sync(0xffffffffu, hit);
          if (lane == 0) s_wcnt[u][w] = __popc(bal[u]);
        }
        __syncthreads();
        int run = 0, off[kFillU];
#pragma unroll
        for (int u = 0; u < kFillU; ++u)
#pragma unroll
          for (int ww = 0; ww < G::NW; ++ww) {
            if (ww == w) off[u] = run;
            run += s_wcnt[u][ww];
          }
#pragma unroll
        for (int u = 0; u < kFillU; ++u)
          if ((bal[u] >> lane) & 1u) {
            const int k = off[u] + __popc(bal[u] & ltm);
            s_hits[k] = sl[u];
            const int64_t o = begin + n_filled + k;
            if (o < end) bsrc.vals_out[o] = sl[u];
            else bad = true;
          }
        nh = run;
        hp = 0;
        n_filled += run;
        bp += (int64_t)kFillU * NT;
        __syncthreads();  // s_hits visible; s_wcnt free again
        if (nh == 0) continue;
      }
      cnt = min(NT, nh - hp);
      if (t < cnt) {
        const Staged st = stage_record(rec, s_hits[hp + t], tx, ty);
        s_mask[t] = (uint8_t)warp_mask<PPT>(st);
        sPk[t] = pack_record(st);
      }
      __syncthreads();
      pos1 = (int)n_staged + 1;
      n_staged += cnt;
      hp += cnt;
    } else {
      const int64_t e = base + t;
      if (e < end) {
        const Staged st = stage_record(rec, vals[e], tx, ty);
        s_mask[t] = (uint8_t)warp_mask<PPT>(st);
        sPk[t] = pack_record(st);
      }
      __syncthreads();
      cnt = (int)min((int64_t)NT, end - base);
      pos1 = (int)(base - begin) + 1;
    }
    if (__all_sync(0xffffffffu, mine_done)) continue;  // nothing left for this warp
    const int nl = warp_list<LT>(s_mask, 0, cnt, w, lane, s_list[w]);
    for (int i0 = 0; i0 < nl; i0 += 32) {
      if (i0 > 0) {
        bool d_all = true;
#pragma unroll
        for (int k = 0; k < 2 * NP; ++k) d_all = d_all && done[k];
        if (__all_sync(0xffffffffu, d_all)) break;
      }
      const int i1 = min(nl, i0 + 32);
#pragma unroll kFwdUnroll
      for (int i = i0; i < i1; ++i) {
        const int j = s_list[w][i];
        const Packed R = sPk[j];
        const int posn = pos1 + j;
        composite_entry<NP, COUNT>(R, posn, nfpx2, npy2, T2, Cr2, Cg2, Cb2, done, lastp, stopn,
                                   n_vis, n_kept);
      }
    }
  }
  if (COUNT) {  // one atomic per warp: per-thread ones on one word serialise
    // the method's evaluations: each pixel visits its tile's list up to its
    // stop (or the whole list), and the backward revisits it up to last
    unsigned long long e_f = 0, e_b = 0;
#pragma unroll
    for (int k = 0; k < PPT; ++k)
      if (inside[k]) {
        e_f += stopn[k] ? (unsigned long long)stopn[k] : (unsigned long long)(end - begin);
        e_b += (unsigned long long)lastp[k];
      }
    const unsigned long long a = warp_sum((unsigned long long)n_vis);
    const unsigned long long b = warp_sum((unsigned long long)n_kept);
    const unsigned long long c = warp_sum(e_f);
    const unsigned long long d = warp_sum(e_b);
    if ((t & 31) == 0) {
      atomicAdd(&px.counters[0], a);
      atomicAdd(&px.counters[1], b);
      atomicAdd(&px.counters[2], c);
      atomicAdd(&px.counters[3], d);
    }
  }
  if (BLK) {
    if (bad) dev_flag(dev_status, GS_DEV_BOUNDS);
    if (t == 0)
      bsrc.ranges_io[2 * ltile + 1] = begin + (n_filled < end - begin ? n_filled : end - begin);
  }
  // epilogue: outputs and the fused L1 terms
  float lsum = 0.0f;
#pragma unroll
  for (int k = 0; k < PPT; ++k) {
    if (!inside[k]) continue;
    const int x = tx * kTile + wp.lx, y = ty * kTile + wp.ly0 + k * G::LROWS;
    const int64_t o = (int64_t)(y - px.y0) * px.pitch + (x - px.x0);
    const float2 T_ = T2[k >> 1], r_ = Cr2[k >> 1], g_ = Cg2[k >> 1], b_ = Cb2[k >> 1];
    const float c[3] = {(k & 1) ? r_.y : r_.x, (k & 1) ? g_.y : g_.x, (k & 1) ? b_.y : b_.x};
    if (px.img) {
      px.img[o] = c[0];
      px.img[o + px.plane] = c[1];
      px.img[o + 2 * px.plane] = c[2];
    }
    px.T_final[o] = (k & 1) ? T_.y : T_.x;
    px.last[o] = lastp[k];
    if (px.target) {
      const int64_t ot = (int64_t)(y - px.ty0) * px.tpitch + (x - px.tx0);
#pragma unroll
      for (int ch = 0; ch < 3; ++ch) {
        const float d = c[ch] - px.target[ot + ch * px.tplane];
        px.dL[o + ch * px.plane] = d > 0.0f ? px.norm : (d < 0.0f ? -px.norm : 0.0f);
        lsum += fabsf(d);
      }
    }
  }
  if (px.target && px.loss_tiles) {
    lsum = warp_sum(lsum);
    if ((t & 31) == 0) s_red[t >> 5] = lsum;
    __syncthreads();
    if (t == 0) {
      float tot = 0.0f;
      for (int w = 0; w < G::NW; ++w) tot += s_red[w];
      px.loss_tiles[(int64_t)ty * TW + tx] = tot * px.norm;
    }
  }
}

// ---------------------------------------------------------------------------
// forward, warp-specialised (the block-list path): one producer warp builds
// the tile's list from its block list and stages the records; the NC
// consumer warps composite them.  No CTA barrier separates the two roles:
//
// - producer: reads kWsU x 32 block-list entries per fill (kWsU loads in
//   flight per lane), keeps the hits ("tile inside the candidate's rect"),
//   in list order, in a circular queue s_q and in the Leaf's vals, and
//   stages up to 32 queued records at a time into stage k % kWsS of a ring
//   (the record's fields, its per-warp mask, the count and the list position
//   of its first record), completing the stage's "full" mbarrier;
// - consumers: each waits for stage k, walks the records whose mask bit is
//   set for it, and arrives on the stage's "empty" mbarrier.  A warp whose
//   pixels are all done counts itself in s_ndone once and from then on only
//   releases stages; the producer stops filling once every consumer warp is
//   done or the block list is exhausted and then publishes a terminal stage
//   (count -1).
//
// Every wait is bounded: on expiry the waiter sets s_abort and
// GS_DEV_TIMEOUT, and both roles leave.  The list prefix the producer
// writes covers every position a consumer composited (positions < last).
// ---------------------------------------------------------------------------
constexpr int kWsS = 8;      // ring stages of 32 records
constexpr int kWsQ = 512;    // hit queue (circular)
constexpr int kWsU = 8;      // block-list entries per producer lane per fill

// A shared flag read once for the whole warp (lane 0's value), so that the
// warp takes the same branch.
__device__ __forceinline__ int warp_flag(const int* f) {
  return __shfl_sync(0xffffffffu, *(const volatile int*)f, 0);
}

// mbar_wait by every lane, true only if every lane saw the phase complete.
__device__ __forceinline__ bool warp_mbar_wait(unsigned long long* bar, unsigned parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

template <int PPT, bool COUNT>
__global__ void __launch_bounds__(TileGeom<PPT>::NT + 32, PPT == 2 ? 6 : 8)
k_raster_fwd_ws(const float4* __restrict__ rec, gs_rect leaf, int W, int H, int TW, PixArgs px,
                BlockSrc bsrc, int32_t* dev_status) {
  using G = TileGeom<PPT>;
  constexpr int NC = G::NW;
  __shared__ Packed sPk[kWsS][32];
  __shared__ uint8_t sM[kWsS][32];
  __shared__ int sCnt[kWsS], sPos[kWsS];
  __shared__ unsigned long long s_full[kWsS], s_empty[kWsS];
  __shared__ int32_t s_q[kWsQ];
  __shared__ int s_ndone, s_abort;
  __shared__ float s_red[NC];
  const int lw = leaf.x1 - leaf.x0;
  const int ltile = blockIdx.x;
  const int tx = leaf.x0 + ltile % lw, ty = leaf.y0 + ltile / lw;
  const int64_t begin = bsrc.ranges_io[2 * ltile], end = bsrc.ranges_io[2 * ltile + 1];
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  if (t == 0) {
    for (int st = 0; st < kWsS; ++st) {
      mbar_init(&s_full[st], 32);
      mbar_init(&s_empty[st], NC);
    }
    s_ndone = 0;
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (w == NC) {  // ---- producer warp ----
    const int64_t b = (int64_t)(ty / GS_TILE_BLOCK) * bsrc.BW + tx / GS_TILE_BLOCK;
    int64_t bp = bsrc.block_ranges[2 * b];
    const int64_t be = bsrc.block_ranges[2 * b + 1];
    const unsigned ltm = (1u << lane) - 1u;
    unsigned qh = 0, qt = 0;  // staged / queued hits (list positions)
    bool exhausted = bp >= be, bad = false, ok = true;
    int k = 0;
    for (;;) {
      // every consumer warp done: stop (the hits queued so far are in vals)
      if (warp_flag(&s_ndone) == NC) break;
      while (!exhausted && qt - qh < 32u) {
        int32_t sl[kWsU];
        short4 rc[kWsU];
#pragma unroll
        for (int u = 0; u < kWsU; ++u) {
          const int64_t q = bp + u * 32 + lane;
          sl[u] = q < be ? bsrc.block_vals[q] : -1;
        }
#pragma unroll
        for (int u = 0; u < kWsU; ++u)
          rc[u] = sl[u] >= 0 ? bsrc.rect[sl[u]] : make_short4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < kWsU; ++u) {
          const bool hit = sl[u] >= 0 && (rc[u].x <= tx) & (tx < rc[u].z) & (rc[u].y <= ty) &
                                             (ty < rc[u].w);
          const unsigned bal = __ballot_sync(0xffffffffu, hit);
          if (hit) {
            const unsigned pos = qt + __popc(bal & ltm);
            s_q[pos & (kWsQ - 1)] = sl[u];
            const int64_t o = begin + pos;
            if (o < end) bsrc.vals_out[o] = sl[u];
            else bad = true;
          }
          qt += __popc(bal);
        }
        bp += kWsU * 32;
        exhausted = bp >= be;
      }
      const int m = (int)min(32u, qt - qh);
      if (m == 0) break;
      const int st = k % kWsS;
      if (k >= kWsS && !warp_mbar_wait(&s_empty[st], (unsigned)((k / kWsS - 1) & 1))) {
        ok = false;
        break;
      }
      __syncwarp();  // the queue entries written by other lanes are visible
      if (lane < m) {
        const Staged g = stage_record(rec, s_q[(qh + lane) & (kWsQ - 1)], tx, ty);
        sM[st][lane] = (uint8_t)warp_mask<PPT>(g);
        sPk[st][lane] = pack_record(g);
      }
      if (lane == 0) {
        sCnt[st] = m;
        sPos[st] = (int)qh;
      }
      qh += m;
      mbar_arrive(&s_full[st]);
      ++k;
      if (warp_flag(&s_abort)) {
        ok = false;
        break;
      }
    }
    if (ok) {  // terminal stage
      const int st = k % kWsS;
      if (k >= kWsS && !warp_mbar_wait(&s_empty[st], (unsigned)((k / kWsS - 1) & 1))) ok = false;
      if (ok) {
        if (lane == 0) sCnt[st] = -1;
        mbar_arrive(&s_full[st]);
      }
    }
    if (!ok) {
      *(volatile int*)&s_abort = 1;
      if (lane == 0) dev_flag(dev_status, GS_DEV_TIMEOUT);
    }
    if (bad) dev_flag(dev_status, GS_DEV_BOUNDS);
    if (lane == 0)
      bsrc.ranges_io[2 * ltile + 1] = begin + ((int64_t)qt < end - begin ? (int64_t)qt : end - begin);
    return;
  }

  // ---- consumer warps ----
  const WarpPix wp = warp_pixels<PPT>(t);
  // the lane's pixels in pairs (NP of them; with an odd PPT the last pair's
  // second pixel is a placeholder that starts done): the per-pixel state of
  // a pair lives in float2s that packed fp32x2 operations update together
  constexpr int NP = (PPT + 1) / 2;
  const float fpx = (float)wp.lx + 0.5f;
  const float2 nfpx2 = make_float2(-fpx, -fpx);
  float2 npy2[NP], T2[NP], Cr2[NP], Cg2[NP], Cb2[NP];
  int lastp[2 * NP];
  int stopn[2 * NP];  // COUNT: 1-based list position of the stopping entry, 0 = none
  bool done[2 * NP], inside[2 * NP];
  unsigned n_vis = 0, n_kept = 0;
#pragma unroll
  for (int k = 0; k < 2 * NP; ++k) {
    const int ly = wp.ly0 + k * G::LROWS;
    const float npy = -((float)ly + 0.5f);
    if (k & 1) npy2[k >> 1].y = npy; else npy2[k >> 1].x = npy;
    inside[k] = k < PPT && (tx * kTile + wp.lx < W) && (ty * kTile + ly < H);
    done[k] = !inside[k];
    lastp[k] = 0;
    stopn[k] = 0;
  }
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    T2[p] = make_float2(1.0f, 1.0f);
    Cr2[p] = Cg2[p] = Cb2[p] = make_float2(0.0f, 0.0f);
  }
  bool counted = false;
  for (int ks = 0;; ++ks) {
    const int st = ks % kWsS;
    if (!warp_mbar_wait(&s_full[st], (unsigned)((ks / kWsS) & 1))) {
      *(volatile int*)&s_abort = 1;
      if (lane == 0) dev_flag(dev_status, GS_DEV_TIMEOUT);
      break;
    }
    const int cnt = sCnt[st];
    if (cnt < 0 || warp_flag(&s_abort)) break;
    bool d_all = true;
#pragma unroll
    for (int k = 0; k < 2 * NP; ++k) d_all = d_all && done[k];
    if (!__all_sync(0xffffffffu, d_all)) {
      const int pos1 = sPos[st] + 1;
      unsigned bits = __ballot_sync(0xffffffffu, lane < cnt && ((sM[st][lane] >> w) & 1u));
      while (bits) {
        const int j = __ffs(bits) - 1;
        bits &= bits - 1u;
        const Packed R = sPk[st][j];
        composite_entry<NP, COUNT>(R, pos1 + j, nfpx2, npy2, T2, Cr2, Cg2, Cb2, done, lastp,
                                   stopn, n_vis, n_kept);
      }
      d_all = true;
#pragma unroll
      for (int k = 0; k < 2 * NP; ++k) d_all = d_all && done[k];
      d_all = __all_sync(0xffffffffu, d_all);
    }
    if (d_all && !counted) {
      counted = true;
      if (lane == 0) atomicAdd(&s_ndone, 1);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s_empty[st]);
  }
  if (COUNT) {  // one atomic per warp: per-thread ones on one word serialise
    unsigned long long e_f = 0, e_b = 0;
#pragma unroll
    for (int k = 0; k < PPT; ++k)
      if (inside[k]) {
        e_f += stopn[k] ? (unsigned long long)stopn[k] : (unsigned long long)(end - begin);
        e_b += (unsigned long long)lastp[k];
      }
    const unsigned long long a = warp_sum((unsigned long long)n_vis);
    const unsigned long long bq = warp_sum((unsigned long long)n_kept);
    const unsigned long long c = warp_sum(e_f);
    const unsigned long long d = warp_sum(e_b);
    if (lane == 0) {
      atomicAdd(&px.counters[0], a);
      atomicAdd(&px.counters[1], bq);
      atomicAdd(&px.counters[2], c);
      atomicAdd(&px.counters[3], d);
    }
  }
  // epilogue: outputs and the fused L1 terms
  float lsum = 0.0f;
#pragma unroll
  for (int k = 0; k < PPT; ++k) {
    if (!inside[k]) continue;
    const int x = tx * kTile + wp.lx, y = ty * kTile + wp.ly0 + k * G::LROWS;
    const int64_t o = (int64_t)(y - px.y0) * px.pitch + (x - px.x0);
    const float2 T_ = T2[k >> 1], r_ = Cr2[k >> 1], g_ = Cg2[k >> 1], b_ = Cb2[k >> 1];
    const float c[3] = {(k & 1) ? r_.y : r_.x, (k & 1) ? g_.y : g_.x, (k & 1) ? b_.y : b_.x};
    if (px.img) {
      px.img[o] = c[0];
      px.img[o + px.plane] = c[1];
      px.img[o + 2 * px.plane] = c[2];
    }
    px.T_final[o] = (k & 1) ? T_.y : T_.x;
    px.last[o] = lastp[k];
    if (px.target) {
      const int64_t ot = (int64_t)(y - px.ty0) * px.tpitch + (x - px.tx0);
#pragma unroll
      for (int ch = 0; ch < 3; ++ch) {
        const float d = c[ch] - px.target[ot + ch * px.tplane];
        px.dL[o + ch * px.plane] = d > 0.0f ? px.norm : (d < 0.0f ? -px.norm : 0.0f);
        lsum += fabsf(d);
      }
    }
  }
  if (px.target && px.loss_tiles) {
    lsum = warp_sum(lsum);
    if (lane == 0) s_red[w] = lsum;
    asm volatile("bar.sync 1, %0;" ::"r"(NC * 32) : "memory");  // the consumer warps only
    if (t == 0) {
      float tot = 0.0f;
      for (int ww = 0; ww < NC; ++ww) tot += s_red[ww];
      px.loss_tiles[(int64_t)ty * TW + tx] = tot * px.norm;
    }
  }
}

// ---------------------------------------------------------------------------
// standalone L1 over a Leaf
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
k_loss_l1(gs_rect leaf, int W, int H, int TW, PixArgs px) {
  __shared__ float s_red[8];
  const int lw = leaf.x1 - leaf.x0;
  const int tx = leaf.x0 + blockIdx.x % lw, ty = leaf.y0 + blockIdx.x / lw;
  const int t = threadIdx.x;
  const int x = tx * kTile + (t & 15), y = ty * kTile + (t >> 4);
  float lsum = 0.0f;
  if (x < W && y < H) {
    const int64_t o = (int64_t)(y - px.y0) * px.pitch + (x - px.x0);
    const int64_t ot = (int64_t)(y - px.ty0) * px.tpitch + (x - px.tx0);
#pragma unroll
    for (int ch = 0; ch < 3; ++ch) {
      const float d = px.img[o + ch * px.plane] - px.target[ot + ch * px.tplane];
      px.dL[o + ch * px.plane] = d > 0.0f ? px.norm : (d < 0.0f ? -px.norm : 0.0f);
      lsum += fabsf(d);
    }
  }
  lsum = warp_sum(lsum);
  if ((t & 31) == 0) s_red[t >> 5] = lsum;
  __syncthreads();
  if (t == 0 && px.loss_tiles) {
    float tot = 0.0f;
    for (int w = 0; w < 8; ++w) tot += s_red[w];
    px.loss_tiles[(int64_t)ty * TW + tx] = tot * px.norm;
  }
}

__global__ void __launch_bounds__(1024)
k_loss_total(const float* __restrict__ tiles, int64_t n, double* __restrict__ out) {
  __shared__ double s[32];
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += 1024) acc += (double)tiles[i];
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) s[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int w = 0; w < 32; ++w) tot += s[w];
    *out = tot;
  }
}

// ---------------------------------------------------------------------------
// backward
// ---------------------------------------------------------------------------

// Sum of 9 values over the warp through a 32 x 9 shared staging area (one
// per warp): every lane stores its 9 values, then lane 3 v + p (v < 9,
// p < 3) adds value v of lanes p, p + 3, p + 6, ... (11 or 10 of them) and
// the three partial sums of value v meet in lane 3 v.  Stride 9 keeps both
// the stores and the loads free of bank conflicts (9 and 27 are odd, and
// 9 p + v < 27 is distinct over the reading lanes).  About 35 instructions
// instead of the ~70 of a nine-value shuffle butterfly.  Returns the total
// of value lane / 3 in lanes 3 v; other lanes return garbage.
__device__ __forceinline__ float warp_reduce9_smem(const float (&v)[9], float* __restrict__ red,
                                                   int lane, int rv, int rp) {
#pragma unroll
  for (int q = 0; q < 9; ++q) red[lane * 9 + q] = v[q];
  __syncwarp();
  float s = 0.0f;
  if (lane < 27) {
    const float* src = red + rp * 9 + rv;
#pragma unroll
    for (int k = 0; k < 11; ++k)
      if (3 * k + rp < 32) s += src[27 * k];
  }
  const float s1 = __shfl_down_sync(0xffffffffu, s, 1);
  const float s2 = __shfl_down_sync(0xffffffffu, s, 2);
  __syncwarp();  // the staging area is free for the next record
  return s + s1 + s2;
}

template <int PPT, bool COUNT>
__global__ void __launch_bounds__(256 / PPT, PPT == 4 ? 14 : 1)
k_raster_bwd(const float4* __restrict__ rec, const int32_t* __restrict__ vals,
             const int64_t* __restrict__ ranges, gs_rect leaf, int W, int H, PixArgs px,
             float* __restrict__ g2d, int32_t* dev_status) {
  using G = TileGeom<PPT>;
  constexpr int NT = G::NT;
  __shared__ PackedB sPk[NT];
  __shared__ float4 sF[NT];  // {2 s1, 2 s2, slot bits, beta}
  __shared__ uint8_t s_mask[NT];
  __shared__ uint8_t s_list[G::NW][NT];
  __shared__ float sg[NT][12];  // the record's 9 sums; word 9: "touched" flag (int)
  __shared__ float s_red[G::NW][32 * 9];
  __shared__ int s_maxlast;
  const int lw = leaf.x1 - leaf.x0;
  const int ltile = blockIdx.x;
  const int tx = leaf.x0 + ltile % lw, ty = leaf.y0 + ltile / lw;
  const int64_t begin = ranges[2 * ltile];
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int rv = lane / 3, rp = lane - 3 * (lane / 3);  // reduction role (warp_reduce9_smem)
  const WarpPix wp = warp_pixels<PPT>(t);
  // the lane's pixels in pairs (an odd PPT's last pair has a placeholder
  // second pixel with last = 0, which never takes part), their state in
  // float2s for packed fp32x2 operations.  NS = -S, S = sum_c g_c A_c with
  // A_c the colour composited behind the current entry.
  constexpr int NP = (PPT + 1) / 2;
  const float fpx = (float)wp.lx + 0.5f;
  const float2 nfpx2 = make_float2(-fpx, -fpx);
  float2 npy2[NP], T2[NP], NS2[NP], gr2[NP], gg2[NP], gb2[NP];
  int lastp[2 * NP];
  if (t == 0) s_maxlast = 0;
  for (int e = t; e < NT * 12; e += NT) (&sg[0][0])[e] = 0.0f;
  __syncthreads();
  int mylast = 0;
#pragma unroll
  for (int k = 0; k < 2 * NP; ++k) {
    const int ly = wp.ly0 + k * G::LROWS;
    const int x = tx * kTile + wp.lx, y = ty * kTile + ly;
    float Tk = 1.0f, r = 0.0f, g = 0.0f, b = 0.0f;
    int lk = 0;
    if (k < PPT && x < W && y < H) {
      const int64_t o = (int64_t)(y - px.y0) * px.pitch + (x - px.x0);
      Tk = px.T_final[o];
      lk = px.last[o];
      r = px.dL[o];
      g = px.dL[o + px.plane];
      b = px.dL[o + 2 * px.plane];
    }
    const float npy = -((float)ly + 0.5f);
    if (k & 1) {
      npy2[k >> 1].y = npy; T2[k >> 1].y = Tk; NS2[k >> 1].y = 0.0f;
      gr2[k >> 1].y = r; gg2[k >> 1].y = g; gb2[k >> 1].y = b;
    } else {
      npy2[k >> 1].x = npy; T2[k >> 1].x = Tk; NS2[k >> 1].x = 0.0f;
      gr2[k >> 1].x = r; gg2[k >> 1].x = g; gb2[k >> 1].x = b;
    }
    lastp[k] = lk;
    mylast = max(mylast, lk);
  }
  const int warp_last = __reduce_max_sync(0xffffffffu, mylast);
  if (lane == 0) atomicMax(&s_maxlast, warp_last);
  __syncthreads();
  const int tile_last = s_maxlast;
  unsigned n_vis = 0, n_kept = 0;
  const float2 one2 = make_float2(1.0f, 1.0f), zero2 = make_float2(0.0f, 0.0f);

  for (int bend = tile_last; bend > 0; bend -= NT) {
    const int bstart = max(0, bend - NT);
    const int cnt = bend - bstart;
    if (t < cnt) {
      const int pos = bend - 1 - t;
      const Staged st = stage_record(rec, vals[begin + pos], tx, ty);
      s_mask[t] = (uint8_t)warp_mask<PPT>(st);
      sPk[t] = pack_record_bwd(st);
      sF[t] = make_float4(2.0f * st.s1, 2.0f * st.s2, __int_as_float(st.slot), st.beta);
    }
    __syncthreads();
    // positions at or beyond every lane's `last` need no work in this warp
    const int jstart = max(0, bend - warp_last);
    const int nl = warp_list<uint8_t>(s_mask, jstart, cnt, w, lane, s_list[w]);
    for (int i = 0; i < nl; ++i) {
      const int j = s_list[w][i];
      const int pos = bend - 1 - j;
      const PackedB R = sPk[j];
      // per pair: m6..m8 = -sum alpha T_before g_c, and the dq moments (the
      // lane's pixels share dx, so the geometric terms need only sum dq,
      // sum dq dy and sum dq dy^2 over them)
      float2 m6 = zero2, m7 = zero2, m8 = zero2, sq2 = zero2, sqy2 = zero2, sqyy2 = zero2;
      bool any = false;
      const float2 dx2 = __fadd2_rn(R.gx, nfpx2);  // gx - px
      // branch-free: an entry at or beyond the pixel's last, or below 1/255,
      // enters with alpha = 0, which leaves T, S and every sum unchanged
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const float2 dy = __fadd2_rn(R.gy, npy2[p]);
        const float2 t1 = __ffma2_rn(R.beta, dy, dx2);
        const float2 qa = __fmul2_rn(R.ns1, t1);
        const float2 qb = __ffma2_rn(__fmul2_rn(R.ns2, dy), dy, R.lo2);
        const float2 e = __ffma2_rn(qa, t1, qb);
        const float raw[2] = {ex2_approx(e.x), ex2_approx(e.y)};  // o e^-q
        float nau[2], nua[2];
        bool use[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const bool inl = pos < lastp[2 * p + h];
          const float na = fmaxf(-raw[h], -kAlphaMax);  // -alpha
          use[h] = inl && na <= -kAlphaMin;
          if (COUNT) {
            n_vis += inl ? 1u : 0u;
            n_kept += use[h] ? 1u : 0u;
          }
          any = any || use[h];
          nau[h] = use[h] ? na : 0.0f;
          // unclamped entries (alpha = araw = o e^-q): dL/dq (natural
          // units) = -alpha dL/dalpha, and o dL/dopacity = alpha dL/dalpha
          nua[h] = raw[h] <= kAlphaMax ? nau[h] : 0.0f;
        }
        const float2 nau2 = make_float2(nau[0], nau[1]);
        // T only scales gradient values here (no decision depends on it), so
        // the hardware reciprocal (about 1 ulp) is enough
        const float2 om = __fadd2_rn(one2, nau2);  // 1 - alpha
        const float2 inv = make_float2(rcp_approx(om.x), rcp_approx(om.y));
        const float2 Tb = __fmul2_rn(T2[p], inv);  // transmittance before this entry
        const float2 nwgt = __fmul2_rn(nau2, Tb);   // -alpha T_before
        m6 = __ffma2_rn(nwgt, gr2[p], m6);
        m7 = __ffma2_rn(nwgt, gg2[p], m7);
        m8 = __ffma2_rn(nwgt, gb2[p], m8);
        // dL/dalpha = sum_c g_c (rgb_c T_before - A_c / (1 - alpha))
        //           = T_before (g . rgb) - S / (1 - alpha)
        const float2 grgb =
            __ffma2_rn(gb2[p], R.b, __ffma2_rn(gg2[p], R.g, __fmul2_rn(gr2[p], R.r)));
        const float2 da = __ffma2_rn(Tb, grgb, __fmul2_rn(NS2[p], inv));
        NS2[p] = __ffma2_rn(nwgt, grgb, NS2[p]);
        T2[p].x = use[0] ? Tb.x : T2[p].x;
        T2[p].y = use[1] ? Tb.y : T2[p].y;
        const float2 dq = __fmul2_rn(make_float2(nua[0], nua[1]), da);
        sq2 = __fadd2_rn(sq2, dq);
        const float2 dqy = __fmul2_rn(dq, dy);
        sqy2 = __fadd2_rn(sqy2, dqy);
        sqyy2 = __ffma2_rn(dqy, dy, sqyy2);
      }
      // the geometric gradients are linear in five moments of dq over the
      // warp's pixels: sum dx dq, sum dx^2 dq, sum dq dy, sum dx dq dy and
      // sum dq dy^2 (turned into du, dv, da, db, dc once per record at the
      // flush below); o dL/do = sum alpha dL/dalpha = -sum dq
      const float dx = dx2.x;
      const float sq = sq2.x + sq2.y, sqy = sqy2.x + sqy2.y;
      float acc[9];
      const float dxq = dx * sq;
      acc[0] = dxq;
      acc[1] = dx * dxq;
      acc[2] = sqy;
      acc[3] = dx * sqy;
      acc[4] = sqyy2.x + sqyy2.y;
      acc[5] = -sq;
      acc[6] = -(m6.x + m6.y);
      acc[7] = -(m7.x + m7.y);
      acc[8] = -(m8.x + m8.y);
      // reduce first: per-lane shared atomics on the same 9 words cost more
      // than the reduction, even with only 2 lanes kept
      if (__any_sync(0xffffffffu, any)) {
        const float tot = warp_reduce9_smem(acc, s_red[w], lane, rv, rp);
        if (lane < 27 && rp == 0) atomicAdd(&sg[j][rv], tot);
        if (lane == 0) reinterpret_cast<int*>(sg[j])[9] = 1;
      }
    }
    __syncthreads();
    if (t < cnt && reinterpret_cast<const int*>(sg[t])[9]) {
      const float4 F = sF[t];
      const int32_t slot = __float_as_int(F.z);
      const float beta = F.w;
      // q = (a dx^2 + c dy^2) / 2 + b dx dy with a = 2 s1, b = beta a,
      // c = 2 s2 + beta b: dq/du = a dx + b dy, dq/dv = b dx + c dy
      // = beta dq/du + 2 s2 dy, dq/da = dx^2 / 2, dq/db = dx dy, dq/dc = dy^2 / 2
      const float du = F.x * fmaf(beta, sg[t][2], sg[t][0]);
      const float dv = fmaf(beta, du, F.y * sg[t][2]);
      float4* dst = reinterpret_cast<float4*>(g2d + (int64_t)slot * 12);
      atomicAdd(dst, make_float4(du, dv, 0.5f * sg[t][1], sg[t][3]));
      // dL/do = sum e^-q dL/dalpha = (sum o e^-q dL/dalpha) / o, 1/o = 2^-log2 o
      const float inv_o = ex2_approx(-sPk[t].lo2.x);
      atomicAdd(dst + 1, make_float4(0.5f * sg[t][4], sg[t][5] * inv_o, sg[t][6], sg[t][7]));
      atomicAdd(dst + 2, make_float4(sg[t][8], 0.0f, 0.0f, 0.0f));
#pragma unroll
      for (int q = 0; q < 9; ++q) sg[t][q] = 0.0f;
      reinterpret_cast<int*>(sg[t])[9] = 0;
    }
    __syncthreads();
  }
  if (COUNT) {  // one atomic per warp: per-thread ones on one word serialise
    const unsigned long long a = warp_sum((unsigned long long)n_vis);
    const unsigned long long b = warp_sum((unsigned long long)n_kept);
    if ((t & 31) == 0) {
      atomicAdd(&px.counters[0], a);
      atomicAdd(&px.counters[1], b);
    }
  }
}

PixArgs to_args(const gs_pixels* p) {
  PixArgs a;
  a.x0 = p->x0; a.y0 = p->y0; a.w = p->w; a.h = p->h;
  a.pitch = p->pitch; a.plane = p->plane;
  a.img = p->img; a.T_final = p->T_final; a.last = p->last; a.dL = p->dL_dimg;
  a.target = p->target; a.tx0 = p->tx0; a.ty0 = p->ty0; a.tpitch = p->tpitch;
  a.tplane = p->tplane; a.loss_tiles = p->loss_tiles;
  a.norm = (float)p->norm;
  a.counters = p->counters;
  return a;
}

// The Leaf's pixels (clipped to the image) must lie inside the buffers.
bool check_pixels(const gs_pixels* p, gs_rect leaf, const gs_camera* cam) {
  if (!p) return false;
  const int64_t X0 = (int64_t)leaf.x0 * kTile, Y0 = (int64_t)leaf.y0 * kTile;
  const int64_t X1 = std::min<int64_t>((int64_t)leaf.x1 * kTile, cam->width);
  const int64_t Y1 = std::min<int64_t>((int64_t)leaf.y1 * kTile, cam->height);
  if (X0 < p->x0 || Y0 < p->y0 || X1 > (int64_t)p->x0 + p->w || Y1 > (int64_t)p->y0 + p->h)
    return false;
  if (p->pitch < p->w || p->plane < p->pitch * (int64_t)p->h) return false;
  if (p->target) {
    if (X0 < p->tx0 || Y0 < p->ty0 || p->tpitch < X1 - p->tx0) return false;
    if (p->tplane < p->tpitch * (Y1 - p->ty0)) return false;
  }
  return true;
}

bool check_leaf(gs_rect leaf, const gs_camera* cam) {
  const int64_t TW = tiles_x(cam->width), TH = tiles_y(cam->height);
  return leaf.x0 >= 0 && leaf.y0 >= 0 && leaf.x1 > leaf.x0 && leaf.y1 > leaf.y0 &&
         leaf.x1 <= TW && leaf.y1 <= TH;
}

int pick_ppt(uint32_t flags, int dflt) {
  const int p = (int)(flags & 7u);
  return (p == 1 || p == 2 || p == 4) ? p : dflt;
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" gs_status gs_raster_fwd(const gs_proj* proj, const int32_t* vals, const int64_t* ranges,
                                   gs_rect leaf, const gs_camera* cam, const gs_pixels* px,
                                   uint32_t flags, int32_t* dev_status, gs_stream stream) {
  if (!proj || !ranges || !cam || !check_leaf(leaf, cam) || !check_pixels(px, leaf, cam))
    return GS_ERR_ARG;
  if (!px->T_final || !px->last || (px->target && !px->dL_dimg)) return GS_ERR_ARG;
  if (!aligned(proj->rec, 16)) return GS_ERR_ARG;
  const int64_t ntiles = (int64_t)(leaf.x1 - leaf.x0) * (leaf.y1 - leaf.y0);
  const PixArgs a = to_args(px);
  const int TW = (int)tiles_x(cam->width);
  cudaStream_t s = to_stream(stream);
  const float4* rec = reinterpret_cast<const float4*>(proj->rec);
  const unsigned nb = (unsigned)ntiles;
  const int W = cam->width, H = cam->height;
  const bool cnt = px->counters != nullptr;
  const BlockSrc none{nullptr, nullptr, nullptr, 0, nullptr, nullptr};
#define GS_FWD(P, C) \
  k_raster_fwd<P, C, false><<<nb, 256 / P, 0, s>>>(rec, vals, ranges, leaf, W, H, TW, a, none, dev_status)
  switch (pick_ppt(flags, 2)) {
    case 1: if (cnt) GS_FWD(1, true); else GS_FWD(1, false); break;
    case 2: if (cnt) GS_FWD(2, true); else GS_FWD(2, false); break;
    default: if (cnt) GS_FWD(4, true); else GS_FWD(4, false); break;
  }
#undef GS_FWD
  GS_LAUNCH_CHECK();
  return GS_OK;
}

extern "C" gs_status gs_raster_fwd_blocks(const gs_proj* proj, const int32_t* block_vals,
                                          const int64_t* block_ranges, gs_rect leaf,
                                          const gs_camera* cam, const gs_pixels* px,
                                          int32_t* vals, int64_t capacity, int64_t n_isect,
                                          int64_t* ranges, int64_t* needed, uint32_t flags,
                                          int32_t* dev_status, gs_stream stream) {
  if (!proj || !ranges || !cam || !block_ranges || !check_leaf(leaf, cam) ||
      !check_pixels(px, leaf, cam) || n_isect < 0)
    return GS_ERR_ARG;
  if (n_isect > capacity) {
    if (needed) *needed = n_isect;
    return GS_ERR_CAPACITY;
  }
  if (!px->T_final || !px->last || (px->target && !px->dL_dimg)) return GS_ERR_ARG;
  if (n_isect > 0 && (!vals || !block_vals || !proj->rect)) return GS_ERR_ARG;
  if (!aligned(proj->rec, 16) || !aligned(proj->rect, 8)) return GS_ERR_ARG;
  const int64_t ntiles = (int64_t)(leaf.x1 - leaf.x0) * (leaf.y1 - leaf.y0);
  const PixArgs a = to_args(px);
  const int TW = (int)tiles_x(cam->width);
  cudaStream_t s = to_stream(stream);
  const float4* rec = reinterpret_cast<const float4*>(proj->rec);
  const unsigned nb = (unsigned)ntiles;
  const int W = cam->width, H = cam->height;
  const bool cnt = px->counters != nullptr;
  const BlockSrc src{reinterpret_cast<const short4*>(proj->rect), block_vals, block_ranges,
                     (TW + GS_TILE_BLOCK - 1) / GS_TILE_BLOCK, vals, ranges};
  if (flags & GS_RASTER_WS) {
    // warp-specialised: a producer warp fills and stages, NC warps composite
#define GS_FWD(P, C) \
  k_raster_fwd_ws<P, C><<<nb, 256 / P + 32, 0, s>>>(rec, leaf, W, H, TW, a, src, dev_status)
    switch (pick_ppt(flags, 2)) {
      case 4: if (cnt) GS_FWD(4, true); else GS_FWD(4, false); break;
      default: if (cnt) GS_FWD(2, true); else GS_FWD(2, false); break;
    }
#undef GS_FWD
    GS_LAUNCH_CHECK();
    return GS_OK;
  }
#define GS_FWD(P, C) \
  k_raster_fwd<P, C, true><<<nb, 256 / P, 0, s>>>(rec, vals, ranges, leaf, W, H, TW, a, src, dev_status)
  switch (pick_ppt(flags, 2)) {
    case 1: if (cnt) GS_FWD(1, true); else GS_FWD(1, false); break;
    case 2: if (cnt) GS_FWD(2, true); else GS_FWD(2, false); break;
    default: if (cnt) GS_FWD(4, true); else GS_FWD(4, false); break;
  }
#undef GS_FWD
  GS_LAUNCH_CHECK();
  return GS_OK;
}

extern "C" gs_status gs_loss_l1(const gs_pixels* px, gs_rect leaf, const gs_camera* cam,
                                gs_stream stream) {
  if (!cam || !check_leaf(leaf, cam) || !check_pixels(px, leaf, cam)) return GS_ERR_ARG;
  if (!px->img || !px->target || !px->dL_dimg) return GS_ERR_ARG;
  const int64_t ntiles = (int64_t)(leaf.x1 - leaf.x0) * (leaf.y1 - leaf.y0);
  k_loss_l1<<<(unsigned)ntiles, 256, 0, to_stream(stream)>>>(leaf, cam->width, cam->height,
                                                             (int)tiles_x(cam->width), to_args(px));
  GS_LAUNCH_CHECK();
  return GS_OK;
}

extern "C" gs_status gs_loss_total(const float* loss_tiles, int64_t n, double* loss,
                                   gs_stream stream) {
  if (n < 0 || !loss || (n > 0 && !loss_tiles)) return GS_ERR_ARG;
  k_loss_total<<<1, 1024, 0, to_stream(stream)>>>(loss_tiles, n, loss);
  GS_LAUNCH_CHECK();
  return GS_OK;
}

extern "C" gs_status gs_raster_bwd(const gs_proj* proj, const int32_t* vals, const int64_t* ranges,
                                   gs_rect leaf, const gs_camera* cam, const gs_pixels* px,
                                   float* g2d, uint32_t flags, int32_t* dev_status,
                                   gs_stream stream) {
  if (!proj || !ranges || !cam || !g2d || !check_leaf(leaf, cam) || !check_pixels(px, leaf, cam))
    return GS_ERR_ARG;
  if (!px->T_final || !px->last || !px->dL_dimg) return GS_ERR_ARG;
  if (!aligned(proj->rec, 16) || !aligned(g2d, 16)) return GS_ERR_ARG;
  const int64_t ntiles = (int64_t)(leaf.x1 - leaf.x0) * (leaf.y1 - leaf.y0);
  const PixArgs a = to_args(px);
  cudaStream_t s = to_stream(stream);
  const float4* rec = reinterpret_cast<const float4*>(proj->rec);
  const unsigned nb = (unsigned)ntiles;
  const int W = cam->width, H = cam->height;
  const bool cnt = px->counters != nullptr;
#define GS_BWD(P, C) k_raster_bwd<P, C><<<nb, 256 / P, 0, s>>>(rec, vals, ranges, leaf, W, H, a, g2d, dev_status)
  switch (pick_ppt(flags, 4)) {
    case 1: if (cnt) GS_BWD(1, true); else GS_BWD(1, false); break;
    case 2: if (cnt) GS_BWD(2, true); else GS_BWD(2, false); break;
    default: if (cnt) GS_BWD(4, true); else GS_BWD(4, false); break;
  }
#undef GS_BWD
  GS_LAUNCH_CHECK();
  return GS_OK;
}
