// gs_project: cull + EWA projection of the candidate Gaussians, ordered
// compaction of the candidates, per-tile intersection counts and their
// summed-area table.
//
// BoundedGS project page, section 02 (C -> D -> E): only Gaussians that can
// touch the view get projected state ("candidate-index projection").
// SkipGS paper notes, "loss function / training strategy": the rasteriser
// projects each Gaussian to a 2D covariance; its colour comes from SH.
//
// One thread per Gaussian.  The arithmetic is fp64: the pass reads ~236
// bytes per candidate from HBM and does a few hundred flops, so fp64 costs
// nothing here, and it makes every integer decision (cull, tile rect, depth
// key) independent of fp32 rounding.  The camera-space position, screen
// position and cull tests use explicitly rounded operations in a fixed order.
#include <cuda_fp16.h>
#include <math.h>

#include "gs_internal.cuh"

namespace gs {
namespace {

#ifndef GS_PROJ_THREADS
#define GS_PROJ_THREADS 256
#endif
#ifndef GS_PROJ_MINB
#define GS_PROJ_MINB 4
#endif
constexpr int kProjThreads = GS_PROJ_THREADS;
// blocks between a block and the one whose geometric planes it prefetches:
// about one wave of resident blocks (148 SMs x GS_PROJ_MINB)
constexpr int kProjAhead = 148 * GS_PROJ_MINB * 256 / GS_PROJ_THREADS;

struct ProjCam {
  double R[9], t[3];
  double fx, fy, cx, cy, limx, limy;
  double campos[3];
  int32_t W, H, TW, TH;
  int32_t RX0, RY0, RX1, RY1;  // tile region the rects are clipped to
};

// Real SH basis, degree <= 3: Y_0 = 1/(2 sqrt(pi)), band l = 1 ordered
// (m = -1, 0, 1) as (-y, z, -x) sqrt(3/(4 pi)), bands 2 and 3 the homogeneous
// polynomials with their closed-form normalisations (Condon-Shortley phase).
__device__ __forceinline__ void sh_basis(double x, double y, double z, int D, double* Y) {
  const double kPi = 3.141592653589793;
  Y[0] = 0.5 / sqrt(kPi);
  if (D < 1) return;
  const double k1 = sqrt(3.0 / (4.0 * kPi));
  Y[1] = -k1 * y;
  Y[2] = k1 * z;
  Y[3] = -k1 * x;
  if (D < 2) return;
  const double xx = x * x, yy = y * y, zz = z * z;
  const double k2a = 0.5 * sqrt(15.0 / kPi), k2b = 0.25 * sqrt(5.0 / kPi),
               k2c = 0.25 * sqrt(15.0 / kPi);
  Y[4] = k2a * x * y;
  Y[5] = -k2a * y * z;
  Y[6] = k2b * (2.0 * zz - xx - yy);
  Y[7] = -k2a * x * z;
  Y[8] = k2c * (xx - yy);
  if (D < 3) return;
  const double k3a = 0.25 * sqrt(35.0 / (2.0 * kPi)), k3b = 0.5 * sqrt(105.0 / kPi),
               k3c = 0.25 * sqrt(21.0 / (2.0 * kPi)), k3d = 0.25 * sqrt(7.0 / kPi),
               k3e = 0.25 * sqrt(105.0 / kPi);
  Y[9] = -k3a * y * (3.0 * xx - yy);
  Y[10] = k3b * x * y * z;
  Y[11] = -k3c * y * (4.0 * zz - xx - yy);
  Y[12] = k3d * z * (2.0 * zz - 3.0 * xx - 3.0 * yy);
  Y[13] = -k3c * x * (4.0 * zz - xx - yy);
  Y[14] = k3e * z * (xx - yy);
  Y[15] = -k3a * x * (xx - 3.0 * yy);
}

// The geometric part of a candidate's projection (everything but colour).
struct ProjGeo {
  double x, y, z;        // mean
  double u, v, hx, hy;   // pixel position, alpha-box half extents
  double c00, c01, c11, det, opac, tz;
  short4 rect;
  int64_t square_tiles;
};

// Cull + geometry of Gaussian i from its 11 geometric planes; true if it is
// a candidate.  The SH planes are read only for candidates (sh_colour).
// `counted` is set once the Gaussian is a candidate of the full view (its
// square tiles in the region then count towards the 3-sigma total, even if
// its tight rect misses the region).
__device__ __forceinline__ bool project_geometry(const float* __restrict__ P, int64_t n_pad,
                                                 int64_t i, const ProjCam& c, ProjGeo& o,
                                                 bool& nonfinite, bool& counted) {
  const double x = P[i], y = P[n_pad + i], z = P[2 * n_pad + i];
  double tc[3];
#pragma unroll
  for (int r = 0; r < 3; ++r)
    tc[r] = __dadd_rn(__dadd_rn(__dadd_rn(__dmul_rn(c.R[3 * r], x), __dmul_rn(c.R[3 * r + 1], y)),
                                __dmul_rn(c.R[3 * r + 2], z)),
                      c.t[r]);
  float pv[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) pv[k] = P[(3 + k) * n_pad + i];
  bool fin = isfinite(x) && isfinite(y) && isfinite(z);
#pragma unroll
  for (int k = 0; k < 8; ++k) fin = fin && isfinite(pv[k]);
  if (!fin) {
    nonfinite = true;
    return false;
  }
  const double tz = tc[2];
  if (!(tz > 0.2)) return false;
  const double xn = __ddiv_rn(tc[0], tz), yn = __ddiv_rn(tc[1], tz);
  if (fabs(xn) > c.limx || fabs(yn) > c.limy) return false;
  const double u = __dadd_rn(__dmul_rn(c.fx, xn), c.cx);
  const double v = __dadd_rn(__dmul_rn(c.fy, yn), c.cy);

  // 3D covariance from the normalised quaternion and the scales
  double qw = pv[3], qx = pv[4], qy = pv[5], qz = pv[6];
  const double qn = sqrt(qw * qw + qx * qx + qy * qy + qz * qz);
  if (!(qn > 0.0)) {
    nonfinite = true;
    return false;
  }
  const double iqn = 1.0 / qn;
  qw *= iqn; qx *= iqn; qy *= iqn; qz *= iqn;
  double Rg[9];
  Rg[0] = 1.0 - 2.0 * (qy * qy + qz * qz); Rg[1] = 2.0 * (qx * qy - qw * qz); Rg[2] = 2.0 * (qx * qz + qw * qy);
  Rg[3] = 2.0 * (qx * qy + qw * qz); Rg[4] = 1.0 - 2.0 * (qx * qx + qz * qz); Rg[5] = 2.0 * (qy * qz - qw * qx);
  Rg[6] = 2.0 * (qx * qz - qw * qy); Rg[7] = 2.0 * (qy * qz + qw * qx); Rg[8] = 1.0 - 2.0 * (qx * qx + qy * qy);
  const double s0 = exp((double)pv[0]), s1 = exp((double)pv[1]), s2 = exp((double)pv[2]);
  double M[9];
#pragma unroll
  for (int r = 0; r < 3; ++r) {
    M[3 * r] = Rg[3 * r] * s0;
    M[3 * r + 1] = Rg[3 * r + 1] * s1;
    M[3 * r + 2] = Rg[3 * r + 2] * s2;
  }
  double Sg[6];  // symmetric 3x3: 00 01 02 11 12 22
  Sg[0] = M[0] * M[0] + M[1] * M[1] + M[2] * M[2];
  Sg[1] = M[0] * M[3] + M[1] * M[4] + M[2] * M[5];
  Sg[2] = M[0] * M[6] + M[1] * M[7] + M[2] * M[8];
  Sg[3] = M[3] * M[3] + M[4] * M[4] + M[5] * M[5];
  Sg[4] = M[3] * M[6] + M[4] * M[7] + M[5] * M[8];
  Sg[5] = M[6] * M[6] + M[7] * M[7] + M[8] * M[8];
  // T = J W, J the perspective Jacobian at t
  const double itz = 1.0 / tz;
  const double j00 = c.fx * itz, j02 = -j00 * xn;
  const double j11 = c.fy * itz, j12 = -j11 * yn;
  double T0[3], T1[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    T0[k] = j00 * c.R[k] + j02 * c.R[6 + k];
    T1[k] = j11 * c.R[3 + k] + j12 * c.R[6 + k];
  }
  // A = T Sigma (2x3), then Sigma2 = A T^T
  double A0[3], A1[3];
  A0[0] = T0[0] * Sg[0] + T0[1] * Sg[1] + T0[2] * Sg[2];
  A0[1] = T0[0] * Sg[1] + T0[1] * Sg[3] + T0[2] * Sg[4];
  A0[2] = T0[0] * Sg[2] + T0[1] * Sg[4] + T0[2] * Sg[5];
  A1[0] = T1[0] * Sg[0] + T1[1] * Sg[1] + T1[2] * Sg[2];
  A1[1] = T1[0] * Sg[1] + T1[1] * Sg[3] + T1[2] * Sg[4];
  A1[2] = T1[0] * Sg[2] + T1[1] * Sg[4] + T1[2] * Sg[5];
  const double c00 = A0[0] * T0[0] + A0[1] * T0[1] + A0[2] * T0[2] + 0.3;
  const double c01 = 0.5 * ((A0[0] * T1[0] + A0[1] * T1[1] + A0[2] * T1[2]) +
                            (A1[0] * T0[0] + A1[1] * T0[1] + A1[2] * T0[2]));
  const double c11 = A1[0] * T1[0] + A1[1] * T1[1] + A1[2] * T1[2] + 0.3;
  const double det = c00 * c11 - c01 * c01;
  if (!(det > 0.0)) return false;
  const double mid = 0.5 * (c00 + c11);
  const double lam = mid + sqrt(fmax(0.1, mid * mid - det));
  const double rad = ceil(3.0 * sqrt(lam));
  const int64_t rx0 = (int64_t)floor((u - rad) / kTile), rx1 = (int64_t)floor((u + rad) / kTile) + 1;
  const int64_t ry0 = (int64_t)floor((v - rad) / kTile), ry1 = (int64_t)floor((v + rad) / kTile) + 1;
  const double opac = 1.0 / (1.0 + exp(-(double)pv[7]));
  // tiles whose pixel-centre box can see alpha >= 1/255: o exp(-q) >= 1/255
  // holds only inside the ellipse q <= ln(255 o); its bounding box, inflated
  // well beyond the fp32 error of the rasteriser's alpha, bounds the rect
  const double lq = log(255.0 * opac);
  if (!(lq > -1e-4)) return false;  // never reaches 1/255 anywhere
  const double qb = fmax(lq, 0.0) * 1.0001 + 1e-4;
  const double hx = sqrt(2.0 * qb * c00) + 0.01, hy = sqrt(2.0 * qb * c11) + 0.01;
  const int64_t bx0 = (int64_t)ceil((u - hx - 15.5) / kTile), bx1 = (int64_t)floor((u + hx - 0.5) / kTile) + 1;
  const int64_t by0 = (int64_t)ceil((v - hy - 15.5) / kTile), by1 = (int64_t)floor((v + hy - 0.5) / kTile) + 1;
  const int64_t cx0 = rx0 > bx0 ? rx0 : bx0, cx1 = rx1 < bx1 ? rx1 : bx1;
  const int64_t cy0 = ry0 > by0 ? ry0 : by0, cy1 = ry1 < by1 ? ry1 : by1;
  {  // a candidate of the full view: its tight rect meets the grid
    const int64_t gx0 = cx0 < 0 ? 0 : cx0, gx1 = cx1 > c.TW ? c.TW : cx1;
    const int64_t gy0 = cy0 < 0 ? 0 : cy0, gy1 = cy1 > c.TH ? c.TH : cy1;
    if (gx0 >= gx1 || gy0 >= gy1) return false;
  }
  counted = true;
  {
    // tiles of the plain 3-sigma square within the region, for the metric
    const int64_t sx0 = rx0 < c.RX0 ? c.RX0 : (rx0 > c.RX1 ? c.RX1 : rx0);
    const int64_t sx1 = rx1 < c.RX0 ? c.RX0 : (rx1 > c.RX1 ? c.RX1 : rx1);
    const int64_t sy0 = ry0 < c.RY0 ? c.RY0 : (ry0 > c.RY1 ? c.RY1 : ry0);
    const int64_t sy1 = ry1 < c.RY0 ? c.RY0 : (ry1 > c.RY1 ? c.RY1 : ry1);
    o.square_tiles = (sx1 > sx0 && sy1 > sy0) ? (sx1 - sx0) * (sy1 - sy0) : 0;
  }
  const int64_t x0 = cx0 < c.RX0 ? c.RX0 : (cx0 > c.RX1 ? c.RX1 : cx0);
  const int64_t x1 = cx1 < c.RX0 ? c.RX0 : (cx1 > c.RX1 ? c.RX1 : cx1);
  const int64_t y0 = cy0 < c.RY0 ? c.RY0 : (cy0 > c.RY1 ? c.RY1 : cy0);
  const int64_t y1 = cy1 < c.RY0 ? c.RY0 : (cy1 > c.RY1 ? c.RY1 : cy1);
  if (x0 >= x1 || y0 >= y1) return false;
  o.x = x; o.y = y; o.z = z;
  o.u = u; o.v = v; o.hx = hx; o.hy = hy;
  o.c00 = c00; o.c01 = c01; o.c11 = c11; o.det = det; o.opac = opac; o.tz = tz;
  o.rect = make_short4((short)x0, (short)y0, (short)x1, (short)y1);

  return true;
}

// Colour from SH at the direction camera centre -> mean, then the record.
template <int D>
__device__ __forceinline__ void sh_record(const float* __restrict__ P, int64_t n_pad, int64_t i,
                                          const ProjCam& c, const ProjGeo& g, float4& r0,
                                          float4& r1, float4& r2) {
  double dx = g.x - c.campos[0], dy = g.y - c.campos[1], dz = g.z - c.campos[2];
  const double idn = 1.0 / sqrt(dx * dx + dy * dy + dz * dz);
  dx *= idn; dy *= idn; dz *= idn;
  constexpr int ksh = (D + 1) * (D + 1);
  float sh[ksh][3];
#pragma unroll
  for (int k = 0; k < ksh; ++k)
#pragma unroll
    for (int ch = 0; ch < 3; ++ch) sh[k][ch] = P[(11 + 3 * k + ch) * n_pad + i];
  double Y[16];
  sh_basis(dx, dy, dz, D, Y);
  double rgb[3] = {0.5, 0.5, 0.5};
#pragma unroll
  for (int k = 0; k < ksh; ++k)
#pragma unroll
    for (int ch = 0; ch < 3; ++ch) rgb[ch] += (double)sh[k][ch] * Y[k];
  const float uh = (float)g.u, vh = (float)g.v;
  // u, v as fp32 + fp16 corrections (|lo| <= ulp(u)/2, so the pair is exact
  // to ~2e-7 px); the alpha box half extents as fp16 rounded up
  const __half2 lo = __floats2half2_rn((float)(g.u - (double)uh), (float)(g.v - (double)vh));
  const __half2 box = __halves2half2(__float2half_ru((float)g.hx), __float2half_ru((float)g.hy));
  r0 = make_float4(uh, vh, __uint_as_float(*reinterpret_cast<const unsigned*>(&lo)),
                   __uint_as_float(*reinterpret_cast<const unsigned*>(&box)));
  // conic (a, b, c) = (c11, -c01, c00) / det; the record keeps s1 = a / 2,
  // beta = b / a = -c01 / c11 and s2 = (c - b^2 / a) / 2 = 1 / (2 c11), so
  // that q = s1 (dx + beta dy)^2 + s2 dy^2
  const double ic11 = 1.0 / g.c11;
  r1 = make_float4((float)(0.5 * g.c11 / g.det), (float)(-g.c01 * ic11), (float)(0.5 * ic11),
                   (float)g.opac);
  const float depth = (float)g.tz;
  r2 = make_float4((float)fmax(rgb[0], 0.0), (float)fmax(rgb[1], 0.0), (float)fmax(rgb[2], 0.0),
                   depth);
}

// 4 CTAs of 256 per SM (64 registers, a few spilled): on the 6M view the
// kernel takes 0.615 ms, against 0.665 ms at 3 CTAs (80 registers) and
// 0.632 ms with 8 CTAs of 128
template <int D>
__global__ void __launch_bounds__(kProjThreads, GS_PROJ_MINB)
k_project(const float* __restrict__ params, int64_t n, int64_t n_pad, ProjCam cam,
          int32_t* __restrict__ cand_idx, int32_t* __restrict__ slot_map, float4* __restrict__ rec,
          short4* __restrict__ rect, uint32_t* __restrict__ depth_key, int32_t* __restrict__ diff,
          unsigned long long* __restrict__ lb, unsigned int* __restrict__ ticket,
          int32_t* __restrict__ n_cand, int64_t n_blocks, int64_t capacity,
          unsigned long long* __restrict__ square_isect, bool dense, bool prefetch,
          int32_t* dev_status) {
  __shared__ unsigned int s_b;
  if (threadIdx.x == 0) s_b = atomicAdd(ticket, 1u);
  __syncthreads();
  const int64_t b = s_b;
  const int64_t i = b * kProjThreads + threadIdx.x;
  // the block's SH segments (1 KB per plane) head for L2 while the geometry,
  // the scan and the look-back run; the geometric planes of the block one
  // wave ahead likewise
  constexpr int kSH = 3 * (D + 1) * (D + 1);
  if (prefetch && threadIdx.x < kSH + 11) {
    const int64_t blk = threadIdx.x < kSH ? b : b + kProjAhead;
    const int plane = threadIdx.x < kSH ? 11 + threadIdx.x : threadIdx.x - kSH;
    const int64_t first = blk * kProjThreads;
    if (first < n) {
      const int64_t cnt = n_pad - first < kProjThreads ? n_pad - first : kProjThreads;
      bulk_prefetch_l2(params + (int64_t)plane * n_pad + first, (unsigned)(cnt * 4));
    }
  }
  ProjGeo o;
  o.square_tiles = 0;
  bool nonfinite = false, counted = false;
  // cull and geometry first, so the CTA's scan below waits only on the 11
  // geometric planes; the 48 SH planes are read after it, by candidates
  const bool cand = i < n && project_geometry(params, n_pad, i, cam, o, nonfinite, counted);
  if (nonfinite) dev_flag(dev_status, GS_DEV_NONFINITE);
  if (dense) {
    // every Gaussian keeps slot i; a culled one gets an empty rect, depth -1
    // and the largest depth key (it is never binned)
    if (i < n) {
      slot_map[i] = (int32_t)i;
      cand_idx[i] = (int32_t)i;
      if (cand) {
        float4 r0, r1, r2;
        sh_record<D>(params, n_pad, i, cam, o, r0, r1, r2);
        rec[3 * i] = r0;
        rec[3 * i + 1] = r1;
        rec[3 * i + 2] = r2;
        rect[i] = o.rect;
        depth_key[i] = __float_as_uint(r2.w);
        const int64_t s = cam.TW + 1;
        atomicAdd(&diff[o.rect.y * s + o.rect.x], 1);
        atomicAdd(&diff[o.rect.y * s + o.rect.z], -1);
        atomicAdd(&diff[o.rect.w * s + o.rect.x], -1);
        atomicAdd(&diff[o.rect.w * s + o.rect.z], 1);
      } else {
        rec[3 * i] = make_float4(0.f, 0.f, 0.f, 0.f);
        rec[3 * i + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
        rec[3 * i + 2] = make_float4(0.f, 0.f, 0.f, -1.f);
        rect[i] = make_short4(0, 0, 0, 0);
        depth_key[i] = 0xffffffffu;
      }
      if (i == n - 1) *n_cand = (int32_t)n;
    }
    if (square_isect) {  // every lane of the warp takes part
      unsigned long long sq = counted ? (unsigned long long)o.square_tiles : 0ull;
      sq = warp_sum(sq);
      if ((threadIdx.x & 31) == 0 && sq) atomicAdd(square_isect, sq);
    }
    return;
  }
  // ordered compaction by warps: each warp publishes its candidate count,
  // forms its candidates' records (which do not depend on the slot), and
  // only then resolves its prefix from the warps before it (numbered by the
  // block ticket, so a warp waits only on warps that have started); no CTA
  // barrier, so a warp never waits for its block's slowest warp
  const unsigned lane = threadIdx.x & 31;
  const unsigned bal = __ballot_sync(0xffffffffu, cand);
  const int total = __popc(bal);
  const int rank = __popc(bal & ((1u << lane) - 1u));
  const int64_t wid = b * (kProjThreads / 32) + (threadIdx.x >> 5);
  lookback_publish(lb, wid, total);
  float4 r0, r1, r2;
  if (cand) sh_record<D>(params, n_pad, i, cam, o, r0, r1, r2);
  const int64_t prefix = lookback_resolve(lb, wid, total, dev_status);
  const int64_t slot = prefix + rank;
  const bool fits = slot < capacity;  // false beyond the caller's capacity (it retries)
  if (cand && !fits) dev_flag(dev_status, GS_DEV_BOUNDS);
  if (i < n) slot_map[i] = (cand && fits) ? (int32_t)slot : -1;
  if (cand && fits) {
    cand_idx[slot] = (int32_t)i;
    rec[3 * slot] = r0;
    rec[3 * slot + 1] = r1;
    rec[3 * slot + 2] = r2;
    rect[slot] = o.rect;
    depth_key[slot] = __float_as_uint(r2.w);
    const int64_t s = cam.TW + 1;
    atomicAdd(&diff[o.rect.y * s + o.rect.x], 1);
    atomicAdd(&diff[o.rect.y * s + o.rect.z], -1);
    atomicAdd(&diff[o.rect.w * s + o.rect.x], -1);
    atomicAdd(&diff[o.rect.w * s + o.rect.z], 1);
  }
  if (wid == n_blocks * (kProjThreads / 32) - 1 && lane == 0) *n_cand = (int32_t)(prefix + total);
  if (square_isect) {
    unsigned long long sq = counted ? (unsigned long long)o.square_tiles : 0ull;
    sq = warp_sum(sq);
    if ((threadIdx.x & 31) == 0 && sq) atomicAdd(square_isect, sq);
  }
}

// Double inclusive prefix along x of each row (y < TH, x < TW).
__global__ void __launch_bounds__(256)
k_sat_rows(const int32_t* __restrict__ diff, int64_t* __restrict__ tmp, int TW, int TH) {
  __shared__ long long s_scan[9];
  const int y = blockIdx.x;
  long long c1 = 0, c2 = 0;
  for (int x0 = 0; x0 < TW; x0 += 256) {
    const int x = x0 + threadIdx.x;
    long long v = x < TW ? (long long)diff[(int64_t)y * (TW + 1) + x] : 0;
    long long t;
    long long e1 = block_exclusive_scan<long long, 8>(v, s_scan, &t);
    long long s1 = c1 + e1 + v;
    c1 += t;
    long long e2 = block_exclusive_scan<long long, 8>(s1, s_scan, &t);
    long long s2 = c2 + e2 + s1;
    c2 += t;
    if (x < TW) tmp[(int64_t)y * TW + x] = s2;
  }
}

// Double inclusive prefix along y of each column, written with a one-cell
// zero border: sat[(y + 1) (TW + 1) + x + 1].
__global__ void __launch_bounds__(256)
k_sat_cols(const int64_t* __restrict__ tmp, int64_t* __restrict__ sat, int TW, int TH) {
  const int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x > TW) return;
  const int64_t s = TW + 1;
  if (x == TW) {  // the zero column
    for (int y = 0; y <= TH; ++y) sat[(int64_t)y * s] = 0;
    return;
  }
  sat[x + 1] = 0;
  long long c1 = 0, c2 = 0;
  for (int y = 0; y < TH; ++y) {
    c1 += tmp[(int64_t)y * TW + x];
    c2 += c1;
    sat[(int64_t)(y + 1) * s + x + 1] = c2;
  }
}

// Corners of each candidate's block rect (blocks of GS_TILE_BLOCK x
// GS_TILE_BLOCK tiles) into a difference grid; the count comes from the
// device (candidates written by the projection).  The grid is small and hot,
// so each CTA accumulates into a shared copy (SHARED) and adds its non-zero
// cells once.
template <bool SHARED>
__global__ void __launch_bounds__(256)
k_block_diff(const short4* __restrict__ rect, const int32_t* __restrict__ n_cand, int64_t cap,
             int BW, int cells, int32_t* __restrict__ diff) {
  extern __shared__ int32_t s_diff[];
  int32_t* d = SHARED ? s_diff : diff;
  if (SHARED) {
    for (int c = threadIdx.x; c < cells; c += 256) s_diff[c] = 0;
    __syncthreads();
  }
  const int64_t n = min((int64_t)*n_cand, cap);
  const int s = BW + 1;
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (int64_t)gridDim.x * 256) {
    const short4 r = rect[i];
    if (r.z <= r.x || r.w <= r.y) continue;  // a culled Gaussian of the dense layout
    const int bx0 = r.x / GS_TILE_BLOCK, by0 = r.y / GS_TILE_BLOCK;
    const int bx1 = (r.z - 1) / GS_TILE_BLOCK + 1, by1 = (r.w - 1) / GS_TILE_BLOCK + 1;
    atomicAdd(&d[by0 * s + bx0], 1);
    atomicAdd(&d[by0 * s + bx1], -1);
    atomicAdd(&d[by1 * s + bx0], -1);
    atomicAdd(&d[by1 * s + bx1], 1);
  }
  if (SHARED) {
    __syncthreads();
    for (int c = threadIdx.x; c < cells; c += 256)
      if (s_diff[c] != 0) atomicAdd(&diff[c], s_diff[c]);
  }
}

struct BlockWs {
  int32_t* diff;
  int64_t* tmp;
  size_t bytes;
};

BlockWs carve_block(void* ws, size_t cap, int64_t BW, int64_t BH) {
  Carver cv(ws, cap);
  BlockWs w;
  w.diff = cv.take<int32_t>((BW + 1) * (BH + 1));
  w.tmp = cv.take<int64_t>(BW * BH);
  w.bytes = cv.off;
  return w;
}

struct ProjWs {
  int32_t* diff;
  int64_t* tmp;
  unsigned long long* lb;
  unsigned int* ticket;
  size_t bytes;
};

ProjWs carve_proj(void* ws, size_t cap, int64_t n, int32_t W, int32_t H) {
  Carver cv(ws, cap);
  const int64_t TW = tiles_x(W), TH = tiles_y(H);
  const int64_t nb = (n + kProjThreads - 1) / kProjThreads;
  ProjWs p;
  p.ticket = cv.take<unsigned int>(64);
  p.lb = cv.take<unsigned long long>(nb > 0 ? nb * (kProjThreads / 32) : 1);  // per warp
  p.diff = cv.take<int32_t>((TW + 1) * (TH + 1));
  p.tmp = cv.take<int64_t>(TW * TH);
  p.bytes = cv.off;
  return p;
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" size_t gs_project_workspace_size(int64_t n, int32_t width, int32_t height) {
  if (n < 0 || width <= 0 || height <= 0) return 0;
  return carve_proj(nullptr, 0, n, width, height).bytes;
}

extern "C" gs_status gs_project(const gs_model* model, const gs_camera* cam, uint32_t flags,
                                const gs_proj* out, int64_t* tile_sat, void* ws, size_t ws_bytes,
                                int32_t* dev_status, gs_stream stream) {
  if (!cam || cam->width <= 0 || cam->height <= 0) return GS_ERR_ARG;
  const gs_rect all{0, 0, (int32_t)tiles_x(cam->width), (int32_t)tiles_y(cam->height)};
  return gs_project_region(model, cam, flags, all, out, tile_sat, ws, ws_bytes, dev_status,
                           stream);
}

extern "C" gs_status gs_project_region(const gs_model* model, const gs_camera* cam,
                                       uint32_t flags, gs_rect region, const gs_proj* out,
                                       int64_t* tile_sat, void* ws, size_t ws_bytes,
                                       int32_t* dev_status, gs_stream stream) {
  if (!model || !cam || !out || !tile_sat) return GS_ERR_ARG;
  if (flags & ~GS_PROJ_DENSE) return GS_ERR_UNSUPPORTED;
  const bool dense = (flags & GS_PROJ_DENSE) != 0;
  if (model->n < 0 || model->n_pad < model->n || (model->n_pad & 3) || model->sh_degree < 0 ||
      model->sh_degree > 3)
    return GS_ERR_ARG;
  if (cam->width <= 0 || cam->height <= 0 || !(cam->fx > 0) || !(cam->fy > 0)) return GS_ERR_ARG;
  const int64_t TW = tiles_x(cam->width), TH = tiles_y(cam->height);
  if (TW > 32767 || TH > 32767) return GS_ERR_UNSUPPORTED;
  if (out->capacity < 0 || !out->n_cand) return GS_ERR_ARG;
  if ((flags & GS_PROJ_DENSE) && out->capacity < model->n) return GS_ERR_ARG;
  if (model->n > 0 && (!model->params || !out->cand_idx || !out->slot || !out->rec || !out->rect ||
                       !out->depth_key))
    return GS_ERR_ARG;
  if (!aligned(out->rec, 16) || !aligned(out->rect, 8) || !aligned(ws, 256)) return GS_ERR_ARG;
  ProjWs w = carve_proj(ws, ws_bytes, model->n, cam->width, cam->height);
  if (w.bytes > ws_bytes || !ws) return GS_ERR_CAPACITY;
  cudaStream_t s = to_stream(stream);

  ProjCam pc;
  for (int k = 0; k < 9; ++k) pc.R[k] = (double)cam->R[k];
  for (int k = 0; k < 3; ++k) pc.t[k] = (double)cam->t[k];
  pc.fx = cam->fx; pc.fy = cam->fy; pc.cx = cam->cx; pc.cy = cam->cy;
  pc.limx = (1.3 * (0.5 * (double)cam->width)) / pc.fx;
  pc.limy = (1.3 * (0.5 * (double)cam->height)) / pc.fy;
  for (int c = 0; c < 3; ++c)
    pc.campos[c] = -(pc.R[c] * pc.t[0] + pc.R[3 + c] * pc.t[1] + pc.R[6 + c] * pc.t[2]);
  pc.W = cam->width; pc.H = cam->height; pc.TW = (int32_t)TW; pc.TH = (int32_t)TH;
  if (region.x0 < 0 || region.y0 < 0 || region.x1 <= region.x0 || region.y1 <= region.y0 ||
      region.x1 > TW || region.y1 > TH)
    return GS_ERR_ARG;
  pc.RX0 = region.x0; pc.RY0 = region.y0; pc.RX1 = region.x1; pc.RY1 = region.y1;

  const int64_t nb = (model->n + kProjThreads - 1) / kProjThreads;
  // ticket, look-back words and the difference grid start at zero
  const size_t zero_bytes = (size_t)((char*)(w.diff + (TW + 1) * (TH + 1)) - (char*)ws);
  GS_TRY(cudaMemsetAsync(ws, 0, zero_bytes, s));
  if (out->square_isect) GS_TRY(cudaMemsetAsync(out->square_isect, 0, sizeof(unsigned long long), s));
  if (nb > 0) {
#define GS_PROJ(DD)                                                                          \
  k_project<DD><<<(unsigned)nb, kProjThreads, 0, s>>>(                                       \
      model->params, model->n, model->n_pad, pc, out->cand_idx, out->slot,                   \
      reinterpret_cast<float4*>(out->rec), reinterpret_cast<short4*>(out->rect), out->depth_key, \
      w.diff, w.lb, w.ticket, out->n_cand, nb, out->capacity, out->square_isect, dense,     \
      aligned(model->params, 16), dev_status)
    switch (model->sh_degree) {
      case 0: GS_PROJ(0); break;
      case 1: GS_PROJ(1); break;
      case 2: GS_PROJ(2); break;
      default: GS_PROJ(3); break;
    }
#undef GS_PROJ
    GS_LAUNCH_CHECK();
  } else {
    GS_TRY(cudaMemsetAsync(out->n_cand, 0, sizeof(int32_t), s));
  }
  k_sat_rows<<<(unsigned)TH, 256, 0, s>>>(w.diff, w.tmp, (int)TW, (int)TH);
  GS_LAUNCH_CHECK();
  k_sat_cols<<<(unsigned)((TW + 1 + 255) / 256), 256, 0, s>>>(w.tmp, tile_sat, (int)TW, (int)TH);
  GS_LAUNCH_CHECK();
  return GS_OK;
}

extern "C" size_t gs_block_sat_workspace_size(int32_t TW, int32_t TH) {
  if (TW <= 0 || TH <= 0) return 0;
  return carve_block(nullptr, 0, (TW + GS_TILE_BLOCK - 1) / GS_TILE_BLOCK,
                     (TH + GS_TILE_BLOCK - 1) / GS_TILE_BLOCK)
      .bytes;
}

extern "C" gs_status gs_block_sat(const gs_proj* proj, int32_t TW, int32_t TH, int64_t* block_sat,
                                  void* ws, size_t ws_bytes, int32_t* dev_status,
                                  gs_stream stream) {
  (void)dev_status;
  if (!proj || !proj->n_cand || !block_sat || TW <= 0 || TH <= 0 || TW > 32767 || TH > 32767)
    return GS_ERR_ARG;
  if (proj->capacity > 0 && !proj->rect) return GS_ERR_ARG;
  if (!aligned(proj->rect, 8) || !aligned(ws, 256)) return GS_ERR_ARG;
  const int64_t BW = (TW + GS_TILE_BLOCK - 1) / GS_TILE_BLOCK;
  const int64_t BH = (TH + GS_TILE_BLOCK - 1) / GS_TILE_BLOCK;
  BlockWs w = carve_block(ws, ws_bytes, BW, BH);
  if (!ws || w.bytes > ws_bytes) return GS_ERR_CAPACITY;
  cudaStream_t s = to_stream(stream);
  GS_TRY(cudaMemsetAsync(w.diff, 0, sizeof(int32_t) * (BW + 1) * (BH + 1), s));
  if (proj->capacity > 0) {
    const int64_t want = (proj->capacity + 255) / 256;
    const int cells = (int)((BW + 1) * (BH + 1));
    const short4* r4 = reinterpret_cast<const short4*>(proj->rect);
    if (cells <= 12 * 1024) {  // 48 KB of shared counters
      // one wave of CTAs, each taking a long strided share of the candidates
      const unsigned nb = (unsigned)(want < 148 * 2 ? want : 148 * 2);
      k_block_diff<true><<<nb, 256, cells * sizeof(int32_t), s>>>(r4, proj->n_cand,
                                                                 proj->capacity, (int)BW, cells,
                                                                 w.diff);
    } else {
      k_block_diff<false><<<(unsigned)(want < 148 * 8 ? want : 148 * 8), 256, 0, s>>>(
          r4, proj->n_cand, proj->capacity, (int)BW, cells, w.diff);
    }
    GS_LAUNCH_CHECK();
  }
  k_sat_rows<<<(unsigned)BH, 256, 0, s>>>(w.diff, w.tmp, (int)BW, (int)BH);
  GS_LAUNCH_CHECK();
  k_sat_cols<<<(unsigned)((BW + 1 + 255) / 256), 256, 0, s>>>(w.tmp, block_sat, (int)BW, (int)BH);
  GS_LAUNCH_CHECK();
  return GS_OK;
}
