// SSIM term of the composite photometric loss (1 - lambda) L1 + lambda (1 - SSIM)
// (SkipGS paper notes, "loss function / training strategy"), with windows local
// to each Leaf's pixel rectangle (BoundedGS page, section 02: local SSIM windows
// differ from full-image ones at their boundary).  SSIM is the structural
// similarity of Wang, Bovik, Sheikh and Simoncelli (IEEE TIP 2004) with its
// 11 x 11 Gaussian window (sigma 1.5) and C1 = 0.01^2, C2 = 0.03^2.
//
// Two launches over the Leaf's tiles, one CTA per 16 x 16 tile:
//  k_ssim_stats: x = render, y = target staged with a 5-pixel halo (zero outside
//    the Leaf's rectangle R); separable window sums (rows, then columns) of x, y,
//    x^2, y^2, x y; per pixel S, the tile's sum of (1 - S), and the partials of S
//    in the three window sums that depend on x (W[x], W[x^2], W[x y]).
//  k_ssim_grad: the window sums of those partials (columns, then rows; the
//    window is symmetric and zero outside R, so the transposed sum is the
//    window sum) combine into
//    d S_sum / dx_p = W[dS/dm](p) + 2 x_p W[dS/de](p) + y_p W[dS/df](p).
// Both stages keep their inputs in registers along a row or a column (each
// thread produces 8 or 16 outputs from 18 or 26 staged values), so shared
// memory traffic stays well below one access per multiply-add.
#include <algorithm>
#include <cmath>

#include "gs_internal.cuh"

namespace gs {
namespace {

constexpr int kR = 5;                   // window radius
constexpr int kN = 2 * kR + 1;          // 11 taps
constexpr int kE = kTile + 2 * kR;      // 26: tile plus halo
constexpr int kXP = kE + 1;             // staged row pitch
constexpr int kHP = kTile + 1;          // row-sum pitch
constexpr float kC1 = 0.01f * 0.01f;
constexpr float kC2 = 0.03f * 0.03f;

struct SsimArgs {
  int X0, Y0, X1, Y1;   // the Leaf's pixel rectangle R (clipped to the image)
  int lx0, ly0, lw;     // the Leaf's first tile and its width in tiles
  int TW;               // tiles per image row (loss tile index)
  int ix0, iy0;         // origin of the render / dL buffers
  int64_t ipitch, iplane;
  const float* img;
  float* dL;
  int tx0, ty0;         // origin of the target buffer
  int64_t tpitch, tplane;
  const float* target;
  float* loss_tiles;
  float* ws;            // [9][Rh][Rw]: (dS/dm, dS/de, dS/df) per channel, or null
  int64_t wpitch, wplane;
  float weight;
  float g[kN];          // the normalised 1D window
};

__device__ __forceinline__ bool in_rect(const SsimArgs& a, int x, int y) {
  return x >= a.X0 && x < a.X1 && y >= a.Y0 && y < a.Y1;
}

__global__ void __launch_bounds__(256, 4) k_ssim_stats(SsimArgs a) {
  __shared__ float s_in[2][3][kE][kXP];     // x, y of the tile and its halo
  __shared__ float s_h[3][5][kE][kHP];      // row sums of x, y, x^2, y^2, xy
  __shared__ float s_red[8];
  // column sums reuse the staging area once the row sums are done
  float(*s_v)[5][kTile][kHP] = reinterpret_cast<float(*)[5][kTile][kHP]>(&s_in[0][0][0][0]);
  static_assert(3 * 5 * kTile * kHP <= 2 * 3 * kE * kXP, "column sums must fit the staging area");

  const int t = threadIdx.x;
  const int tx = a.lx0 + blockIdx.x % a.lw, ty = a.ly0 + blockIdx.x / a.lw;
  const int ox = tx * kTile - kR, oy = ty * kTile - kR;

  // staging: warp w takes rows w, w + 8, ...; lane = column of the halo tile
  {
    const int lane = t & 31, gx = ox + lane;
    const bool colok = lane < kE && gx >= a.X0 && gx < a.X1;
    for (int r = t >> 5; r < kE; r += 8) {
      const int gy = oy + r;
      float xv[3] = {0.0f, 0.0f, 0.0f}, yv[3] = {0.0f, 0.0f, 0.0f};
      if (colok && gy >= a.Y0 && gy < a.Y1) {
        const float* xp = a.img + (int64_t)(gy - a.iy0) * a.ipitch + (gx - a.ix0);
        const float* yp = a.target + (int64_t)(gy - a.ty0) * a.tpitch + (gx - a.tx0);
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          xv[c] = xp[c * a.iplane];
          yv[c] = yp[c * a.tplane];
        }
      }
      if (lane < kE) {
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          s_in[0][c][r][lane] = xv[c];
          s_in[1][c][r][lane] = yv[c];
        }
      }
    }
  }
  __syncthreads();

  // rows: thread (c, r, half) -> 8 outputs of the five sums from 18 inputs,
  // consumed input by input so only the accumulators stay live
  if (t < 3 * kE * 2) {
    const int c = t / (2 * kE), r = (t >> 1) % kE, hf = t & 1;
    const float* xr = &s_in[0][c][r][hf * 8];
    const float* yr = &s_in[1][c][r][hf * 8];
    float mx[8], my[8], ex[8], ey[8], fx[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) mx[j] = my[j] = ex[j] = ey[j] = fx[j] = 0.0f;
#pragma unroll
    for (int k = 0; k < 8 + 2 * kR; ++k) {
      const float x = xr[k], y = yr[k];
      const float xx = x * x, yy = y * y, xy = x * y;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int tap = k - j;
        if (tap >= 0 && tap < kN) {
          const float w = a.g[tap];
          mx[j] = fmaf(w, x, mx[j]);
          my[j] = fmaf(w, y, my[j]);
          ex[j] = fmaf(w, xx, ex[j]);
          ey[j] = fmaf(w, yy, ey[j]);
          fx[j] = fmaf(w, xy, fx[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int col = hf * 8 + j;
      s_h[c][0][r][col] = mx[j];
      s_h[c][1][r][col] = my[j];
      s_h[c][2][r][col] = ex[j];
      s_h[c][3][r][col] = ey[j];
      s_h[c][4][r][col] = fx[j];
    }
  }
  __syncthreads();

  // columns: thread (c, map, col) -> 16 outputs from 26 row sums
  if (t < 3 * 5 * kTile) {
    const int col = t & 15, cm = t >> 4, c = cm / 5, mp = cm % 5;
    float acc[kTile];
#pragma unroll
    for (int i = 0; i < kTile; ++i) acc[i] = 0.0f;
#pragma unroll
    for (int k = 0; k < kE; ++k) {
      const float v = s_h[c][mp][k][col];
#pragma unroll
      for (int i = 0; i < kTile; ++i) {
        const int tap = k - i;
        if (tap >= 0 && tap < kN) acc[i] = fmaf(a.g[tap], v, acc[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < kTile; ++i) s_v[c][mp][i][col] = acc[i];
  }
  __syncthreads();

  const int px = t & 15, py = t >> 4;
  const int gx = tx * kTile + px, gy = ty * kTile + py;
  const bool inside = in_rect(a, gx, gy);
  const int64_t o = (int64_t)(gy - a.Y0) * a.wpitch + (gx - a.X0);
  float lsum = 0.0f;
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    const float m1 = s_v[c][0][py][px], m2 = s_v[c][1][py][px];
    const float vx = s_v[c][2][py][px] - m1 * m1;
    const float vy = s_v[c][3][py][px] - m2 * m2;
    const float cxy = s_v[c][4][py][px] - m1 * m2;
    const float A = 2.0f * m1 * m2 + kC1;
    const float Bc = 2.0f * cxy + kC2;
    const float Cc = m1 * m1 + m2 * m2 + kC1;
    const float D = vx + vy + kC2;
    const float inv = 1.0f / (Cc * D);
    const float S = A * Bc * inv;
    if (inside) {
      lsum += 1.0f - S;
      if (a.ws) {
        // partials of S = A B / (C D) in W[x], W[x^2], W[x y] (sigma terms
        // expanded), written with the one reciprocal 1 / (C D)
        const float dm = (2.0f * m2 * (Bc - A) + 2.0f * m1 * S * (Cc - D)) * inv;
        const float de = -S * Cc * inv;
        const float df = 2.0f * A * inv;
        a.ws[(3 * c + 0) * a.wplane + o] = dm;
        a.ws[(3 * c + 1) * a.wplane + o] = de;
        a.ws[(3 * c + 2) * a.wplane + o] = df;
      }
    }
  }
  lsum = warp_sum(lsum);
  if ((t & 31) == 0) s_red[t >> 5] = lsum;
  __syncthreads();
  if (t == 0) {
    float tot = 0.0f;
    for (int w = 0; w < 8; ++w) tot += s_red[w];
    a.loss_tiles[(int64_t)ty * a.TW + tx] += a.weight * tot;
  }
}

constexpr int kGradIn = 9 * kE * kXP;       // staged partials with halo
constexpr int kGradCol = 9 * kTile * kXP;    // their column sums (16 rows x 26)
constexpr int kGradSmem = (kGradIn + kGradCol) * 4;

__global__ void __launch_bounds__(256) k_ssim_grad(SsimArgs a) {
  extern __shared__ float smem[];
  float(*s_p)[kE][kXP] = reinterpret_cast<float(*)[kE][kXP]>(smem);
  float(*s_c)[kTile][kXP] = reinterpret_cast<float(*)[kTile][kXP]>(smem + kGradIn);
  float(*s_v)[kTile][kHP] = reinterpret_cast<float(*)[kTile][kHP]>(smem);
  static_assert(9 * kTile * kHP <= kGradIn, "window sums must fit the staging area");

  const int t = threadIdx.x;
  const int tx = a.lx0 + blockIdx.x % a.lw, ty = a.ly0 + blockIdx.x / a.lw;
  const int ox = tx * kTile - kR, oy = ty * kTile - kR;

  {
    const int lane = t & 31, gx = ox + lane;
    const bool colok = lane < kE && gx >= a.X0 && gx < a.X1;
    for (int r = t >> 5; r < kE; r += 8) {
      const int gy = oy + r;
      float v[9];
#pragma unroll
      for (int p = 0; p < 9; ++p) v[p] = 0.0f;
      if (colok && gy >= a.Y0 && gy < a.Y1) {
        const float* wp = a.ws + (int64_t)(gy - a.Y0) * a.wpitch + (gx - a.X0);
#pragma unroll
        for (int p = 0; p < 9; ++p) v[p] = wp[p * a.wplane];
      }
      if (lane < kE) {
#pragma unroll
        for (int p = 0; p < 9; ++p) s_p[p][r][lane] = v[p];
      }
    }
  }
  __syncthreads();

  // columns first: thread (plane, col of 26) -> 16 outputs from 26 inputs
  if (t < 9 * kE) {
    const int p = t / kE, col = t % kE;
    float acc[kTile];
#pragma unroll
    for (int i = 0; i < kTile; ++i) acc[i] = 0.0f;
#pragma unroll
    for (int k = 0; k < kE; ++k) {
      const float v = s_p[p][k][col];
#pragma unroll
      for (int i = 0; i < kTile; ++i) {
        const int tap = k - i;
        if (tap >= 0 && tap < kN) acc[i] = fmaf(a.g[tap], v, acc[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < kTile; ++i) s_c[p][i][col] = acc[i];
  }
  __syncthreads();

  // rows: thread (plane, row) -> 16 outputs from 26 column sums
  if (t < 9 * kTile) {
    const int p = t >> 4, r = t & 15;
    const float* row = &s_c[p][r][0];
    float acc[kTile];
#pragma unroll
    for (int j = 0; j < kTile; ++j) acc[j] = 0.0f;
#pragma unroll
    for (int k = 0; k < kE; ++k) {
      const float v = row[k];
#pragma unroll
      for (int j = 0; j < kTile; ++j) {
        const int tap = k - j;
        if (tap >= 0 && tap < kN) acc[j] = fmaf(a.g[tap], v, acc[j]);
      }
    }
#pragma unroll
    for (int j = 0; j < kTile; ++j) s_v[p][r][j] = acc[j];
  }
  __syncthreads();

  const int px = t & 15, py = t >> 4;
  const int gx = tx * kTile + px, gy = ty * kTile + py;
  if (!in_rect(a, gx, gy)) return;
  const int64_t oi = (int64_t)(gy - a.iy0) * a.ipitch + (gx - a.ix0);
  const int64_t ot = (int64_t)(gy - a.ty0) * a.tpitch + (gx - a.tx0);
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    const float x = a.img[oi + c * a.iplane], y = a.target[ot + c * a.tplane];
    const float gS = s_v[3 * c][py][px] + 2.0f * x * s_v[3 * c + 1][py][px] + y * s_v[3 * c + 2][py][px];
    a.dL[oi + c * a.iplane] -= a.weight * gS;
  }
}

std::atomic<unsigned long long> g_grad_attr{0};

struct LeafRect {
  int X0, Y0, X1, Y1;
};

bool leaf_rect(gs_rect leaf, const gs_camera* cam, LeafRect* r) {
  if (!cam || leaf.x0 < 0 || leaf.y0 < 0 || leaf.x1 <= leaf.x0 || leaf.y1 <= leaf.y0 ||
      leaf.x1 > tiles_x(cam->width) || leaf.y1 > tiles_y(cam->height))
    return false;
  r->X0 = leaf.x0 * kTile;
  r->Y0 = leaf.y0 * kTile;
  r->X1 = std::min<int>(leaf.x1 * kTile, cam->width);
  r->Y1 = std::min<int>(leaf.y1 * kTile, cam->height);
  return true;
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" size_t gs_ssim_workspace_size(gs_rect leaf, const gs_camera* cam) {
  LeafRect r;
  if (!leaf_rect(leaf, cam, &r)) return 0;
  return (size_t)9 * (size_t)(r.X1 - r.X0) * (size_t)(r.Y1 - r.Y0) * sizeof(float);
}

extern "C" gs_status gs_loss_ssim(const gs_pixels* px, gs_rect leaf, const gs_camera* cam,
                                  double weight, void* ws, size_t ws_bytes, gs_stream stream) {
  LeafRect r;
  if (!px || !leaf_rect(leaf, cam, &r)) return GS_ERR_ARG;
  if (!px->img || !px->target || !px->loss_tiles || (ws && !px->dL_dimg)) return GS_ERR_ARG;
  // the render, dL and target buffers must cover R
  if (r.X0 < px->x0 || r.Y0 < px->y0 || r.X1 > (int64_t)px->x0 + px->w ||
      r.Y1 > (int64_t)px->y0 + px->h || px->pitch < px->w || px->plane < px->pitch * (int64_t)px->h)
    return GS_ERR_ARG;
  if (r.X0 < px->tx0 || r.Y0 < px->ty0 || px->tpitch < r.X1 - px->tx0 ||
      px->tplane < px->tpitch * (int64_t)(r.Y1 - px->ty0))
    return GS_ERR_ARG;
  if (ws && (!aligned(ws, 16) || ws_bytes < gs_ssim_workspace_size(leaf, cam))) return GS_ERR_ARG;

  SsimArgs a;
  a.X0 = r.X0; a.Y0 = r.Y0; a.X1 = r.X1; a.Y1 = r.Y1;
  a.lx0 = leaf.x0; a.ly0 = leaf.y0; a.lw = leaf.x1 - leaf.x0;
  a.TW = (int)tiles_x(cam->width);
  a.ix0 = px->x0; a.iy0 = px->y0; a.ipitch = px->pitch; a.iplane = px->plane;
  a.img = px->img; a.dL = px->dL_dimg;
  a.tx0 = px->tx0; a.ty0 = px->ty0; a.tpitch = px->tpitch; a.tplane = px->tplane;
  a.target = px->target;
  a.loss_tiles = px->loss_tiles;
  a.ws = static_cast<float*>(ws);
  a.wpitch = r.X1 - r.X0;
  a.wplane = a.wpitch * (r.Y1 - r.Y0);
  a.weight = (float)weight;
  // the window in fp64, rounded once to fp32
  double g[kN], sum = 0.0;
  for (int k = 0; k < kN; ++k) {
    const double d = k - kR;
    g[k] = std::exp(-d * d / (2.0 * 1.5 * 1.5));
    sum += g[k];
  }
  for (int k = 0; k < kN; ++k) a.g[k] = (float)(g[k] / sum);

  const unsigned nb = (unsigned)((int64_t)(leaf.x1 - leaf.x0) * (leaf.y1 - leaf.y0));
  cudaStream_t s = to_stream(stream);
  k_ssim_stats<<<nb, 256, 0, s>>>(a);
  GS_LAUNCH_CHECK();
  if (ws) {
    GS_TRY(smem_attrs_once(reinterpret_cast<const void*>(&k_ssim_grad), kGradSmem, &g_grad_attr));
    k_ssim_grad<<<nb, 256, kGradSmem, s>>>(a);
    GS_LAUNCH_CHECK();
  }
  return GS_OK;
}
