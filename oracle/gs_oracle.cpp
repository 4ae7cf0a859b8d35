// CPU oracle for one 3D Gaussian Splatting training step.
//
// TEST INFRASTRUCTURE ONLY: called by the tests, the smoke check and the
// CPU-baseline leg of the benchmark, never by the product path.  It shares
// no code, header or constant table with the CUDA library.
//
// Sources.  The stages are the ones the SkipGS paper notes name for the
// tile-based differentiable rasteriser ("SkipGS: Post-Densification Backward
// Skipping for Efficient 3DGS Training", sections "research background" and
// "loss function / training strategy": differentiable rasterisation of
// anisotropic 3D Gaussians, gradients flowing back through the projected 2D
// covariance and the transmittance accumulation to means, quaternions,
// scales, opacities and SH coefficients; section "key design 2": the
// backward is gradient back-propagation, atomic accumulation and coordinate /
// covariance differentiation).  The memory scheme (two-stage backward,
// load-budgeted Leaves, candidate-only projection, compact gradients) is
// from the BoundedGS project page ("BoundedGS", sections 01 and 02).  The
// numeric constants of the rasteriser (0.3 px^2 low-pass, 3-sigma radius,
// alpha = min(0.99, o exp(-q)), skip below 1/255, stop when T < 1e-4, near
// plane 0.2, guard band 1.3) are the plain 3DGS choices; the pages give
// none of them, so each is a stated reading.
//
// Precision: fp64 throughout.  Where a floating-point value decides an
// integer (cull, tile rect, depth key) the expression is evaluated in fp64
// in the exact order written below with no contraction (built with
// -ffp-contract=off), and the fp32 depth key is the correctly rounded fp32
// of the fp64 depth.

#include "gs_oracle.h"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <numeric>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

constexpr double kPi = 3.14159265358979323846;
constexpr int kTile = 16;

struct Cam {
  double R[9], t[3], fx, fy, cx, cy;
};

Cam load_cam(const double* c) {
  Cam k;
  for (int i = 0; i < 9; ++i) k.R[i] = c[i];
  for (int i = 0; i < 3; ++i) k.t[i] = c[9 + i];
  k.fx = c[12]; k.fy = c[13]; k.cx = c[14]; k.cy = c[15];
  return k;
}

inline int64_t floor_div_tile(double x) { return (int64_t)std::floor(x / kTile); }

inline int64_t clampi(int64_t x, int64_t lo, int64_t hi) {
  return x < lo ? lo : (x > hi ? hi : x);
}

// Real spherical harmonics up to degree 3 (orthonormal on the unit sphere,
// Condon-Shortley phase), ordered m = -l .. l within each band, written as
// homogeneous polynomials of the unit direction (x, y, z) with their
// textbook normalisations.
void sh_eval(double x, double y, double z, double* Y, double* dY) {
  const double c0 = 0.5 / std::sqrt(kPi);
  const double c1 = std::sqrt(3.0 / (4.0 * kPi));
  const double c2a = 0.5 * std::sqrt(15.0 / kPi);
  const double c2b = 0.25 * std::sqrt(5.0 / kPi);
  const double c2c = 0.25 * std::sqrt(15.0 / kPi);
  const double c3a = 0.25 * std::sqrt(35.0 / (2.0 * kPi));
  const double c3b = 0.5 * std::sqrt(105.0 / kPi);
  const double c3c = 0.25 * std::sqrt(21.0 / (2.0 * kPi));
  const double c3d = 0.25 * std::sqrt(7.0 / kPi);
  const double c3e = 0.25 * std::sqrt(105.0 / kPi);
  double xx = x * x, yy = y * y, zz = z * z;
  Y[0] = c0;
  Y[1] = -c1 * y;
  Y[2] = c1 * z;
  Y[3] = -c1 * x;
  Y[4] = c2a * x * y;
  Y[5] = -c2a * y * z;
  Y[6] = c2b * (2 * zz - xx - yy);
  Y[7] = -c2a * x * z;
  Y[8] = c2c * (xx - yy);
  Y[9] = -c3a * y * (3 * xx - yy);
  Y[10] = c3b * x * y * z;
  Y[11] = -c3c * y * (4 * zz - xx - yy);
  Y[12] = c3d * z * (2 * zz - 3 * xx - 3 * yy);
  Y[13] = -c3c * x * (4 * zz - xx - yy);
  Y[14] = c3e * z * (xx - yy);
  Y[15] = -c3a * x * (xx - 3 * yy);
  if (!dY) return;
  auto set = [&](int k, double gx, double gy, double gz) {
    dY[3 * k] = gx; dY[3 * k + 1] = gy; dY[3 * k + 2] = gz;
  };
  set(0, 0, 0, 0);
  set(1, 0, -c1, 0);
  set(2, 0, 0, c1);
  set(3, -c1, 0, 0);
  set(4, c2a * y, c2a * x, 0);
  set(5, 0, -c2a * z, -c2a * y);
  set(6, -2 * c2b * x, -2 * c2b * y, 4 * c2b * z);
  set(7, -c2a * z, 0, -c2a * x);
  set(8, 2 * c2c * x, -2 * c2c * y, 0);
  set(9, -c3a * 6 * x * y, -c3a * (3 * xx - 3 * yy), 0);
  set(10, c3b * y * z, c3b * x * z, c3b * x * y);
  set(11, c3c * 2 * x * y, -c3c * (4 * zz - xx - 3 * yy), -c3c * 8 * y * z);
  set(12, -c3d * 6 * x * z, -c3d * 6 * y * z, c3d * (6 * zz - 3 * xx - 3 * yy));
  set(13, -c3c * (4 * zz - 3 * xx - yy), c3c * 2 * x * y, -c3c * 8 * x * z);
  set(14, c3e * 2 * x * z, -c3e * 2 * y * z, c3e * (xx - yy));
  set(15, -c3a * (3 * xx - 3 * yy), c3a * 6 * x * y, 0);
}

// Rotation matrix (row-major) of a unit quaternion (w, x, y, z).
void quat_to_R(const double q[4], double R[9]) {
  double w = q[0], x = q[1], y = q[2], z = q[3];
  R[0] = 1 - 2 * (y * y + z * z); R[1] = 2 * (x * y - w * z); R[2] = 2 * (x * z + w * y);
  R[3] = 2 * (x * y + w * z); R[4] = 1 - 2 * (x * x + z * z); R[5] = 2 * (y * z - w * x);
  R[6] = 2 * (x * z - w * y); R[7] = 2 * (y * z + w * x); R[8] = 1 - 2 * (x * x + y * y);
}

// dR[k][i] = d R_k / d q_i for the matrix above (k = 0..8, i = w,x,y,z).
void quat_to_R_jac(const double q[4], double dR[9][4]) {
  double w = q[0], x = q[1], y = q[2], z = q[3];
  double t[9][4] = {
      {0, 0, -4 * y, -4 * z},
      {-2 * z, 2 * y, 2 * x, -2 * w},
      {2 * y, 2 * z, 2 * w, 2 * x},
      {2 * z, 2 * y, 2 * x, 2 * w},
      {0, -4 * x, 0, -4 * z},
      {-2 * x, -2 * w, 2 * z, 2 * y},
      {-2 * y, 2 * z, -2 * w, 2 * x},
      {2 * x, 2 * w, 2 * z, 2 * y},
      {0, -4 * x, -4 * y, 0}};
  std::memcpy(dR, t, sizeof t);
}

struct Forward3D {
  // all the intermediates of one Gaussian's projection
  double mean[3], tcam[3], xn, yn, u, v;
  double qn[4], qnorm, Rq[9], s[3], M[9], Sigma[9];
  double J[6], T[6], S2[3], S2p[3], det, conic[3];
  double radius;
  int64_t rect[4];
  int64_t square_tiles;
  double dir[3], dnorm, rgb_raw[3], rgb[3], opac;
  bool cand;
  uint8_t flags;
};

// Cull + EWA projection of Gaussian i (cull rules and constants: readings).
// `tight` selects the rect: the tiles of the 3-sigma square that meet the
// alpha >= 1/255 box (the library's binning), or the plain square.
void project_one(const double* params, int64_t n_pad, int32_t D, const Cam& k,
                 int32_t W, int32_t H, int64_t i, Forward3D& f, bool tight) {
  const int TW = (W + kTile - 1) / kTile, TH = (H + kTile - 1) / kTile;
  auto P = [&](int plane) { return params[(int64_t)plane * n_pad + i]; };
  f.cand = false;
  f.flags = 0;
  for (int j = 0; j < 3; ++j) f.mean[j] = P(j);
  double x = f.mean[0], y = f.mean[1], z = f.mean[2];
  // camera coordinates, fixed summation order
  for (int r = 0; r < 3; ++r)
    f.tcam[r] = ((k.R[3 * r] * x + k.R[3 * r + 1] * y) + k.R[3 * r + 2] * z) + k.t[r];
  double tz = f.tcam[2];
  for (int j = 0; j < 11; ++j)
    if (!std::isfinite(P(j))) { f.flags |= OR_F_NONFINITE; return; }
  if (!(tz > 0.2)) return;                       // near plane
  f.xn = f.tcam[0] / tz;
  f.yn = f.tcam[1] / tz;
  double limx = (1.3 * (0.5 * (double)W)) / k.fx;
  double limy = (1.3 * (0.5 * (double)H)) / k.fy;
  if (std::fabs(f.xn) > limx || std::fabs(f.yn) > limy) return;  // guard band
  f.u = k.fx * f.xn + k.cx;
  f.v = k.fy * f.yn + k.cy;
  // 3D covariance Sigma = R S S^T R^T from the normalised quaternion
  double q[4] = {P(6), P(7), P(8), P(9)};
  f.qnorm = std::sqrt(q[0] * q[0] + q[1] * q[1] + q[2] * q[2] + q[3] * q[3]);
  if (!(f.qnorm > 0)) { f.flags |= OR_F_NONFINITE; return; }
  for (int j = 0; j < 4; ++j) f.qn[j] = q[j] / f.qnorm;
  quat_to_R(f.qn, f.Rq);
  for (int j = 0; j < 3; ++j) f.s[j] = std::exp(P(3 + j));
  for (int r = 0; r < 3; ++r)
    for (int c = 0; c < 3; ++c) f.M[3 * r + c] = f.Rq[3 * r + c] * f.s[c];
  for (int r = 0; r < 3; ++r)
    for (int c = 0; c < 3; ++c) {
      double acc = 0;
      for (int j = 0; j < 3; ++j) acc += f.M[3 * r + j] * f.M[3 * c + j];
      f.Sigma[3 * r + c] = acc;
    }
  // Jacobian of the perspective projection at t, then T = J W
  f.J[0] = k.fx / tz; f.J[1] = 0; f.J[2] = -k.fx * f.xn / tz;
  f.J[3] = 0; f.J[4] = k.fy / tz; f.J[5] = -k.fy * f.yn / tz;
  for (int r = 0; r < 2; ++r)
    for (int c = 0; c < 3; ++c) {
      double acc = 0;
      for (int j = 0; j < 3; ++j) acc += f.J[3 * r + j] * k.R[3 * j + c];
      f.T[3 * r + c] = acc;
    }
  // 2D covariance T Sigma T^T, plus the 0.3 px^2 low-pass on the diagonal
  double TS[6];
  for (int r = 0; r < 2; ++r)
    for (int c = 0; c < 3; ++c) {
      double acc = 0;
      for (int j = 0; j < 3; ++j) acc += f.T[3 * r + j] * f.Sigma[3 * j + c];
      TS[3 * r + c] = acc;
    }
  double s2[4];
  for (int r = 0; r < 2; ++r)
    for (int c = 0; c < 2; ++c) {
      double acc = 0;
      for (int j = 0; j < 3; ++j) acc += TS[3 * r + j] * f.T[3 * c + j];
      s2[2 * r + c] = acc;
    }
  f.S2[0] = s2[0]; f.S2[1] = 0.5 * (s2[1] + s2[2]); f.S2[2] = s2[3];
  f.S2p[0] = f.S2[0] + 0.3; f.S2p[1] = f.S2[1]; f.S2p[2] = f.S2[2] + 0.3;
  f.det = f.S2p[0] * f.S2p[2] - f.S2p[1] * f.S2p[1];
  if (!(f.det > 0)) return;
  f.conic[0] = f.S2p[2] / f.det;
  f.conic[1] = -f.S2p[1] / f.det;
  f.conic[2] = f.S2p[0] / f.det;
  double mid = 0.5 * (f.S2p[0] + f.S2p[2]);
  double lam = mid + std::sqrt(std::max(0.1, mid * mid - f.det));
  double r3 = 3.0 * std::sqrt(lam);
  f.radius = std::ceil(r3);
  if (std::fabs(r3 - std::nearbyint(r3)) <= 1e-9 * r3) f.flags |= OR_F_RADIUS_NEAR;
  // tiles covered by the closed square [u-r, u+r] x [v-r, v+r] ...
  int64_t sq[4] = {floor_div_tile(f.u - f.radius), floor_div_tile(f.v - f.radius),
                   floor_div_tile(f.u + f.radius) + 1, floor_div_tile(f.v + f.radius) + 1};
  f.square_tiles = (clampi(sq[2], 0, TW) - clampi(sq[0], 0, TW)) *
                   (clampi(sq[3], 0, TH) - clampi(sq[1], 0, TH));
  // ... restricted to the tiles whose pixel-centre box (16 t + 0.5 .. 16 t
  // + 15.5) meets the bounding box of {alpha >= 1/255} = {q <= ln(255 o)},
  // inflated (1e-4 relative + 1e-4 in q, 0.01 px) beyond fp32 rounding.
  // Reading: a tile outside it would skip the Gaussian at every pixel, so
  // the image and gradients are those of the plain square.
  f.opac = 1.0 / (1.0 + std::exp(-P(10)));
  if (tight) {
    double lq = std::log(255.0 * f.opac);
    if (std::fabs(lq + 1e-4) <= 1e-9) f.flags |= OR_F_RADIUS_NEAR;
    if (!(lq > -1e-4)) return;  // alpha never reaches 1/255
    double qb = std::max(lq, 0.0) * 1.0001 + 1e-4;
    double hx = std::sqrt(2.0 * qb * f.S2p[0]) + 0.01;
    double hy = std::sqrt(2.0 * qb * f.S2p[2]) + 0.01;
    double e[4] = {(f.u - hx - 15.5) / kTile, (f.v - hy - 15.5) / kTile,
                   (f.u + hx - 0.5) / kTile, (f.v + hy - 0.5) / kTile};
    for (double x : e)
      if (std::fabs(x - std::nearbyint(x)) <= 1e-9 * std::max(1.0, std::fabs(x)))
        f.flags |= OR_F_RADIUS_NEAR;
    int64_t bb[4] = {(int64_t)std::ceil(e[0]), (int64_t)std::ceil(e[1]),
                     (int64_t)std::floor(e[2]) + 1, (int64_t)std::floor(e[3]) + 1};
    f.rect[0] = clampi(std::max(sq[0], bb[0]), 0, TW);
    f.rect[1] = clampi(std::max(sq[1], bb[1]), 0, TH);
    f.rect[2] = clampi(std::min(sq[2], bb[2]), 0, TW);
    f.rect[3] = clampi(std::min(sq[3], bb[3]), 0, TH);
  } else {
    // the plain closed 3-sigma square, clamped to the grid
    f.rect[0] = clampi(sq[0], 0, TW);
    f.rect[1] = clampi(sq[1], 0, TH);
    f.rect[2] = clampi(sq[2], 0, TW);
    f.rect[3] = clampi(sq[3], 0, TH);
  }
  if (f.rect[0] >= f.rect[2] || f.rect[1] >= f.rect[3]) return;
  // view-dependent colour from SH at the direction camera centre -> mean
  double cc[3];
  for (int c = 0; c < 3; ++c)
    cc[c] = -(k.R[c] * k.t[0] + k.R[3 + c] * k.t[1] + k.R[6 + c] * k.t[2]);
  for (int j = 0; j < 3; ++j) f.dir[j] = f.mean[j] - cc[j];
  f.dnorm = std::sqrt(f.dir[0] * f.dir[0] + f.dir[1] * f.dir[1] + f.dir[2] * f.dir[2]);
  double d[3] = {f.dir[0] / f.dnorm, f.dir[1] / f.dnorm, f.dir[2] / f.dnorm};
  double Y[16];
  sh_eval(d[0], d[1], d[2], Y, nullptr);
  int ksh = (D + 1) * (D + 1);
  for (int ch = 0; ch < 3; ++ch) {
    double acc = 0;
    for (int kk = 0; kk < ksh; ++kk) acc += P(11 + 3 * kk + ch) * Y[kk];
    f.rgb_raw[ch] = acc + 0.5;
    f.rgb[ch] = f.rgb_raw[ch] < 0 ? 0.0 : f.rgb_raw[ch];
    if (std::fabs(f.rgb_raw[ch]) <= 1e-9) f.flags |= OR_F_CLAMP_NEAR;
  }
  f.cand = true;
}

inline uint64_t mix(uint64_t h, uint64_t v) {
  h ^= v + 0x9e3779b97f4a7c15ULL + (h << 6) + (h >> 2);
  return h;
}

// One pixel's front-to-back pass over its tile list.  When `kept` is given
// it receives the list positions composited, in order, with alpha, the
// transmittance before each, exp(-q), the clamp state and (dx, dy).
struct Kept {
  int32_t pos;
  double alpha, T, G, dx, dy;
  bool clamped;
};

struct PixelOut {
  double C[3], T;
  int32_t last, n_eval;
  uint8_t flags;
  uint64_t sig;
  double T_err;  // relative error bound of an fp32 evaluation of T
};

void composite_pixel(const double* rec, const int32_t* list, int64_t len,
                     double px, double py, PixelOut& o, std::vector<Kept>* kept) {
  o.C[0] = o.C[1] = o.C[2] = 0;
  o.T = 1.0;
  o.last = 0;
  o.n_eval = 0;
  o.flags = 0;
  o.sig = 0x12345;
  o.T_err = 0.0;
  int32_t n_kept = 0;
  for (int64_t p = 0; p < len; ++p) {
    const double* r = rec + (int64_t)list[p] * OR_REC;
    o.n_eval++;
    double dx = r[OR_U] - px, dy = r[OR_V] - py;
    double a = r[OR_A], b = r[OR_B], c = r[OR_C];
    double q = 0.5 * (a * dx * dx + c * dy * dy) + b * dx * dy;
    // fp32 evaluation bound of q on the GPU side (no cancellation form)
    double qmag = 0.5 * (std::fabs(a) * dx * dx + std::fabs(c) * dy * dy) + std::fabs(b * dx * dy);
    if (q < 0) {
      if (q > -1e-9 * (1 + qmag)) o.flags |= OR_P_NEAR;
      o.sig = mix(o.sig, 2 * p + 1);
      continue;
    }
    double G = std::exp(-q);
    double araw = r[OR_OPAC] * G;
    double da = 1e-5 + 1e-6 * qmag;      // relative margin of the fp32 alpha
    bool clamped = araw > 0.99;
    if (std::fabs(araw - 0.99) <= da * 0.99) o.flags |= OR_P_NEAR;
    double alpha = clamped ? 0.99 : araw;
    if (std::fabs(alpha - 1.0 / 255.0) <= da / 255.0) o.flags |= OR_P_NEAR;
    if (alpha < 1.0 / 255.0) {
      o.sig = mix(o.sig, 2 * p + 1);
      continue;
    }
    double Tn = o.T * (1.0 - alpha);
    double dT = 1e-5 + 4.0 * (n_kept + 1) * 5.96e-8 + da;  // relative margin of fp32 T
    if (std::fabs(Tn - 1e-4) <= dT * 1e-4) o.flags |= OR_P_NEAR;
    if (Tn < 1e-4) {
      o.sig = mix(o.sig, 0xdead0000ULL + p);
      break;
    }
    if (kept) kept->push_back({(int32_t)p, alpha, o.T, G, dx, dy, clamped});
    for (int ch = 0; ch < 3; ++ch) o.C[ch] += r[OR_R + ch] * alpha * o.T;
    // fp32 T = prod (1 - alpha): each factor carries the relative error of
    // its alpha (exp and q rounding, unless clamped) scaled by
    // alpha / (1 - alpha), plus one rounding of the product
    o.T_err += (clamped ? 0.0 : alpha / (1.0 - alpha) * (3e-7 + 5e-7 * q)) + 1.2e-7;
    o.T = Tn;
    o.last = (int32_t)p + 1;
    n_kept++;
    o.sig = mix(o.sig, 2 * p + (clamped ? 0x100000000ULL : 0));
  }
}

}  // namespace

extern "C" {

int32_t or_version(void) { return 1; }

int32_t or_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void or_sh_basis(const double* d, double* Y, double* dY) {
  sh_eval(d[0], d[1], d[2], Y, dY);
}

int64_t or_project_rects(const double* params, int64_t n, int64_t n_pad,
                         int32_t D, const double* cam, int32_t W, int32_t H,
                         int32_t tight, uint8_t* is_cand, double* rec,
                         int32_t* rect, uint32_t* depth_key, uint8_t* flags) {
  Cam k = load_cam(cam);
  int64_t count = 0;
#pragma omp parallel for schedule(static) reduction(+ : count)
  for (int64_t i = 0; i < n; ++i) {
    Forward3D f;
    project_one(params, n_pad, D, k, W, H, i, f, tight != 0);
    is_cand[i] = f.cand ? 1 : 0;
    flags[i] = f.flags;
    double* r = rec + i * OR_REC;
    std::fill(r, r + OR_REC, 0.0);
    for (int j = 0; j < 4; ++j) rect[4 * i + j] = 0;
    depth_key[i] = 0;
    if (!f.cand) continue;
    count++;
    r[OR_U] = f.u; r[OR_V] = f.v; r[OR_DEPTH] = f.tcam[2]; r[OR_RADIUS] = f.radius;
    r[OR_A] = f.conic[0]; r[OR_B] = f.conic[1]; r[OR_C] = f.conic[2];
    r[OR_OPAC] = f.opac;
    r[OR_R] = f.rgb[0]; r[OR_G] = f.rgb[1]; r[OR_BL] = f.rgb[2];
    r[OR_S00] = f.S2p[0]; r[OR_S01] = f.S2p[1]; r[OR_S11] = f.S2p[2];
    r[OR_SQUARE] = (double)f.square_tiles;
    for (int j = 0; j < 4; ++j) rect[4 * i + j] = (int32_t)f.rect[j];
    float dz = (float)f.tcam[2];
    uint32_t bits;
    std::memcpy(&bits, &dz, 4);
    depth_key[i] = bits;
  }
  return count;
}

int64_t or_project(const double* params, int64_t n, int64_t n_pad, int32_t D,
                   const double* cam, int32_t W, int32_t H, uint8_t* is_cand,
                   double* rec, int32_t* rect, uint32_t* depth_key,
                   uint8_t* flags) {
  return or_project_rects(params, n, n_pad, D, cam, W, H, 1, is_cand, rec,
                          rect, depth_key, flags);
}

int64_t or_tile_lists_scan(int64_t C, const int32_t* rect, const uint32_t* key,
                           int32_t TW, const int32_t* tiles, int64_t n_tiles,
                           int64_t* offsets, int32_t* vals) {
  std::vector<int64_t> cnt(n_tiles, 0);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t k = 0; k < n_tiles; ++k) {
    int32_t tx = tiles[k] % TW, ty = tiles[k] / TW;
    int64_t c = 0;
    for (int64_t j = 0; j < C; ++j) {
      const int32_t* r = rect + 4 * j;
      if (tx >= r[0] && tx < r[2] && ty >= r[1] && ty < r[3]) c++;
    }
    cnt[k] = c;
  }
  offsets[0] = 0;
  for (int64_t k = 0; k < n_tiles; ++k) offsets[k + 1] = offsets[k] + cnt[k];
  if (!vals) return offsets[n_tiles];
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t k = 0; k < n_tiles; ++k) {
    int32_t tx = tiles[k] % TW, ty = tiles[k] / TW;
    int32_t* out = vals + offsets[k];
    int64_t c = 0;
    for (int64_t j = 0; j < C; ++j) {
      const int32_t* r = rect + 4 * j;
      if (tx >= r[0] && tx < r[2] && ty >= r[1] && ty < r[3]) out[c++] = (int32_t)j;
    }
    // ascending candidate position already; stable sort by depth key
    std::stable_sort(out, out + c, [&](int32_t p, int32_t q) { return key[p] < key[q]; });
  }
  return offsets[n_tiles];
}

int64_t or_tile_lists_scatter(int64_t C, const int32_t* rect,
                              const uint32_t* key, int32_t TW, int32_t TH,
                              int64_t* offsets, int32_t* vals) {
  int64_t T = (int64_t)TW * TH;
  std::vector<int64_t> cnt(T + 1, 0);
  for (int64_t j = 0; j < C; ++j) {
    const int32_t* r = rect + 4 * j;
    for (int32_t ty = r[1]; ty < r[3]; ++ty)
      for (int32_t tx = r[0]; tx < r[2]; ++tx) cnt[(int64_t)ty * TW + tx]++;
  }
  offsets[0] = 0;
  for (int64_t t = 0; t < T; ++t) offsets[t + 1] = offsets[t] + cnt[t];
  if (!vals) return offsets[T];
  std::vector<int64_t> fill(offsets, offsets + T);
  for (int64_t j = 0; j < C; ++j) {
    const int32_t* r = rect + 4 * j;
    for (int32_t ty = r[1]; ty < r[3]; ++ty)
      for (int32_t tx = r[0]; tx < r[2]; ++tx) vals[fill[(int64_t)ty * TW + tx]++] = (int32_t)j;
  }
#pragma omp parallel for schedule(dynamic, 64)
  for (int64_t t = 0; t < T; ++t)
    std::stable_sort(vals + offsets[t], vals + offsets[t + 1],
                     [&](int32_t p, int32_t q) { return key[p] < key[q]; });
  return offsets[T];
}

int32_t or_raster_fwd(int64_t C, const double* rec, int32_t TW, int32_t W,
                      int32_t H, const int32_t* tiles, int64_t n_tiles,
                      const int64_t* offsets, const int32_t* vals, double* img,
                      double* T_final, int32_t* last, uint8_t* pflags,
                      int32_t* n_eval, uint64_t* sig, double* T_err) {
  (void)C;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t k = 0; k < n_tiles; ++k) {
    int32_t tx = tiles[k] % TW, ty = tiles[k] / TW;
    const int32_t* list = vals + offsets[k];
    int64_t len = offsets[k + 1] - offsets[k];
    for (int j = 0; j < kTile * kTile; ++j) {
      int32_t x = tx * kTile + (j % kTile), y = ty * kTile + (j / kTile);
      int64_t o = k * 256 + j;
      PixelOut po;
      if (x >= W || y >= H) {
        po = PixelOut{{0, 0, 0}, 1.0, 0, 0, OR_P_INVALID, 0, 0.0};
      } else {
        composite_pixel(rec, list, len, x + 0.5, y + 0.5, po, nullptr);
      }
      for (int ch = 0; ch < 3; ++ch) img[(k * 3 + ch) * 256 + j] = po.C[ch];
      T_final[o] = po.T;
      last[o] = po.last;
      pflags[o] = po.flags;
      n_eval[o] = po.n_eval;
      sig[o] = po.sig;
      if (T_err) T_err[o] = po.T_err;
    }
  }
  return 0;
}

int32_t or_raster_bwd(int64_t C, const double* rec, int32_t TW, int32_t W,
                      int32_t H, const int32_t* tiles, int64_t n_tiles,
                      const int64_t* offsets, const int32_t* vals,
                      const double* dL_dpix, double* g2d) {
  (void)C;
#pragma omp parallel
  {
    std::vector<Kept> kept;
    std::vector<double> tg;   // this tile's gradient per list position
#pragma omp for schedule(dynamic, 1)
    for (int64_t k = 0; k < n_tiles; ++k) {
      int32_t tx = tiles[k] % TW, ty = tiles[k] / TW;
      const int32_t* list = vals + offsets[k];
      int64_t len = offsets[k + 1] - offsets[k];
      tg.assign((size_t)len * 9, 0.0);
      for (int j = 0; j < 256; ++j) {
        int32_t x = tx * kTile + (j % kTile), y = ty * kTile + (j / kTile);
        if (x >= W || y >= H) continue;
        kept.clear();
        PixelOut po;
        composite_pixel(rec, list, len, x + 0.5, y + 0.5, po, &kept);
        double gC[3];
        for (int ch = 0; ch < 3; ++ch) gC[ch] = dL_dpix[(k * 3 + ch) * 256 + j];
        // reverse over the composited entries: A = colour accumulated behind
        double A[3] = {0, 0, 0};
        for (int64_t e = (int64_t)kept.size() - 1; e >= 0; --e) {
          const Kept& K = kept[e];
          const double* r = rec + (int64_t)list[K.pos] * OR_REC;
          double* out = tg.data() + (int64_t)K.pos * 9;
          double dalpha = 0;
          for (int ch = 0; ch < 3; ++ch) {
            double col = r[OR_R + ch];
            out[6 + ch] += K.alpha * K.T * gC[ch];
            dalpha += gC[ch] * (col * K.T - A[ch] / (1.0 - K.alpha));
            A[ch] += col * K.alpha * K.T;
          }
          if (K.clamped) continue;
          double dopac = K.G * dalpha;
          double dq = -K.alpha * dalpha;
          double a = r[OR_A], b = r[OR_B], c = r[OR_C];
          out[0] += dq * (a * K.dx + b * K.dy);
          out[1] += dq * (b * K.dx + c * K.dy);
          out[2] += dq * 0.5 * K.dx * K.dx;
          out[3] += dq * K.dx * K.dy;
          out[4] += dq * 0.5 * K.dy * K.dy;
          out[5] += dopac;
        }
      }
      for (int64_t p = 0; p < len; ++p) {
        double* dst = g2d + (int64_t)list[p] * 9;
        for (int e = 0; e < 9; ++e) {
          double val = tg[(size_t)p * 9 + e];
          if (val == 0.0) continue;
#pragma omp atomic
          dst[e] += val;
        }
      }
    }
  }
  return 0;
}

int32_t or_project_bwd(const double* params, int64_t n_pad, int32_t D,
                       const double* cam, int64_t C, const int32_t* cand_idx,
                       const double* g2d, double* g3d) {
  Cam k = load_cam(cam);
  const int P = 11 + 3 * (D + 1) * (D + 1);
  const int ksh = (D + 1) * (D + 1);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < C; ++j) {
    int64_t i = cand_idx[j];
    auto Pm = [&](int plane) { return params[(int64_t)plane * n_pad + i]; };
    auto out = [&](int plane) -> double& { return g3d[(int64_t)plane * C + j]; };
    for (int p = 0; p < P; ++p) out(p) = 0;
    // forward intermediates (same formulas as project_one, no cull)
    Forward3D f;
    for (int q = 0; q < 3; ++q) f.mean[q] = Pm(q);
    for (int r = 0; r < 3; ++r)
      f.tcam[r] = ((k.R[3 * r] * f.mean[0] + k.R[3 * r + 1] * f.mean[1]) + k.R[3 * r + 2] * f.mean[2]) + k.t[r];
    double tx = f.tcam[0], ty = f.tcam[1], tz = f.tcam[2];
    double q4[4] = {Pm(6), Pm(7), Pm(8), Pm(9)};
    f.qnorm = std::sqrt(q4[0] * q4[0] + q4[1] * q4[1] + q4[2] * q4[2] + q4[3] * q4[3]);
    for (int q = 0; q < 4; ++q) f.qn[q] = q4[q] / f.qnorm;
    quat_to_R(f.qn, f.Rq);
    for (int q = 0; q < 3; ++q) f.s[q] = std::exp(Pm(3 + q));
    for (int r = 0; r < 3; ++r)
      for (int c = 0; c < 3; ++c) f.M[3 * r + c] = f.Rq[3 * r + c] * f.s[c];
    for (int r = 0; r < 3; ++r)
      for (int c = 0; c < 3; ++c) {
        double acc = 0;
        for (int q = 0; q < 3; ++q) acc += f.M[3 * r + q] * f.M[3 * c + q];
        f.Sigma[3 * r + c] = acc;
      }
    f.J[0] = k.fx / tz; f.J[1] = 0; f.J[2] = -k.fx * tx / (tz * tz);
    f.J[3] = 0; f.J[4] = k.fy / tz; f.J[5] = -k.fy * ty / (tz * tz);
    for (int r = 0; r < 2; ++r)
      for (int c = 0; c < 3; ++c) {
        double acc = 0;
        for (int q = 0; q < 3; ++q) acc += f.J[3 * r + q] * k.R[3 * q + c];
        f.T[3 * r + c] = acc;
      }
    double TS[6];
    for (int r = 0; r < 2; ++r)
      for (int c = 0; c < 3; ++c) {
        double acc = 0;
        for (int q = 0; q < 3; ++q) acc += f.T[3 * r + q] * f.Sigma[3 * q + c];
        TS[3 * r + c] = acc;
      }
    double S2p[4];
    for (int r = 0; r < 2; ++r)
      for (int c = 0; c < 2; ++c) {
        double acc = 0;
        for (int q = 0; q < 3; ++q) acc += TS[3 * r + q] * f.T[3 * c + q];
        S2p[2 * r + c] = acc;
      }
    S2p[1] = S2p[2] = 0.5 * (S2p[1] + S2p[2]);
    S2p[0] += 0.3; S2p[3] += 0.3;
    double det = S2p[0] * S2p[3] - S2p[1] * S2p[1];
    double Q[4] = {S2p[3] / det, -S2p[1] / det, -S2p[1] / det, S2p[0] / det};
    const double* g = g2d + j * 9;
    double du = g[0], dv = g[1], dA = g[2], dB = g[3], dCc = g[4], dO = g[5];
    // opacity logit
    double o = 1.0 / (1.0 + std::exp(-Pm(10)));
    out(10) = dO * o * (1 - o);
    // conic -> 2D covariance: dS = -Q Gbar Q, Gbar symmetric
    double Gb[4] = {dA, 0.5 * dB, 0.5 * dB, dCc};
    double QG[4], dS2[4];
    for (int r = 0; r < 2; ++r)
      for (int c = 0; c < 2; ++c) QG[2 * r + c] = Q[2 * r] * Gb[c] + Q[2 * r + 1] * Gb[2 + c];
    for (int r = 0; r < 2; ++r)
      for (int c = 0; c < 2; ++c) dS2[2 * r + c] = -(QG[2 * r] * Q[c] + QG[2 * r + 1] * Q[2 + c]);
    // 2D covariance -> Sigma (T^T dS2 T) and -> T (2 dS2 T Sigma)
    double dSigma[9], dT[6];
    for (int r = 0; r < 3; ++r)
      for (int c = 0; c < 3; ++c) {
        double acc = 0;
        for (int a = 0; a < 2; ++a)
          for (int b = 0; b < 2; ++b) acc += f.T[3 * a + r] * dS2[2 * a + b] * f.T[3 * b + c];
        dSigma[3 * r + c] = acc;
      }
    for (int r = 0; r < 2; ++r)
      for (int c = 0; c < 3; ++c) {
        double acc = 0;
        for (int b = 0; b < 2; ++b) acc += dS2[2 * r + b] * TS[3 * b + c];
        dT[3 * r + c] = 2.0 * acc;
      }
    // T = J W  ->  dJ = dT W^T
    double dJ[6];
    for (int r = 0; r < 2; ++r)
      for (int c = 0; c < 3; ++c) {
        double acc = 0;
        for (int q = 0; q < 3; ++q) acc += dT[3 * r + q] * k.R[3 * c + q];
        dJ[3 * r + c] = acc;
      }
    double dt[3] = {0, 0, 0};
    double tz2 = tz * tz, tz3 = tz2 * tz;
    dt[0] += dJ[2] * (-k.fx / tz2);
    dt[1] += dJ[5] * (-k.fy / tz2);
    dt[2] += dJ[0] * (-k.fx / tz2) + dJ[2] * (2 * k.fx * tx / tz3) +
             dJ[4] * (-k.fy / tz2) + dJ[5] * (2 * k.fy * ty / tz3);
    // screen position u = fx tx/tz + cx, v = fy ty/tz + cy
    dt[0] += du * k.fx / tz;
    dt[2] += du * (-k.fx * tx / tz2);
    dt[1] += dv * k.fy / tz;
    dt[2] += dv * (-k.fy * ty / tz2);
    double dmean[3];
    for (int c = 0; c < 3; ++c) dmean[c] = k.R[c] * dt[0] + k.R[3 + c] * dt[1] + k.R[6 + c] * dt[2];
    // Sigma = M M^T, M = R S
    double dM[9];
    for (int r = 0; r < 3; ++r)
      for (int c = 0; c < 3; ++c) {
        double acc = 0;
        for (int q = 0; q < 3; ++q) acc += dSigma[3 * r + q] * f.M[3 * q + c];
        dM[3 * r + c] = 2.0 * acc;
      }
    for (int c = 0; c < 3; ++c) {
      double ds = 0;
      for (int r = 0; r < 3; ++r) ds += dM[3 * r + c] * f.Rq[3 * r + c];
      out(3 + c) = ds * f.s[c];
    }
    double dRq[9];
    for (int r = 0; r < 3; ++r)
      for (int c = 0; c < 3; ++c) dRq[3 * r + c] = dM[3 * r + c] * f.s[c];
    double jac[9][4];
    quat_to_R_jac(f.qn, jac);
    double dqn[4] = {0, 0, 0, 0};
    for (int e = 0; e < 9; ++e)
      for (int q = 0; q < 4; ++q) dqn[q] += dRq[e] * jac[e][q];
    double dot = 0;
    for (int q = 0; q < 4; ++q) dot += dqn[q] * f.qn[q];
    for (int q = 0; q < 4; ++q) out(6 + q) = (dqn[q] - f.qn[q] * dot) / f.qnorm;
    // colour: SH coefficients and the view direction
    double cc[3];
    for (int c = 0; c < 3; ++c)
      cc[c] = -(k.R[c] * k.t[0] + k.R[3 + c] * k.t[1] + k.R[6 + c] * k.t[2]);
    double dir[3] = {f.mean[0] - cc[0], f.mean[1] - cc[1], f.mean[2] - cc[2]};
    double dn = std::sqrt(dir[0] * dir[0] + dir[1] * dir[1] + dir[2] * dir[2]);
    double d[3] = {dir[0] / dn, dir[1] / dn, dir[2] / dn};
    double Y[16], dY[48];
    sh_eval(d[0], d[1], d[2], Y, dY);
    double dd[3] = {0, 0, 0};
    for (int ch = 0; ch < 3; ++ch) {
      double raw = 0.5;
      for (int kk = 0; kk < ksh; ++kk) raw += Pm(11 + 3 * kk + ch) * Y[kk];
      if (raw < 0) continue;
      double gc = g[6 + ch];
      for (int kk = 0; kk < ksh; ++kk) {
        out(11 + 3 * kk + ch) = gc * Y[kk];
        double coef = Pm(11 + 3 * kk + ch);
        for (int a = 0; a < 3; ++a) dd[a] += gc * coef * dY[3 * kk + a];
      }
    }
    double ddot = dd[0] * d[0] + dd[1] * d[1] + dd[2] * d[2];
    for (int a = 0; a < 3; ++a) dmean[a] += (dd[a] - d[a] * ddot) / dn;
    for (int a = 0; a < 3; ++a) out(a) = dmean[a];
  }
  return 0;
}

namespace {
struct LeafCtx {
  const int64_t* sat;
  int32_t TW, TH, W, H;
  const int64_t* lm;
  int64_t budget;
  int32_t* leaves;
  int64_t* leaf_isect;
  int64_t* leaf_bytes;
  uint8_t* over;
  int32_t max_leaves, n;
  bool overflow;
};

int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

int64_t sat_sum(const LeafCtx& c, int32_t x0, int32_t y0, int32_t x1, int32_t y1) {
  int64_t s = c.TW + 1;
  return c.sat[(int64_t)y1 * s + x1] - c.sat[(int64_t)y0 * s + x1] -
         c.sat[(int64_t)y1 * s + x0] + c.sat[(int64_t)y0 * s + x0];
}

// BoundedGS section 02 (B -> C): split any region whose estimated load is
// over budget.  Reading: cut at the midpoint of the longer tile side.
void split(LeafCtx& c, int32_t x0, int32_t y0, int32_t x1, int32_t y1) {
  int64_t I = sat_sum(c, x0, y0, x1, y1);
  int64_t px = (int64_t)(std::min(x1 * kTile, c.W) - x0 * kTile) *
               (std::min(y1 * kTile, c.H) - y0 * kTile);
  int64_t T = (int64_t)(x1 - x0) * (y1 - y0);
  int64_t al = c.lm[4];
  int64_t load = align_up(I * c.lm[0], al) + align_up(px * c.lm[1], al) +
                 align_up(T * c.lm[2], al) + c.lm[3];
  int32_t w = x1 - x0, h = y1 - y0;
  if (load <= c.budget || (w == 1 && h == 1)) {
    if (c.n >= c.max_leaves) { c.overflow = true; return; }
    int32_t* L = c.leaves + 4 * c.n;
    L[0] = x0; L[1] = y0; L[2] = x1; L[3] = y1;
    c.leaf_isect[c.n] = I;
    c.leaf_bytes[c.n] = load;
    c.over[c.n] = load > c.budget ? 1 : 0;
    c.n++;
    return;
  }
  if (w >= h) {
    int32_t xm = x0 + w / 2;
    split(c, x0, y0, xm, y1);
    split(c, xm, y0, x1, y1);
  } else {
    int32_t ym = y0 + h / 2;
    split(c, x0, y0, x1, ym);
    split(c, x0, ym, x1, y1);
  }
}
}  // namespace

int32_t or_leaf_partition(const int64_t* sat, int32_t TW, int32_t TH,
                          int32_t W, int32_t H, const int64_t* lm,
                          int64_t budget, int32_t* leaves, int64_t* leaf_isect,
                          int64_t* leaf_bytes, uint8_t* over_budget,
                          int32_t max_leaves) {
  LeafCtx c{sat, TW, TH, W, H, lm, budget, leaves, leaf_isect, leaf_bytes,
            over_budget, max_leaves, 0, false};
  if (TW <= 0 || TH <= 0) return 0;
  split(c, 0, 0, TW, TH);
  return c.overflow ? -1 : c.n;
}

}  // extern "C"
