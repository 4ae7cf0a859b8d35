// Projection backward (stage 2 of the two-stage backward) and Adam.
//
// BoundedGS project page, section 02 (A -> B): raster backward first
// collects the projected-attribute gradients; projection backward runs
// after the raster buffers are gone.  Section 01: the whole view's gradient
// is summed before ONE parameter update.  SkipGS paper notes, "loss
// function / training strategy": gradients reach means, quaternions, scales,
// opacities and SH coefficients and Adam updates the parameters.
//
// The fused variant runs one thread per Gaussian over all n: candidates
// differentiate their projection and update their parameters in the same
// pass; non-candidates take the Adam step with a zero gradient.  Parameters,
// moments and gradients stream through once (24 bytes per float), and the
// compact 3D gradients are never materialised.
#include <math.h>

#include "gs_internal.cuh"

namespace gs {
namespace {

constexpr int kThreads = 256;

struct BwdCam {
  double R[9], t[3], fx, fy, campos[3];
};

struct AdamK {
  float lr, b1, b2, omb1, omb2, eps, bc1, bc2;
  float step;     // lr / (1 - b1^t)
  float rsbc2;    // 1 / sqrt(1 - b2^t)
};

__device__ __forceinline__ void adam_update(float* __restrict__ p, float* __restrict__ m,
                                            float* __restrict__ v, int64_t idx, float g,
                                            const AdamK& a) {
  const float mm = fmaf(a.b1, m[idx], a.omb1 * g);
  const float vv = fmaf(a.b2, v[idx], a.omb2 * g * g);
  m[idx] = mm;
  v[idx] = vv;
  p[idx] = fmaf(-a.step, __fdividef(mm, fmaf(sqrtf(vv), a.rsbc2, a.eps)), p[idx]);
}

// Gradients of one candidate.  `emit(plane, g)` receives every parameter's
// gradient exactly once, SH planes first, then planes 10 .. 0.  Real: the
// type of the geometric chain (the SH part is fp64).
template <bool WITH_SH, class Real, class Emit>
__device__ __forceinline__ void candidate_grad(const float* __restrict__ P, int64_t n_pad, int64_t i,
                                               int D, const BwdCam& c, const float* __restrict__ g2,
                                               const float4 rgb_rec, Emit&& emit) {
  const Real mx = P[i], my = P[n_pad + i], mz = P[2 * n_pad + i];
  Real tc[3];
#pragma unroll
  for (int r = 0; r < 3; ++r) tc[r] = Real(c.R[3 * r]) * mx + Real(c.R[3 * r + 1]) * my + Real(c.R[3 * r + 2]) * mz + Real(c.t[r]);
  const Real tx = tc[0], ty = tc[1], tz = tc[2];
  Real qw = P[6 * n_pad + i], qx = P[7 * n_pad + i], qy = P[8 * n_pad + i], qz = P[9 * n_pad + i];
  const Real qn = sqrt(qw * qw + qx * qx + qy * qy + qz * qz);
  qw /= qn; qx /= qn; qy /= qn; qz /= qn;
  Real Rg[9];
  Rg[0] = Real(1.0) - Real(2.0) * (qy * qy + qz * qz); Rg[1] = Real(2.0) * (qx * qy - qw * qz); Rg[2] = Real(2.0) * (qx * qz + qw * qy);
  Rg[3] = Real(2.0) * (qx * qy + qw * qz); Rg[4] = Real(1.0) - Real(2.0) * (qx * qx + qz * qz); Rg[5] = Real(2.0) * (qy * qz - qw * qx);
  Rg[6] = Real(2.0) * (qx * qz - qw * qy); Rg[7] = Real(2.0) * (qy * qz + qw * qx); Rg[8] = Real(1.0) - Real(2.0) * (qx * qx + qy * qy);
  Real sc[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) sc[k] = exp((Real)P[(3 + k) * n_pad + i]);
  Real M[9];
#pragma unroll
  for (int r = 0; r < 3; ++r)
#pragma unroll
    for (int k = 0; k < 3; ++k) M[3 * r + k] = Rg[3 * r + k] * sc[k];
  Real Sg[9];
#pragma unroll
  for (int r = 0; r < 3; ++r)
#pragma unroll
    for (int k = 0; k < 3; ++k)
      Sg[3 * r + k] = M[3 * r] * M[3 * k] + M[3 * r + 1] * M[3 * k + 1] + M[3 * r + 2] * M[3 * k + 2];
  const Real tz2 = tz * tz;
  const Real j00 = Real(c.fx) / tz, j02 = -Real(c.fx) * tx / tz2, j11 = Real(c.fy) / tz, j12 = -Real(c.fy) * ty / tz2;
  Real T0[3], T1[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    T0[k] = j00 * Real(c.R[k]) + j02 * Real(c.R[6 + k]);
    T1[k] = j11 * Real(c.R[3 + k]) + j12 * Real(c.R[6 + k]);
  }
  Real A0[3], A1[3];  // rows of T Sigma
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    A0[k] = T0[0] * Sg[k] + T0[1] * Sg[3 + k] + T0[2] * Sg[6 + k];
    A1[k] = T1[0] * Sg[k] + T1[1] * Sg[3 + k] + T1[2] * Sg[6 + k];
  }
  const Real c00 = A0[0] * T0[0] + A0[1] * T0[1] + A0[2] * T0[2] + Real(0.3);
  const Real c01 = Real(0.5) * ((A0[0] * T1[0] + A0[1] * T1[1] + A0[2] * T1[2]) +
                            (A1[0] * T0[0] + A1[1] * T0[1] + A1[2] * T0[2]));
  const Real c11 = A1[0] * T1[0] + A1[1] * T1[1] + A1[2] * T1[2] + Real(0.3);
  const Real det = c00 * c11 - c01 * c01;
  const Real qa = c11 / det, qb = -c01 / det, qc = c00 / det;  // conic

  const Real du = g2[0], dv = g2[1], dA = g2[2], dB = g2[3], dC = g2[4], dO = g2[5];
  const Real dcol[3] = {g2[6], g2[7], g2[8]};

  // conic -> Sigma': dS = -Q Gbar Q,  Gbar = [[dA, dB/2], [dB/2, dC]]
  const Real hB = Real(0.5) * dB;
  const Real m00 = qa * dA + qb * hB, m01 = qa * hB + qb * dC;
  const Real m10 = qb * dA + qc * hB, m11 = qb * hB + qc * dC;
  const Real G00 = -(m00 * qa + m01 * qb);
  const Real G01 = -(m00 * qb + m01 * qc);
  const Real G11 = -(m10 * qb + m11 * qc);
  // Sigma' = T Sigma T^T + Real(0.3) I  ->  dSigma = T^T G T,  dT = 2 G T Sigma
  Real dS[9];
#pragma unroll
  for (int r = 0; r < 3; ++r)
#pragma unroll
    for (int k = 0; k < 3; ++k)
      dS[3 * r + k] = T0[r] * (G00 * T0[k] + G01 * T1[k]) + T1[r] * (G01 * T0[k] + G11 * T1[k]);
  Real dT0[3], dT1[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    dT0[k] = Real(2.0) * (G00 * A0[k] + G01 * A1[k]);
    dT1[k] = Real(2.0) * (G01 * A0[k] + G11 * A1[k]);
  }
  // T = J W
  const Real dJ00 = dT0[0] * Real(c.R[0]) + dT0[1] * Real(c.R[1]) + dT0[2] * Real(c.R[2]);
  const Real dJ02 = dT0[0] * Real(c.R[6]) + dT0[1] * Real(c.R[7]) + dT0[2] * Real(c.R[8]);
  const Real dJ11 = dT1[0] * Real(c.R[3]) + dT1[1] * Real(c.R[4]) + dT1[2] * Real(c.R[5]);
  const Real dJ12 = dT1[0] * Real(c.R[6]) + dT1[1] * Real(c.R[7]) + dT1[2] * Real(c.R[8]);
  const Real tz3 = tz2 * tz;
  const Real dtx = -dJ02 * Real(c.fx) / tz2 + du * Real(c.fx) / tz;
  const Real dty = -dJ12 * Real(c.fy) / tz2 + dv * Real(c.fy) / tz;
  const Real dtz = -dJ00 * Real(c.fx) / tz2 + dJ02 * Real(2.0) * Real(c.fx) * tx / tz3 - dJ11 * Real(c.fy) / tz2 +
                     dJ12 * Real(2.0) * Real(c.fy) * ty / tz3 - du * Real(c.fx) * tx / tz2 - dv * Real(c.fy) * ty / tz2;
  Real dmean[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) dmean[k] = Real(c.R[k]) * dtx + Real(c.R[3 + k]) * dty + Real(c.R[6 + k]) * dtz;
  // Sigma = M M^T,  M = R S
  Real dM[9];
#pragma unroll
  for (int r = 0; r < 3; ++r)
#pragma unroll
    for (int k = 0; k < 3; ++k)
      dM[3 * r + k] = Real(2.0) * (dS[3 * r] * M[k] + dS[3 * r + 1] * M[3 + k] + dS[3 * r + 2] * M[6 + k]);
  Real dls[3];
#pragma unroll
  for (int k = 0; k < 3; ++k)
    dls[k] = (dM[k] * Rg[k] + dM[3 + k] * Rg[3 + k] + dM[6 + k] * Rg[6 + k]) * sc[k];
  Real gR[9];
#pragma unroll
  for (int r = 0; r < 3; ++r)
#pragma unroll
    for (int k = 0; k < 3; ++k) gR[3 * r + k] = dM[3 * r + k] * sc[k];
  // rotation of the unit quaternion -> (w, x, y, z)
  const Real gw = Real(2.0) * (-qz * gR[1] + qy * gR[2] + qz * gR[3] - qx * gR[5] - qy * gR[6] + qx * gR[7]);
  const Real gx = Real(2.0) * (qy * gR[1] + qz * gR[2] + qy * gR[3] - Real(2.0) * qx * gR[4] - qw * gR[5] +
                           qz * gR[6] + qw * gR[7] - Real(2.0) * qx * gR[8]);
  const Real gy = Real(2.0) * (-Real(2.0) * qy * gR[0] + qx * gR[1] + qw * gR[2] + qx * gR[3] + qz * gR[5] -
                           qw * gR[6] + qz * gR[7] - Real(2.0) * qy * gR[8]);
  const Real gz = Real(2.0) * (-Real(2.0) * qz * gR[0] - qw * gR[1] + qx * gR[2] + qw * gR[3] - Real(2.0) * qz * gR[4] +
                           qy * gR[5] + qx * gR[6] + qy * gR[7]);
  const Real qdot = gw * qw + gx * qx + gy * qy + gz * qz;
  const Real dq[4] = {(gw - qw * qdot) / qn, (gx - qx * qdot) / qn, (gy - qy * qdot) / qn,
                        (gz - qz * qdot) / qn};
  // opacity logit
  const Real o = Real(1.0) / (Real(1.0) + exp(-(Real)P[10 * n_pad + i]));
  const Real dlogit = dO * o * (Real(1.0) - o);

  if constexpr (WITH_SH) {
  // SH coefficients and the view direction
  double ex = mx - c.campos[0], ey = my - c.campos[1], ez = mz - c.campos[2];
  const double en = sqrt(ex * ex + ey * ey + ez * ez);
  ex /= en; ey /= en; ez /= en;
  const bool live[3] = {rgb_rec.x > 0.0f, rgb_rec.y > 0.0f, rgb_rec.z > 0.0f};
  const double kPi = 3.141592653589793;
  double Y[16], dY[16][3];
  {
    const double x = ex, y = ey, z = ez, xx = x * x, yy = y * y, zz = z * z;
    Y[0] = 0.5 / sqrt(kPi);
    dY[0][0] = dY[0][1] = dY[0][2] = 0.0;
    const double k1 = sqrt(3.0 / (4.0 * kPi));
    Y[1] = -k1 * y; dY[1][0] = 0; dY[1][1] = -k1; dY[1][2] = 0;
    Y[2] = k1 * z; dY[2][0] = 0; dY[2][1] = 0; dY[2][2] = k1;
    Y[3] = -k1 * x; dY[3][0] = -k1; dY[3][1] = 0; dY[3][2] = 0;
    const double k2a = 0.5 * sqrt(15.0 / kPi), k2b = 0.25 * sqrt(5.0 / kPi), k2c = 0.25 * sqrt(15.0 / kPi);
    Y[4] = k2a * x * y; dY[4][0] = k2a * y; dY[4][1] = k2a * x; dY[4][2] = 0;
    Y[5] = -k2a * y * z; dY[5][0] = 0; dY[5][1] = -k2a * z; dY[5][2] = -k2a * y;
    Y[6] = k2b * (2 * zz - xx - yy); dY[6][0] = -2 * k2b * x; dY[6][1] = -2 * k2b * y; dY[6][2] = 4 * k2b * z;
    Y[7] = -k2a * x * z; dY[7][0] = -k2a * z; dY[7][1] = 0; dY[7][2] = -k2a * x;
    Y[8] = k2c * (xx - yy); dY[8][0] = 2 * k2c * x; dY[8][1] = -2 * k2c * y; dY[8][2] = 0;
    const double k3a = 0.25 * sqrt(35.0 / (2.0 * kPi)), k3b = 0.5 * sqrt(105.0 / kPi),
                 k3c = 0.25 * sqrt(21.0 / (2.0 * kPi)), k3d = 0.25 * sqrt(7.0 / kPi),
                 k3e = 0.25 * sqrt(105.0 / kPi);
    Y[9] = -k3a * y * (3 * xx - yy); dY[9][0] = -6 * k3a * x * y; dY[9][1] = -3 * k3a * (xx - yy); dY[9][2] = 0;
    Y[10] = k3b * x * y * z; dY[10][0] = k3b * y * z; dY[10][1] = k3b * x * z; dY[10][2] = k3b * x * y;
    Y[11] = -k3c * y * (4 * zz - xx - yy); dY[11][0] = 2 * k3c * x * y;
    dY[11][1] = -k3c * (4 * zz - xx - 3 * yy); dY[11][2] = -8 * k3c * y * z;
    Y[12] = k3d * z * (2 * zz - 3 * xx - 3 * yy); dY[12][0] = -6 * k3d * x * z; dY[12][1] = -6 * k3d * y * z;
    dY[12][2] = k3d * (6 * zz - 3 * xx - 3 * yy);
    Y[13] = -k3c * x * (4 * zz - xx - yy); dY[13][0] = -k3c * (4 * zz - 3 * xx - yy);
    dY[13][1] = 2 * k3c * x * y; dY[13][2] = -8 * k3c * x * z;
    Y[14] = k3e * z * (xx - yy); dY[14][0] = 2 * k3e * x * z; dY[14][1] = -2 * k3e * y * z; dY[14][2] = k3e * (xx - yy);
    Y[15] = -k3a * x * (xx - 3 * yy); dY[15][0] = -3 * k3a * (xx - yy); dY[15][1] = 6 * k3a * x * y; dY[15][2] = 0;
  }
  const int ksh = (D + 1) * (D + 1);
  double dd[3] = {0.0, 0.0, 0.0};
  for (int k = 0; k < ksh; ++k) {
#pragma unroll
    for (int ch = 0; ch < 3; ++ch) {
      const int plane = 11 + 3 * k + ch;
      double g = 0.0;
      if (live[ch]) {
        g = dcol[ch] * Y[k];
        const double coef = dcol[ch] * (double)P[plane * n_pad + i];
        dd[0] += coef * dY[k][0];
        dd[1] += coef * dY[k][1];
        dd[2] += coef * dY[k][2];
      }
      emit(plane, g);
    }
  }
  const double ddot = dd[0] * ex + dd[1] * ey + dd[2] * ez;
  dmean[0] += (dd[0] - ex * ddot) / en;
  dmean[1] += (dd[1] - ey * ddot) / en;
  dmean[2] += (dd[2] - ez * ddot) / en;
  }
  emit(10, dlogit);
#pragma unroll
  for (int k = 0; k < 4; ++k) emit(6 + k, dq[k]);
#pragma unroll
  for (int k = 0; k < 3; ++k) emit(3 + k, dls[k]);
#pragma unroll
  for (int k = 0; k < 3; ++k) emit(k, dmean[k]);
}

__global__ void __launch_bounds__(kThreads)
k_project_bwd(const float* __restrict__ P, int64_t n_pad, int D, BwdCam cam, int64_t n_cand,
              const int32_t* __restrict__ cand_idx, const float4* __restrict__ rec,
              const float* __restrict__ g2d, float* __restrict__ g3d, int64_t stride) {
  const int64_t j = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (j >= n_cand) return;
  const int64_t i = cand_idx[j];
  if (rec[3 * j + 2].w < 0.f) {  // culled Gaussian of the dense layout: no gradient
    for (int plane = 0; plane < 11 + 3 * (D + 1) * (D + 1); ++plane)
      g3d[(int64_t)plane * stride + j] = 0.f;
    return;
  }
  candidate_grad<true, double>(P, n_pad, i, D, cam, g2d + 12 * j, rec[3 * j + 2],
                 [&](int plane, double g) { g3d[(int64_t)plane * stride + j] = (float)g; });
}

__global__ void __launch_bounds__(kThreads)
k_adam(float* __restrict__ P, float* __restrict__ m, float* __restrict__ v,
       const float* __restrict__ g, int64_t g_stride, const int32_t* __restrict__ slot, int64_t n,
       int64_t n_pad, int nP, AdamK a) {
  const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (i >= n) return;
  int64_t col = i;
  bool has = true;
  if (slot) {
    const int32_t s = slot[i];
    has = s >= 0;
    col = s;
  }
  for (int plane = 0; plane < nP; ++plane) {
    const float gg = has ? g[(int64_t)plane * g_stride + col] : 0.0f;
    adam_update(P, m, v, (int64_t)plane * n_pad + i, gg, a);
  }
}

// ---------------------------------------------------------------------------
// Fused path, stage 1: geometric gradients of each candidate, i.e.
// everything except the SH coefficients and the view-direction term of the
// mean, which stage 2 forms (fp64) while it streams the SH planes.  The
// chain runs in fp32 (per-tensor relative L2 error about 3e-6 against the
// fp64 oracle; the parity bound is 1e-4).  Scratch layout (14 floats per
// candidate): double mean[3][C] (stage 2 adds the view-direction term, and
// the sum may cancel), then float rest[8][C] for planes 3..10 (log-scale,
// quaternion, logit).
// ---------------------------------------------------------------------------
// 4 CTAs per SM (64 registers): the chain is latency-bound on its gathers
__global__ void __launch_bounds__(kThreads, 4)
k_project_bwd_geo(const float* __restrict__ P, int64_t n_pad, BwdCam cam, int64_t n_cand,
                  const int32_t* __restrict__ cand_idx, const float4* __restrict__ rec,
                  const float* __restrict__ g2d, double* __restrict__ g_mean,
                  float* __restrict__ g_rest) {
  const int64_t j = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (j >= n_cand) return;
  const int64_t i = cand_idx[j];
  if (rec[3 * j + 2].w < 0.f) {  // culled Gaussian of the dense layout
    for (int plane = 0; plane < 3; ++plane) g_mean[(int64_t)plane * n_cand + j] = 0.0;
    for (int plane = 0; plane < 8; ++plane) g_rest[(int64_t)plane * n_cand + j] = 0.f;
    return;
  }
  candidate_grad<false, float>(P, n_pad, i, 0, cam, g2d + 12 * j, make_float4(0.f, 0.f, 0.f, 0.f),
                 [&](int plane, double gv) {
                   if (plane < 3) g_mean[(int64_t)plane * n_cand + j] = gv;
                   else if (plane < 11) g_rest[(int64_t)(plane - 3) * n_cand + j] = (float)gv;
                 });
}

// fp64 real SH basis function k (same ordering and normalisation as
// candidate_grad's) and its gradient; k is a compile-time constant after
// unrolling, so the switch folds away.
__device__ __forceinline__ void sh_term(int k, double x, double y, double z, double& Y,
                                        double& Yx, double& Yy, double& Yz) {
  const double kPi = 3.141592653589793;
  const double xx = x * x, yy = y * y, zz = z * z;
  const double k1 = sqrt(3.0 / (4.0 * kPi));
  const double k2a = 0.5 * sqrt(15.0 / kPi), k2b = 0.25 * sqrt(5.0 / kPi),
               k2c = 0.25 * sqrt(15.0 / kPi);
  const double k3a = 0.25 * sqrt(35.0 / (2.0 * kPi)), k3b = 0.5 * sqrt(105.0 / kPi),
               k3c = 0.25 * sqrt(21.0 / (2.0 * kPi)), k3d = 0.25 * sqrt(7.0 / kPi),
               k3e = 0.25 * sqrt(105.0 / kPi);
  switch (k) {
    case 0: Y = 0.5 / sqrt(kPi); Yx = Yy = Yz = 0.0; break;
    case 1: Y = -k1 * y; Yx = 0.0; Yy = -k1; Yz = 0.0; break;
    case 2: Y = k1 * z; Yx = 0.0; Yy = 0.0; Yz = k1; break;
    case 3: Y = -k1 * x; Yx = -k1; Yy = 0.0; Yz = 0.0; break;
    case 4: Y = k2a * x * y; Yx = k2a * y; Yy = k2a * x; Yz = 0.0; break;
    case 5: Y = -k2a * y * z; Yx = 0.0; Yy = -k2a * z; Yz = -k2a * y; break;
    case 6: Y = k2b * (2.0 * zz - xx - yy); Yx = -2.0 * k2b * x; Yy = -2.0 * k2b * y;
            Yz = 4.0 * k2b * z; break;
    case 7: Y = -k2a * x * z; Yx = -k2a * z; Yy = 0.0; Yz = -k2a * x; break;
    case 8: Y = k2c * (xx - yy); Yx = 2.0 * k2c * x; Yy = -2.0 * k2c * y; Yz = 0.0; break;
    case 9: Y = -k3a * y * (3.0 * xx - yy); Yx = -6.0 * k3a * x * y; Yy = -3.0 * k3a * (xx - yy);
            Yz = 0.0; break;
    case 10: Y = k3b * x * y * z; Yx = k3b * y * z; Yy = k3b * x * z; Yz = k3b * x * y; break;
    case 11: Y = -k3c * y * (4.0 * zz - xx - yy); Yx = 2.0 * k3c * x * y;
             Yy = -k3c * (4.0 * zz - xx - 3.0 * yy); Yz = -8.0 * k3c * y * z; break;
    case 12: Y = k3d * z * (2.0 * zz - 3.0 * xx - 3.0 * yy); Yx = -6.0 * k3d * x * z;
             Yy = -6.0 * k3d * y * z; Yz = k3d * (6.0 * zz - 3.0 * xx - 3.0 * yy); break;
    case 13: Y = -k3c * x * (4.0 * zz - xx - yy); Yx = -k3c * (4.0 * zz - 3.0 * xx - yy);
             Yy = 2.0 * k3c * x * y; Yz = -8.0 * k3c * x * z; break;
    case 14: Y = k3e * z * (xx - yy); Yx = 2.0 * k3e * x * z; Yy = -2.0 * k3e * y * z;
             Yz = k3e * (xx - yy); break;
    default: Y = -k3a * x * (xx - 3.0 * yy); Yx = -3.0 * k3a * (xx - yy); Yy = 6.0 * k3a * x * y;
             Yz = 0.0; break;
  }
}

// p -= lr (m / bc1) / (sqrt(v / bc2) + eps), with the bias corrections
// folded into two host-computed factors and one fast division (2 ulp).
__device__ __forceinline__ void adam_vals(float& p, float& m, float& v, float g, const AdamK& a) {
  m = fmaf(a.b1, m, a.omb1 * g);
  v = fmaf(a.b2, v, a.omb2 * g * g);
  p = fmaf(-a.step, __fdividef(m, fmaf(sqrtf(v), a.rsbc2, a.eps)), p);
}

// Fused path, stage 2, staged through shared memory: a CTA owns kThreads
// consecutive Gaussians (one per compute thread).  Each (plane, array)
// segment of p, m, v is a contiguous run of kThreads floats, moved by bulk
// asynchronous copies into a ring of kStages stages (one group of up to 4
// planes x 3 arrays each).  A producer warp fills a stage (its loads
// complete on the stage's "full" mbarrier); the 8 compute warps update it in
// place and arrive on its "empty" mbarrier; the producer then writes the
// group back with bulk stores and refills the stage once they have read it.
// Groups: the SH planes by coefficient (3 planes), then log-scale,
// quaternion, logit, and the mean last (it needs the view-direction term
// summed over the SH planes).  Every wait is bounded; on expiry the CTA
// flags GS_DEV_TIMEOUT, lets its own copies finish and exits.
#ifndef GS_ADAM_STAGES
#define GS_ADAM_STAGES 6
#endif
#ifndef GS_ADAM_CTA
#define GS_ADAM_CTA 256
#endif
constexpr int kStages = GS_ADAM_STAGES;
constexpr int kGroupPlanes = 4;
constexpr int kAT = GS_ADAM_CTA;  // Gaussians (compute threads) per CTA
constexpr int kComputeWarps = kAT / 32;

template <int D>
struct AdamGroups {
  static constexpr int KS = (D + 1) * (D + 1);
  static constexpr int N = KS + 4;
  __device__ static int first(int g) {
    return g < KS ? 11 + 3 * g : (g == KS ? 3 : g == KS + 1 ? 6 : g == KS + 2 ? 10 : 0);
  }
  __device__ static int count(int g) {
    return g < KS ? 3 : (g == KS ? 3 : g == KS + 1 ? 4 : g == KS + 2 ? 1 : 3);
  }
};

// GEO: the candidate's fp32 geometric chain runs in the compute warps'
// prologue (its inputs are the candidate's own parameters, g2d row and
// record), overlapping the first groups' loads; otherwise its results come
// from k_project_bwd_geo through g_mean / g_rest.
template <int D, bool GEO>
__global__ void __launch_bounds__(kAT + 32, 3)
k_adam_stream(float* __restrict__ P, float* __restrict__ m, float* __restrict__ v, int64_t n,
              int64_t n_pad, BwdCam cam, const int32_t* __restrict__ slot_map,
              const float4* __restrict__ rec, const float* __restrict__ g2d,
              const double* __restrict__ g_mean, const float* __restrict__ g_rest,
              int64_t n_cand, AdamK a, int32_t* dev_status) {
  using G = AdamGroups<D>;
  extern __shared__ __align__(128) float s_ring[];  // [kStages][3][kGroupPlanes][kAT]
  __shared__ unsigned long long s_full[kStages], s_empty[kStages];
  __shared__ int s_abort;
  const int t = threadIdx.x;
  const int64_t i0 = (int64_t)blockIdx.x * kAT;
  const int cnt = (int)min((int64_t)kAT, n - i0);
  const unsigned seg = (unsigned)(((cnt + 3) & ~3) * sizeof(float));  // <= n_pad - i0
  auto slot_ptr = [&](int st, int aj, int pl) {
    return s_ring + ((st * 3 + aj) * kGroupPlanes + pl) * kAT;
  };
  if (t == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&s_full[st], 1);
      mbar_init(&s_empty[st], kComputeWarps);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (t >= kAT) {  // ---- producer warp (one lane) ----
    if (t == kAT) {
      float* arr[3] = {P, m, v};
      auto issue = [&](int g) {
        const int st = g % kStages, f = G::first(g), c = G::count(g);
        mbar_arrive_expect_tx(&s_full[st], 3u * c * seg);
        for (int aj = 0; aj < 3; ++aj)
          for (int pl = 0; pl < c; ++pl)
            bulk_load(slot_ptr(st, aj, pl), arr[aj] + (int64_t)(f + pl) * n_pad + i0, seg,
                      &s_full[st]);
      };
      auto writeback = [&](int g) {
        const int st = g % kStages, f = G::first(g), c = G::count(g);
        for (int aj = 0; aj < 3; ++aj)
          for (int pl = 0; pl < c; ++pl)
            bulk_store(arr[aj] + (int64_t)(f + pl) * n_pad + i0, slot_ptr(st, aj, pl), seg);
        bulk_commit();
      };
      int issued = 0;
      for (; issued < kStages && issued < G::N; ++issued) issue(issued);
      bool ok = true;
      for (int g = 0; g < G::N && ok; ++g) {
        const int st = g % kStages;
        if (!mbar_wait(&s_empty[st], (unsigned)((g / kStages) & 1)) ||
            *(volatile int*)&s_abort) {
          ok = false;
          break;
        }
        writeback(g);
        if (issued < G::N) {
          bulk_wait_read_all();  // the stage's data have left for global memory
          issue(issued++);
        }
      }
      if (!ok) {
        *(volatile int*)&s_abort = 1;
        dev_flag(dev_status, GS_DEV_TIMEOUT);
      }
      bulk_wait_all();
      if (!ok)  // loads still in flight (the latest of each stage) must land
                // before the CTA's memory goes
        for (int h = issued > kStages ? issued - kStages : 0; h < issued; ++h)
          mbar_wait(&s_full[h % kStages], (unsigned)((h / kStages) & 1));
    }
    return;
  }

  // ---- compute warps: per-Gaussian state, read while the groups stream in
  const int64_t i = i0 + t;
  const int lane = t & 31;
  const bool in = i < n;
  const int32_t sl = in ? slot_map[i] : -1;
  const bool cand = sl >= 0;
  double gc[3] = {0.0, 0.0, 0.0};
  double dx = 0.0, dy = 0.0, dz = 0.0, dn = 1.0;
  double gm[3] = {0.0, 0.0, 0.0};
  float gr[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) gr[k] = 0.f;
  if (cand) {
    const float4 rgb = rec[3 * (int64_t)sl + 2];
    const float* g2 = g2d + 12 * (int64_t)sl;
    gc[0] = rgb.x > 0.f ? (double)g2[6] : 0.0;
    gc[1] = rgb.y > 0.f ? (double)g2[7] : 0.0;
    gc[2] = rgb.z > 0.f ? (double)g2[8] : 0.0;
    dx = (double)P[i] - cam.campos[0];
    dy = (double)P[n_pad + i] - cam.campos[1];
    dz = (double)P[2 * n_pad + i] - cam.campos[2];
    dn = sqrt(dx * dx + dy * dy + dz * dz);
    dx /= dn; dy /= dn; dz /= dn;
    if (GEO) {
      if (rgb.w >= 0.f)  // not a culled Gaussian of the dense layout
        candidate_grad<false, float>(P, n_pad, i, 0, cam, g2, make_float4(0.f, 0.f, 0.f, 0.f),
                                     [&](int plane, double gv) {
                                       if (plane < 3) gm[plane] = gv;
                                       else if (plane < 11) gr[plane - 3] = (float)gv;
                                     });
    } else {
#pragma unroll
      for (int k = 0; k < 3; ++k) gm[k] = g_mean[(int64_t)k * n_cand + sl];
#pragma unroll
      for (int k = 0; k < 8; ++k) gr[k] = g_rest[(int64_t)k * n_cand + sl];
    }
  }
  double ddx = 0.0, ddy = 0.0, ddz = 0.0;
#pragma unroll 1
  for (int g = 0; g < G::N; ++g) {
    const int st = g % kStages;
    const bool got = mbar_wait(&s_full[st], (unsigned)((g / kStages) & 1));
    if (!got || *(volatile int*)&s_abort) {
      *(volatile int*)&s_abort = 1;
      break;
    }
    if (in) {
      float* pp = slot_ptr(st, 0, 0) + t;
      float* mp = slot_ptr(st, 1, 0) + t;
      float* vp = slot_ptr(st, 2, 0) + t;
      if (g < G::KS) {
        float pv[3], mv[3], vv[3];
#pragma unroll
        for (int ch = 0; ch < 3; ++ch) {
          pv[ch] = pp[ch * kAT];
          mv[ch] = mp[ch * kAT];
          vv[ch] = vp[ch * kAT];
        }
        float gy[3] = {0.f, 0.f, 0.f};
        if (cand) {
          double Y, Yx, Yy, Yz;
          sh_term(g, dx, dy, dz, Y, Yx, Yy, Yz);
          const double w = gc[0] * pv[0] + gc[1] * pv[1] + gc[2] * pv[2];
          ddx = fma(w, Yx, ddx);
          ddy = fma(w, Yy, ddy);
          ddz = fma(w, Yz, ddz);
#pragma unroll
          for (int ch = 0; ch < 3; ++ch) gy[ch] = (float)(gc[ch] * Y);
        }
#pragma unroll
        for (int ch = 0; ch < 3; ++ch) {
          adam_vals(pv[ch], mv[ch], vv[ch], gy[ch], a);
          pp[ch * kAT] = pv[ch];
          mp[ch * kAT] = mv[ch];
          vp[ch * kAT] = vv[ch];
        }
      } else {
        const int f = G::first(g), c = G::count(g);
        float gv[4];
        if (f == 0) {  // the mean: geometric + view-direction terms
          const double ddot = ddx * dx + ddy * dy + ddz * dz;
          gv[0] = cand ? (float)(gm[0] + (ddx - dx * ddot) / dn) : 0.f;
          gv[1] = cand ? (float)(gm[1] + (ddy - dy * ddot) / dn) : 0.f;
          gv[2] = cand ? (float)(gm[2] + (ddz - dz * ddot) / dn) : 0.f;
          gv[3] = 0.f;
        } else if (f == 3) {  // log-scale
          gv[0] = gr[0]; gv[1] = gr[1]; gv[2] = gr[2]; gv[3] = 0.f;
        } else if (f == 6) {  // quaternion
          gv[0] = gr[3]; gv[1] = gr[4]; gv[2] = gr[5]; gv[3] = gr[6];
        } else {  // opacity logit
          gv[0] = gr[7]; gv[1] = gv[2] = gv[3] = 0.f;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (k >= c) break;
          float pk = pp[k * kAT], mk = mp[k * kAT], vk = vp[k * kAT];
          adam_vals(pk, mk, vk, gv[k], a);
          pp[k * kAT] = pk;
          mp[k * kAT] = mk;
          vp[k * kAT] = vk;
        }
      }
    }
    fence_proxy_async_smem();  // this thread's updates before the bulk stores
    __syncwarp();
    if (lane == 0) mbar_arrive(&s_empty[st]);
  }
}

// Dense gradient accumulation: G[plane][cand_idx[j]] += g3d[plane][j].  A
// Gaussian is at most one candidate of a projection, so no two threads add
// to one element.
__global__ void __launch_bounds__(kThreads)
k_grad_accumulate(const float* __restrict__ g3d, int64_t stride,
                  const int32_t* __restrict__ cand_idx, int64_t n_cand, int nP,
                  float* __restrict__ G, int64_t n_pad) {
  const int64_t j = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (j >= n_cand) return;
  const int64_t i = cand_idx[j];
  for (int plane = 0; plane < nP; ++plane)
    G[(int64_t)plane * n_pad + i] += g3d[(int64_t)plane * stride + j];
}

BwdCam make_cam(const gs_camera* cam) {
  BwdCam c;
  for (int k = 0; k < 9; ++k) c.R[k] = cam->R[k];
  for (int k = 0; k < 3; ++k) c.t[k] = cam->t[k];
  c.fx = cam->fx;
  c.fy = cam->fy;
  for (int k = 0; k < 3; ++k)
    c.campos[k] = -(c.R[k] * c.t[0] + c.R[3 + k] * c.t[1] + c.R[6 + k] * c.t[2]);
  return c;
}

bool make_adam(const gs_adam_args* args, AdamK* a) {
  if (!args || args->step < 1 || !(args->lr >= 0) || !(args->beta1 >= 0 && args->beta1 < 1) ||
      !(args->beta2 >= 0 && args->beta2 < 1) || !(args->eps > 0))
    return false;
  a->lr = (float)args->lr;
  a->b1 = (float)args->beta1;
  a->b2 = (float)args->beta2;
  a->omb1 = (float)(1.0 - args->beta1);
  a->omb2 = (float)(1.0 - args->beta2);
  a->eps = (float)args->eps;
  const double bc1 = 1.0 - pow(args->beta1, (double)args->step);
  const double bc2 = 1.0 - pow(args->beta2, (double)args->step);
  a->bc1 = (float)bc1;
  a->bc2 = (float)bc2;
  a->step = (float)(args->lr / bc1);
  a->rsbc2 = (float)(1.0 / sqrt(bc2));
  return true;
}

}  // namespace
}  // namespace gs

using namespace gs;

extern "C" gs_status gs_project_bwd(const gs_model* model, const gs_camera* cam,
                                    const gs_proj* proj, int64_t n_cand, const float* g2d,
                                    float* g3d, int64_t g3d_stride, float* adam_m, float* adam_v,
                                    const gs_adam_args* fused, int32_t* dev_status,
                                    gs_stream stream) {
  (void)dev_status;
  if (!model || !cam || !proj || n_cand < 0 || n_cand > proj->capacity) return GS_ERR_ARG;
  if (model->sh_degree < 0 || model->sh_degree > 3 || model->n_pad < model->n) return GS_ERR_ARG;
  if (n_cand > 0 && (!g2d || !proj->rec || !aligned(g2d, 16))) return GS_ERR_ARG;
  const BwdCam c = make_cam(cam);
  const int D = model->sh_degree;
  cudaStream_t s = to_stream(stream);
  const float4* rec = reinterpret_cast<const float4*>(proj->rec);
  if (!fused) {
    if (n_cand == 0) return GS_OK;
    if (!g3d || g3d_stride < n_cand || !proj->cand_idx) return GS_ERR_ARG;
    k_project_bwd<<<(unsigned)((n_cand + kThreads - 1) / kThreads), kThreads, 0, s>>>(
        model->params, model->n_pad, D, c, n_cand, proj->cand_idx, rec, g2d, g3d, g3d_stride);
    GS_LAUNCH_CHECK();
    return GS_OK;
  }
  AdamK a;
  if (!make_adam(fused, &a)) return GS_ERR_ARG;
  if (!adam_m || !adam_v || !proj->slot) return GS_ERR_ARG;
  if (model->n == 0) return GS_OK;
  // two-pass form: 14 floats per candidate of scratch (8-byte aligned) in g3d;
  // g3d = NULL runs the geometric chain inside the stream
  const bool two_pass = g3d != nullptr;
  if (two_pass && n_cand > 0 && (g3d_stride < 14 * n_cand || !proj->cand_idx || !aligned(g3d, 8)))
    return GS_ERR_ARG;
  double* g_mean = reinterpret_cast<double*>(g3d);
  float* g_rest = two_pass ? g3d + 6 * n_cand : nullptr;
  if (two_pass && n_cand > 0) {
    k_project_bwd_geo<<<(unsigned)((n_cand + kThreads - 1) / kThreads), kThreads, 0, s>>>(
        model->params, model->n_pad, c, n_cand, proj->cand_idx, rec, g2d, g_mean, g_rest);
    GS_LAUNCH_CHECK();
  }
  // bulk copies want 16-byte aligned segments: planes of n_pad (a multiple
  // of 4) floats, arrays 16-byte aligned
  if ((model->n_pad & 3) || !aligned(model->params, 16) || !aligned(adam_m, 16) ||
      !aligned(adam_v, 16))
    return GS_ERR_ARG;
  const size_t ring = sizeof(float) * kStages * 3 * kGroupPlanes * kAT;
  const unsigned nbs = (unsigned)((model->n + kAT - 1) / kAT);
#define GS_ADAM_FUSED2(DD, GG)                                                                \
  do {                                                                                          \
    static std::atomic<unsigned long long> done{0};                                             \
    GS_TRY(smem_attrs_once((const void*)k_adam_stream<DD, GG>, (int)ring, &done));              \
    k_adam_stream<DD, GG><<<nbs, kAT + 32, ring, s>>>(model->params, adam_m, adam_v, model->n,  \
                                                     model->n_pad, c, proj->slot, rec, g2d,     \
                                                     g_mean, g_rest, n_cand, a, dev_status);    \
  } while (0)
#define GS_ADAM_FUSED(DD)                       \
  do {                                          \
    if (two_pass) GS_ADAM_FUSED2(DD, false);    \
    else GS_ADAM_FUSED2(DD, true);              \
  } while (0)
  switch (D) {
    case 0: GS_ADAM_FUSED(0); break;
    case 1: GS_ADAM_FUSED(1); break;
    case 2: GS_ADAM_FUSED(2); break;
    default: GS_ADAM_FUSED(3); break;
  }
#undef GS_ADAM_FUSED
#undef GS_ADAM_FUSED2
  GS_LAUNCH_CHECK();
  return GS_OK;
}

extern "C" gs_status gs_adam(float* params, float* m, float* v, const float* g, int64_t g_stride,
                             const int32_t* slot, int64_t n, int64_t n_pad, int32_t P,
                             const gs_adam_args* args, gs_stream stream) {
  AdamK a;
  if (!make_adam(args, &a) || n < 0 || n_pad < n || P <= 0) return GS_ERR_ARG;
  if (n == 0) return GS_OK;
  if (!params || !m || !v || !g) return GS_ERR_ARG;
  if (!slot && g_stride < n) return GS_ERR_ARG;
  k_adam<<<(unsigned)((n + kThreads - 1) / kThreads), kThreads, 0, to_stream(stream)>>>(
      params, m, v, g, g_stride, slot, n, n_pad, P, a);
  GS_LAUNCH_CHECK();
  return GS_OK;
}

extern "C" gs_status gs_grad_accumulate(const float* g3d, int64_t g3d_stride,
                                        const int32_t* cand_idx, int64_t n_cand, int32_t P,
                                        float* G, int64_t n_pad, gs_stream stream) {
  if (n_cand < 0 || P <= 0 || n_pad < 0 || g3d_stride < n_cand) return GS_ERR_ARG;
  if (n_cand == 0) return GS_OK;
  if (!g3d || !cand_idx || !G) return GS_ERR_ARG;
  k_grad_accumulate<<<(unsigned)((n_cand + kThreads - 1) / kThreads), kThreads, 0,
                      to_stream(stream)>>>(g3d, g3d_stride, cand_idx, n_cand, P, G, n_pad);
  GS_LAUNCH_CHECK();
  return GS_OK;
}
